"""Helpers shared by the GPU parity tests: build a case from the seeded
generator, run the CUDA path through the C ABI, run the oracle, compare."""
from __future__ import annotations

from dataclasses import dataclass
from typing import List, Optional

import numpy as np

import oracle
import synthetic

# tolerances of the acceptance rule: relative Frobenius and max-abs error
TOL = {"bf16": (1e-2, 2e-2), "fp32": (1e-4, 1e-4)}
TIE_REL = 1e-4   # top-K near-tie band, relative to the larger of the two boundary scores


@dataclass
class Case:
    batch: int
    heads: int
    H: int
    W: int
    d: int = 64
    B: int = 16
    L: int = 3
    K: int = 8
    dtype: str = "bf16"
    sigma: float = 4.0
    enrich_mask: Optional[int] = None
    seed: int = 0

    def problems(self):
        from hierarchical_top_sparse_b200 import llsa
        p = llsa.Problem(batch=self.batch, heads=self.heads, height=self.H, width=self.W, d=self.d, B=self.B,
                         L=self.L, K=self.K, enrich_mask=self.enrich_mask,
                         dtype=llsa.BF16 if self.dtype == "bf16" else llsa.FP32)
        op = oracle.Problem(H=self.H, W=self.W, d=self.d, B=self.B, L=self.L, K=self.K,
                            enrich_mask=p.enrich_mask, scale=p.scale)
        return p, op

    def inputs(self):
        bf = self.dtype == "bf16"
        q, k, v = synthetic.qkv(self.seed, self.batch, self.heads, self.H, self.W, self.d, self.sigma, bf16=bf)
        g = synthetic.upstream_grad(self.seed + 1, self.batch, self.heads, self.H * self.W, self.d, bf16=bf)
        return q, k, v, g


def to_dev(x: np.ndarray, bf16: bool):
    import torch
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).cuda()
    return t.to(torch.bfloat16) if bf16 else t


def to_np(t) -> np.ndarray:
    return t.float().cpu().numpy()


def errors(got: np.ndarray, want: np.ndarray):
    got = got.astype(np.float64)
    want = want.astype(np.float64)
    rel = np.linalg.norm(got - want) / max(np.linalg.norm(want), 1e-30)
    return rel, float(np.abs(got - want).max())


def assert_close(name: str, got, want, dtype: str):
    rtol, atol = TOL[dtype]
    rel, mx = errors(got, want)
    assert rel <= rtol and mx <= atol, f"{name}: rel Frobenius {rel:.3g} (<= {rtol}), max abs {mx:.3g} (<= {atol})"
    return rel, mx


def check_level_picks(gpu_l: np.ndarray, ora_l: np.ndarray, ranked_id: np.ndarray, ranked_sc: np.ndarray, Kl: int):
    """Index lists must match exactly, except rows whose K-th and (K+1)-th oracle
    scores are a near-tie; there the two sets may differ only by candidates whose
    oracle scores sit inside the tie band.  Returns the number of tie rows."""
    diff = np.any(gpu_l != ora_l, axis=-1)
    ties = 0
    for s, a in zip(*np.nonzero(diff)):
        sc = ranked_sc[s, a]
        ids = ranked_id[s, a]
        assert len(sc) > Kl, "need the (K+1)-th score to judge a tie"
        sK, sK1 = sc[Kl - 1], sc[Kl]
        band = TIE_REL * max(abs(sK), abs(sK1))
        assert abs(sK - sK1) <= band, f"slice {s} token {a}: picks differ without a near-tie ({sK} vs {sK1})"
        score_of = dict(zip(ids.tolist(), sc.tolist()))
        for c in set(gpu_l[s, a].tolist()) ^ set(ora_l[s, a].tolist()):
            assert c in score_of and abs(score_of[c] - sK) <= band, f"slice {s} token {a}: id {c} outside the tie band"
        ties += 1
    return ties


class GpuRun:
    """Runs the CUDA path on one case and keeps every intermediate on the host."""

    def __init__(self, case: Case, backward: bool = True, hier_inputs=None):
        import torch
        from hierarchical_top_sparse_b200 import llsa
        self.case = case
        self.p, self.op = case.problems()
        bf = case.dtype == "bf16"
        if hier_inputs is None:
            q, k, v, g = case.inputs()
            hier_inputs = [oracle.reorder(self.op, x, True).astype(np.float32) for x in (q, k, v, g)]
        BH, N = case.batch * case.heads, case.H * case.W
        hier_inputs = [np.ascontiguousarray(x, dtype=np.float32).reshape(BH, N, case.d) for x in hier_inputs]
        self.qh, self.kh, self.vh, self.gh = hier_inputs
        dq_, dk_, dv_, dg_ = (to_dev(x, bf) for x in hier_inputs)
        pipe = llsa.Pipeline(self.p, backward=backward)
        pipe.forward(dq_, dk_, dv_)
        if backward:
            pipe.backward_pass(dq_, dk_, dv_, dg_)
        torch.cuda.synchronize()
        # no bounded device wait gave up during the run (reading clears the word)
        assert llsa.device_error() == 0, "a bounded device wait gave up"
        p = self.p
        self.pyrQ = [to_np(t) for t in llsa.level_views(p, pipe.pyrQ, p.d)]
        self.pyrK = [to_np(t) for t in llsa.level_views(p, pipe.pyrK, p.d)]
        self.pyrV = [to_np(t) for t in llsa.level_views(p, pipe.pyrV, p.d)]
        self.idx = [t.cpu().numpy() for t in llsa.level_views(p, pipe.idx, -1)]
        shape = (p.BH, p.N, p.d)
        self.o = to_np(pipe.o).reshape(shape)
        self.lse = to_np(pipe.lse).reshape(p.BH, p.N)
        if backward:
            self.offs = [t.cpu().numpy() for t in llsa.offs_views(p, pipe.offs)]
            self.qlist = [t.cpu().numpy().reshape(p.BH, -1) for t in llsa.level_views(p, pipe.qlist, -1)]
            self.dq = to_np(pipe.dq).reshape(shape)
            self.dk = to_np(pipe.dk).reshape(shape)
            self.dv = to_np(pipe.dv).reshape(shape)
        self.pipe = pipe


def slices(x: List[np.ndarray], sel) -> List[np.ndarray]:
    return [a[sel] for a in x]
