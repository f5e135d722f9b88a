"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle on the
same seeded inputs.

* reorder, pyramids: exact / fp32 rounding only;
* index lists: bit-exact per level with the oracle fed the GPU's parent lists,
  except near-ties (K-th and (K+1)-th oracle scores within 1e-4 relative);
* CSC lists: bit-exact against the oracle's transpose of the GPU's lists;
* O, LSE, dQ, dK, dV: relative Frobenius <= 1e-2 and max-abs <= 2e-2 for bf16
  (1e-4 for fp32), with the oracle fed the GPU's index lists, and end to end on
  every row whose lists the oracle selected identically.
"""
import numpy as np
import pytest

import oracle
import synthetic
from parity_util import Case, GpuRun, assert_close, check_level_picks, errors, to_dev, to_np

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from hierarchical_top_sparse_b200 import llsa
    llsa.lib()


def check_selection(run: GpuRun):
    """Level by level, coarsest first, the oracle fed the GPU's parent lists."""
    op = run.op
    n, kl = op.levels()
    pq, pk = oracle.pool(op, run.qh), oracle.pool(op, run.kh)
    ties = 0
    for l in range(op.L, 0, -1):
        want, rid, rsc = oracle.select_level(op, l, pq, pk, run.idx, R=kl[l] + 4)
        got = run.idx[l - 1]
        assert got.shape == want.shape
        assert np.all(np.diff(got, axis=-1) > 0), f"level {l}: lists not strictly ascending"
        if kl[l] < rsc.shape[-1]:
            ties += check_level_picks(got, want, rid, rsc, kl[l])
        else:
            np.testing.assert_array_equal(got, want)
    return ties


def check_pyramids(run: GpuRun):
    op = run.op
    for name, src, got in (("Q", run.qh, run.pyrQ), ("K", run.kh, run.pyrK), ("V", run.vh, run.pyrV)):
        want = oracle.pool(op, src)
        for l in range(op.L):
            np.testing.assert_allclose(got[l], want[l], rtol=2e-6, atol=2e-6, err_msg=f"pyramid {name} level {l + 1}")


def check_transpose(run: GpuRun):
    offs, ql = oracle.index_transpose(run.op, run.idx)
    for l in range(run.op.L):
        np.testing.assert_array_equal(run.offs[l], offs[l], err_msg=f"offsets level {l + 1}")
        np.testing.assert_array_equal(run.qlist[l], ql[l], err_msg=f"query lists level {l + 1}")


def check_attention(run: GpuRun, backward: bool, sel=slice(None)):
    """Teacher-forced: the oracle attends with the GPU's index lists."""
    op, dt = run.op, run.case.dtype
    idx = [a[sel] for a in run.idx]
    pk, pv = oracle.pool(op, run.kh[sel]), oracle.pool(op, run.vh[sel])
    o, lse = oracle.attn_fwd(op, run.qh[sel], run.kh[sel], run.vh[sel], pk, pv, idx)
    res = {"o": assert_close("O", run.o[sel], o, dt), "lse": assert_close("LSE", run.lse[sel], lse, dt)}
    if backward:
        dq, dk, dv, _, _ = oracle.attn_bwd(op, run.qh[sel], run.kh[sel], run.vh[sel], pk, pv, idx, run.gh[sel])
        res["dq"] = assert_close("dQ", run.dq[sel], dq, dt)
        res["dk"] = assert_close("dK", run.dk[sel], dk, dt)
        res["dv"] = assert_close("dV", run.dv[sel], dv, dt)
    return res


def agreeing_rows(op, gpu_idx, ora_idx):
    """[BH, N] bool: fine rows whose lists (every level's list of every one of
    their ancestors) are identical in the two selections."""
    n, _ = op.levels()
    same = np.ones((gpu_idx[0].shape[0], n[0]), bool)
    for l in range(1, op.L + 1):
        eq = np.all(gpu_idx[l - 1] == ora_idx[l - 1], axis=-1)          # [BH, n_l]
        same &= np.repeat(eq, op.B ** l, axis=1)
    return same


def agreeing_keys(op, gpu_idx, ora_idx, same):
    """[BH, N] bool: fine keys whose gradient is formed by the same query rows,
    all of them agreeing rows, in both selections: no query token with a
    disagreeing row picked the key's block (level 1), nor, for every enriched
    level l >= 2, the key's level-l ancestor, in either selection."""
    n, _ = op.levels()
    BH, N = same.shape
    ok = np.ones((BH, N), bool)
    for l in range(1, op.L + 1):
        if l > 1 and not (op.enrich_mask >> (l - 1)) & 1:
            continue
        rowok = same.reshape(BH, n[l], op.B ** l).all(axis=2)          # [BH, n_l] query tokens
        bad = np.zeros((BH, n[l]), bool)
        for s, a in zip(*np.nonzero(~rowok)):
            for lists in (gpu_idx, ora_idx):
                u = lists[l - 1][s, a]
                bad[s, u[(u >= 0) & (u < n[l])]] = True
        ok &= ~np.repeat(bad, op.B ** l, axis=1)
    return ok


def check_end_to_end(run: GpuRun, sel=slice(None), min_match=0.99, grads=True):
    """The oracle's own selection, forward and backward: rows whose lists all
    agree must agree in O and dQ; keys whose gradients are formed by agreeing
    rows only must agree in dK and dV."""
    op, dt = run.op, run.case.dtype
    qh, kh, vh = run.qh[sel], run.kh[sel], run.vh[sel]
    r = oracle.forward(op, qh, kh, vh)
    gpu_idx = [a[sel] for a in run.idx]
    same = agreeing_rows(op, gpu_idx, r["idx"])
    frac = same.mean()
    assert frac >= min_match, f"only {frac:.4f} of the rows have identical index lists"
    assert_close("O (end to end)", run.o[sel][same], r["o"][same], dt)
    assert_close("LSE (end to end)", run.lse[sel][same], r["lse"][same], dt)
    if grads:
        dq, dk, dv, _, _ = oracle.attn_bwd(op, qh, kh, vh, r["pyrK"], r["pyrV"], r["idx"], run.gh[sel])
        kok = agreeing_keys(op, gpu_idx, r["idx"], same)
        assert kok.mean() >= min_match - 0.05, f"only {kok.mean():.4f} of the keys are formed by agreeing rows"
        assert_close("dQ (end to end)", run.dq[sel][same], dq[same], dt)
        assert_close("dK (end to end)", run.dk[sel][kok], dk[kok], dt)
        assert_close("dV (end to end)", run.dv[sel][kok], dv[kok], dt)
    return frac


CASES = {
    # the smallest workload: 32 x 32 pixels, fp32, B = 16, L = 2, K = 4
    "tiny32_fp32": Case(batch=1, heads=1, H=32, W=32, L=2, K=4, dtype="fp32"),
    "px64_bf16": Case(batch=2, heads=2, H=64, W=64, L=3, K=8),
    "px64_fp32_E2": Case(batch=1, heads=2, H=64, W=64, L=3, K=8, dtype="fp32", enrich_mask=0b010),
    "px64_noenrich": Case(batch=1, heads=2, H=64, W=64, L=2, K=6, enrich_mask=0),
    "single_level": Case(batch=1, heads=2, H=64, W=64, L=1, K=8),
    "B4": Case(batch=1, heads=2, H=32, W=32, B=4, L=3, K=6, dtype="fp32"),
    "B64": Case(batch=1, heads=2, H=64, W=64, B=64, L=2, K=3, d=32),
    "d128_ragged_K": Case(batch=1, heads=1, H=64, W=48, L=2, K=5, d=128),
    # tensor-core forward: level 1 not enriched; K = 16 (unions larger than the slot ring)
    "px64_E23": Case(batch=2, heads=1, H=64, W=64, L=3, K=8, enrich_mask=0b110),
    "px64_K16": Case(batch=1, heads=2, H=64, W=64, L=3, K=16),
}


@pytest.mark.parametrize("name", sorted(CASES))
def test_small_cases_full_parity(name):
    case = CASES[name]
    run = GpuRun(case)
    check_pyramids(run)
    check_selection(run)
    check_transpose(run)
    check_attention(run, backward=True)
    check_end_to_end(run, min_match=0.98)


def test_reorder_roundtrip_is_exact():
    case = Case(batch=1, heads=3, H=64, W=32, L=2)
    from hierarchical_top_sparse_b200 import llsa
    p, op = case.problems()
    q, _, _, _ = case.inputs()
    x = to_dev(q, True)
    y = torch.empty_like(x)
    z = torch.empty_like(x)
    llsa.reorder(p, x, y, True)
    llsa.reorder(p, y, z, False)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(to_np(y), oracle.reorder(op, q, True).astype(np.float32))
    assert torch.equal(x, z)
    p32 = llsa.Problem(batch=1, heads=3, height=64, width=32, L=2, dtype=llsa.FP32)
    x32 = torch.from_numpy(q).cuda()
    y32 = torch.empty_like(x32)
    llsa.reorder(p32, x32, y32, True)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(y32.cpu().numpy(), oracle.reorder(op, q, True).astype(np.float32))


def test_dense_when_k_covers_everything():
    # K >= every candidate count and no enrichment: plain softmax attention
    case = Case(batch=1, heads=1, H=32, W=32, L=2, K=10 ** 6, dtype="fp32", enrich_mask=0)
    run = GpuRun(case)
    q, k, v = run.qh[0], run.kh[0], run.vh[0]
    S = (q.astype(np.float64) @ k.T.astype(np.float64)) * run.p.scale
    P = np.exp(S - S.max(1, keepdims=True))
    o = (P / P.sum(1, keepdims=True)) @ v
    assert_close("O dense", run.o[0], o, "fp32")
    check_attention(run, backward=True)
    check_transpose(run)


def check_selects_everything(run: GpuRun):
    """K at least every candidate count: every list holds every token of its level."""
    n, kl = run.op.levels()
    for l in range(1, run.op.L + 1):
        assert kl[l] == n[l]
        got = run.idx[l - 1]
        np.testing.assert_array_equal(got, np.broadcast_to(np.arange(n[l], dtype=np.int32), got.shape))


# bf16 K = all without enrichment, through the tensor-core kernels: every
# level-1 list holds every block, so the backward's unions span the whole
# slice (256 and 1024 blocks); compared with dense softmax attention
DENSE_BF16 = {
    "px64_dense": Case(batch=1, heads=2, H=64, W=64, L=3, K=10 ** 6, enrich_mask=0),
    "px128_dense": Case(batch=1, heads=2, H=128, W=128, L=3, K=10 ** 6, enrich_mask=0),
}


@pytest.mark.parametrize("name", sorted(DENSE_BF16))
def test_dense_bf16_on_the_tensor_cores(name):
    from hierarchical_top_sparse_b200 import llsa
    case = DENSE_BF16[name]
    p, _ = case.problems()
    assert llsa.attn_paths(p) == {"fwd": "tensor", "bwd": "tensor"}
    run = GpuRun(case)
    check_selects_everything(run)
    check_transpose(run)
    N = case.H * case.W
    ref = oracle.dense_attention(run.qh, run.kh, run.vh, run.p.scale, dO=run.gh, keys=np.arange(N))
    assert_close("O dense", run.o, ref["o"], "bf16")
    assert_close("LSE dense", run.lse, ref["lse"], "bf16")
    assert_close("dQ dense", run.dq, ref["dq"], "bf16")
    assert_close("dK dense", run.dk, ref["dk"], "bf16")
    assert_close("dV dense", run.dv, ref["dv"], "bf16")
    if case.H == 64:   # and the loop oracle, fed the (complete) lists
        check_attention(run, backward=True)


def test_dense_bf16_full_size_sampled():
    """The 256 x 256 workload with K = all and no enrichment against dense
    attention: O, LSE and dQ on 256 seeded rows of every slice, dK and dV on
    256 seeded keys of the first slice, the gradient sums on every slice."""
    from hierarchical_top_sparse_b200 import llsa
    c = synthetic.CONFIGS["px256"]
    case = Case(batch=c["batch"], heads=c["heads"], H=c["H"], W=c["W"], L=c["L"], K=10 ** 6, sigma=c["sigma"],
                enrich_mask=0)
    p, op = case.problems()
    assert llsa.attn_paths(p) == {"fwd": "tensor", "bwd": "tensor"}
    run = GpuRun(case)
    check_selects_everything(run)
    rows = sampled_rows(op.N, 256, 5)
    ref = oracle.dense_attention(run.qh, run.kh, run.vh, run.p.scale, dO=run.gh, rows=rows)
    assert_close("O dense rows", run.o[:, rows], ref["o"], "bf16")
    assert_close("LSE dense rows", run.lse[:, rows], ref["lse"], "bf16")
    assert_close("dQ dense rows", run.dq[:, rows], ref["dq"], "bf16")
    keys = sampled_rows(op.N, 256, 6)
    ref0 = oracle.dense_attention(run.qh[:1], run.kh[:1], run.vh[:1], run.p.scale, dO=run.gh[:1], rows=rows[:8],
                                  keys=keys)
    assert_close("dK dense keys", run.dk[:1, keys], ref0["dk"], "bf16")
    assert_close("dV dense keys", run.dv[:1, keys], ref0["dv"], "bf16")
    check_gradient_sums(run)


def test_select_and_transpose_are_deterministic():
    case = Case(batch=2, heads=2, H=64, W=64, L=3, K=8)
    a, b = GpuRun(case), GpuRun(case)
    for l in range(3):
        np.testing.assert_array_equal(a.idx[l], b.idx[l])
        np.testing.assert_array_equal(a.qlist[l], b.qlist[l])


@pytest.mark.parametrize("cfg", ["px128", "px128_fwd"])
def test_workload_128(cfg):
    c = synthetic.CONFIGS[cfg]
    case = Case(batch=c["batch"], heads=c["heads"], H=c["H"], W=c["W"], L=c["L"], K=c["K"], sigma=c["sigma"])
    run = GpuRun(case, backward=c["backward"])
    check_pyramids(run)
    ties = check_selection(run)
    if c["backward"]:
        check_transpose(run)
    check_attention(run, backward=c["backward"])
    check_end_to_end(run, grads=c["backward"])
    print(f"{cfg}: {ties} near-tie rows")


def sampled_rows(N, count, seed):
    rng = np.random.default_rng(seed)
    return np.sort(rng.choice(N, size=count, replace=False))


@pytest.mark.parametrize("cfg,full_slices", [("px256", (0, 7)), ("px512", (0,))])
def test_workload_full_size(cfg, full_slices):
    """The full-size workloads in the launch configuration the benchmark times:
    every selection level and the transposes in full, O / LSE / dQ on sampled
    rows of every slice, dK / dV of whole slices where the oracle finishes in
    seconds, and the gradient-sum identities everywhere."""
    c = synthetic.CONFIGS[cfg]
    case = Case(batch=c["batch"], heads=c["heads"], H=c["H"], W=c["W"], L=c["L"], K=c["K"], sigma=c["sigma"])
    run = GpuRun(case, backward=True)
    op = run.op
    check_pyramids(run)
    check_selection(run)
    check_transpose(run)
    rows = sampled_rows(op.N, 512, 3)
    pk, pv = oracle.pool(op, run.kh), oracle.pool(op, run.vh)
    o, lse = oracle.attn_fwd(op, run.qh, run.kh, run.vh, pk, pv, run.idx, rows=rows)
    assert_close("O rows", run.o[:, rows], o[:, rows], "bf16")
    assert_close("LSE rows", run.lse[:, rows], lse[:, rows], "bf16")
    dq = oracle.attn_dq_rows(op, run.qh, run.kh, run.vh, pk, pv, run.idx, run.gh, rows)
    assert_close("dQ rows", run.dq[:, rows], dq[:, rows], "bf16")
    check_gradient_sums(run)
    for s in full_slices:
        check_attention(run, backward=True, sel=slice(s, s + 1))
    # end to end (the oracle's own selection): O and LSE on every slice, the
    # gradients on the first
    check_end_to_end(run, grads=False)
    check_end_to_end(run, sel=slice(0, 1))


def check_gradient_sums(run: GpuRun):
    # every row's softmax weights sum to one and its dS to zero: sum_t dV_t =
    # sum_i dO_i and sum_t dK_t = 0, per slice and channel
    sv = run.dv.astype(np.float64).sum(axis=1)
    np.testing.assert_allclose(sv, run.gh.astype(np.float64).sum(axis=1), rtol=0, atol=0.5 + 2e-3 * np.abs(sv).max())
    sk = run.dk.astype(np.float64).sum(axis=1)
    scale_k = np.abs(run.dk).sum(axis=1)
    assert np.all(np.abs(sk) <= 2e-2 * scale_k + 1e-3), "sum of dK is not ~0"


@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
def test_level1_pyramid_contract(dtype):
    """Level 1 of pyrK / pyrV must be llsa_pool's output for the same K / V.
    The tensor-core kernels (bf16, d = 64, B = 16) derive level-1 pooled
    tokens from K and V and never read that level: a perturbed level 1 leaves
    every output bit unchanged.  The CUDA-core kernels (fp32 here) read it:
    their outputs follow the oracle fed the perturbed pyramid."""
    from hierarchical_top_sparse_b200 import llsa
    case = Case(batch=1, heads=2, H=64, W=64, L=3, K=8, dtype=dtype)
    p, op = case.problems()
    tc = llsa.attn_paths(p)
    assert tc == ({"fwd": "tensor", "bwd": "tensor"} if dtype == "bf16" else {"fwd": "cuda-core", "bwd": "cuda-core"})
    base = GpuRun(case)
    pipe = base.pipe
    qd, kd, vd, gd = (to_dev(x, dtype == "bf16") for x in (base.qh, base.kh, base.vh, base.gh))
    lvK = llsa.level_views(p, pipe.pyrK, p.d)[0]
    lvV = llsa.level_views(p, pipe.pyrV, p.d)[0]
    gen = torch.Generator(device="cuda").manual_seed(9)
    lvK.add_(0.5 * torch.randn(lvK.shape, device="cuda", generator=gen))
    lvV.add_(0.5 * torch.randn(lvV.shape, device="cuda", generator=gen))
    o = torch.empty_like(pipe.o)
    lse = torch.empty_like(pipe.lse)
    llsa.attn_fwd(p, qd, kd, vd, pipe.pyrK, pipe.pyrV, pipe.idx, o, lse)
    dq, dk, dv = torch.empty_like(pipe.dq), torch.empty_like(pipe.dk), torch.empty_like(pipe.dv)
    llsa.attn_bwd(p, qd, kd, vd, o, gd, lse, pipe.pyrK, pipe.pyrV, pipe.idx, pipe.offs, pipe.qlist, dq, dk, dv,
                  pipe.work)
    torch.cuda.synchronize()
    assert llsa.device_error() == 0
    shape = (p.BH, p.N, p.d)
    got = {"o": to_np(o).reshape(shape), "lse": to_np(lse).reshape(p.BH, p.N), "dq": to_np(dq).reshape(shape),
           "dk": to_np(dk).reshape(shape), "dv": to_np(dv).reshape(shape)}
    if dtype == "bf16":
        # O, LSE and dQ are deterministic: bit for bit.  dK and dV add the
        # pooled-key gradients, summed with fp32 atomics in arbitrary order:
        # within one bf16 rounding step of the unperturbed run (the 0.5
        # perturbation would move them by far more if level 1 were read).
        for name in ("o", "lse", "dq"):
            np.testing.assert_array_equal(got[name], getattr(base, name), err_msg=f"{name} read level 1")
        for name in ("dk", "dv"):
            ref = getattr(base, name)
            assert np.all(np.abs(got[name] - ref) <= 2.0 ** -7 * np.abs(ref) + 1e-6), f"{name} read level 1"
        return
    pk = [t.cpu().numpy().astype(np.float64) for t in llsa.level_views(p, pipe.pyrK, p.d)]
    pv = [t.cpu().numpy().astype(np.float64) for t in llsa.level_views(p, pipe.pyrV, p.d)]
    ro, rlse = oracle.attn_fwd(op, base.qh, base.kh, base.vh, pk, pv, base.idx)
    rdq, rdk, rdv, _, _ = oracle.attn_bwd(op, base.qh, base.kh, base.vh, pk, pv, base.idx, base.gh)
    assert errors(got["o"], base.o)[0] > 1e-3, "the perturbation did not reach the output"
    for name, want in (("o", ro), ("lse", rlse), ("dq", rdq), ("dk", rdk), ("dv", rdv)):
        assert_close(name + " (perturbed level 1)", got[name], want, dtype)
