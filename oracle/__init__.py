"""CPU oracle for Log-linear Sparse Attention (LLSA) -- TEST INFRASTRUCTURE.

Only the test suite, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The CUDA product path never imports,
loads or calls it, and the two share no code.

The arithmetic lives in ``llsa_oracle.c`` (plain loops, fp64 accumulation);
this module only compiles it with gcc, marshals numpy arrays across ctypes
and runs independent (batch, head) slices on a thread pool.

Arrays use the same shapes as the CUDA path's public API, but per level:
  tokens   [BH, N, d] (or [batch, heads, N, d])       float64 inside
  pyramid  list over l = 1..L of [BH, n_l, d]
  indices  list over l = 1..L of [BH, n_l, K_l]        int32, rows ascending
  offsets  list over l = 1..L of [BH, n_l + 1]         int32
  qlists   list over l = 1..L of [BH, n_l * K_l]       int32

Pinning status of every routine (the tests in ``tests/test_oracle.py``):
  reorder_index / reorder   pinned: bijection, square-tile property, hand-worked table
  pool                      pinned: direct block means, raster-square means
  select                    pinned: brute-force top-K, child invariant, ties, K = all; one level =
                            block top-K by the block means
  attn_fwd                  pinned: dense softmax attention at K = all; B^l copies identity; each
                            enrichment mask against explicitly listed pooled tokens; one level
  attn_bwd                  pinned: central finite differences (also at one level); dense autograd
                            at K = all
  attn_dq_rows              pinned: equals the rows of attn_bwd's dQ
  index_transpose           pinned: exact inverse of the query-major lists
  dense_attention           pinned: torch autograd (fp64) on CPU; equals attn_fwd / attn_bwd at K = all
                            without enrichment
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, field
from math import sqrt
from typing import List, Optional, Sequence

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "llsa_oracle.c")
_LIB = os.path.join(_HERE, "_build", "liboracle.so")


def build_library(force: bool = False) -> str:
    """Compile the C oracle with gcc (IEEE arithmetic: no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        os.makedirs(os.path.dirname(_LIB), exist_ok=True)
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


class _CProblem(ctypes.Structure):
    _fields_ = [("H", ctypes.c_int), ("W", ctypes.c_int), ("d", ctypes.c_int), ("B", ctypes.c_int),
                ("L", ctypes.c_int), ("K", ctypes.c_int), ("enrich_mask", ctypes.c_uint),
                ("scale", ctypes.c_double)]


_lib = None


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build_library())
        P = ctypes.POINTER(_CProblem)
        vp = ctypes.c_void_p
        lib.oracle_levels.argtypes = [P, vp, vp]
        lib.oracle_levels.restype = ctypes.c_int
        lib.oracle_reorder_index.argtypes = [P, vp]
        lib.oracle_reorder.argtypes = [P, vp, vp, ctypes.c_int]
        lib.oracle_pool.argtypes = [P, vp, vp]
        lib.oracle_select_level.argtypes = [P, ctypes.c_int, vp, vp, vp, ctypes.c_int, vp, vp]
        lib.oracle_select.argtypes = [P, vp, vp, vp]
        lib.oracle_attn_fwd_rows.argtypes = [P, vp, vp, vp, vp, vp, vp, vp, ctypes.c_int64, vp, vp]
        lib.oracle_attn_bwd.argtypes = [P, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp]
        lib.oracle_attn_bwd_rows.argtypes = [P, vp, vp, vp, vp, vp, vp, vp, vp, ctypes.c_int64, vp, vp, vp, vp, vp]
        lib.oracle_index_transpose.argtypes = [P, vp, vp, vp]
        lib.oracle_attn_dq_rows.argtypes = [P, vp, vp, vp, vp, vp, vp, vp, vp, ctypes.c_int64, vp]
        _lib = lib
    return _lib


@dataclass
class Problem:
    """One LLSA problem: image H x W of pixel tokens, head dim d, block size B,
    L pooled levels, top-K, enriched levels (bit l-1 = level l), softmax scale."""
    H: int
    W: int
    d: int
    B: int = 16
    L: int = 2
    K: int = 8
    enrich_mask: Optional[int] = None
    scale: Optional[float] = None

    def __post_init__(self):
        if self.enrich_mask is None:
            self.enrich_mask = (1 << self.L) - 1
        if self.scale is None:
            self.scale = 1.0 / sqrt(self.d)

    @property
    def N(self) -> int:
        return self.H * self.W

    def c(self) -> _CProblem:
        return _CProblem(self.H, self.W, self.d, self.B, self.L, self.K, self.enrich_mask, float(self.scale))

    def levels(self):
        """(n[0..L], K_l[0..L]) with K_l[0] = 0."""
        n = np.zeros(self.L + 1, np.int64)
        kl = np.zeros(self.L + 1, np.int64)
        if _load().oracle_levels(ctypes.byref(self.c()), n.ctypes.data, kl.ctypes.data):
            raise ValueError("image does not tile into sqrt(B)^L squares, or bad B/L/K")
        return [int(x) for x in n], [int(x) for x in kl]


def _threads() -> int:
    return max(1, os.cpu_count() or 1)


def _as_slices(x: np.ndarray, tail: int) -> np.ndarray:
    """Flatten leading dims into BH; contiguous float64."""
    x = np.asarray(x)
    lead = x.shape[: x.ndim - tail]
    return np.ascontiguousarray(x.reshape((int(np.prod(lead)) if lead else 1,) + x.shape[x.ndim - tail:]),
                                dtype=np.float64)


def _pack(levels: Sequence[np.ndarray], s: int, dtype) -> np.ndarray:
    return np.concatenate([np.ascontiguousarray(a[s], dtype=dtype).ravel() for a in levels])


def _map(fn, count: int):
    if count == 1:
        return [fn(0)]
    with ThreadPoolExecutor(max_workers=min(_threads(), count)) as ex:
        return list(ex.map(fn, range(count)))


def reorder_index(p: Problem) -> np.ndarray:
    """hier[y*W + x] = position of pixel (y, x) in hierarchical order."""
    out = np.empty(p.N, np.int64)
    _load().oracle_reorder_index(ctypes.byref(p.c()), out.ctypes.data)
    return out


def reorder(p: Problem, x: np.ndarray, to_hier: bool) -> np.ndarray:
    shape = np.asarray(x).shape
    xs = _as_slices(x, 2)
    out = np.empty_like(xs)
    cp = p.c()
    for s in range(xs.shape[0]):
        _load().oracle_reorder(ctypes.byref(cp), xs[s].ctypes.data, out[s].ctypes.data, int(to_hier))
    return out.reshape(shape)


def pool(p: Problem, x: np.ndarray) -> List[np.ndarray]:
    """Pyramid levels 1..L of one hierarchical-order tensor."""
    n, _ = p.levels()
    xs = _as_slices(x, 2)
    BH = xs.shape[0]
    total = sum(n[l] for l in range(1, p.L + 1)) * p.d
    packed = np.empty((BH, total), np.float64)
    cp = p.c()

    def run(s):
        _load().oracle_pool(ctypes.byref(cp), xs[s].ctypes.data, packed[s].ctypes.data)

    _map(run, BH)
    out, o = [], 0
    for l in range(1, p.L + 1):
        out.append(packed[:, o:o + n[l] * p.d].reshape(BH, n[l], p.d).copy())
        o += n[l] * p.d
    return out


def _unpack_idx(p: Problem, packed: np.ndarray) -> List[np.ndarray]:
    n, kl = p.levels()
    out, o = [], 0
    for l in range(1, p.L + 1):
        out.append(packed[:, o:o + n[l] * kl[l]].reshape(-1, n[l], kl[l]).copy())
        o += n[l] * kl[l]
    return out


def select(p: Problem, pyrQ: Sequence[np.ndarray], pyrK: Sequence[np.ndarray]) -> List[np.ndarray]:
    """Index lists of every level, coarsest first (no teacher forcing)."""
    n, kl = p.levels()
    BH = pyrQ[0].shape[0]
    tot = sum(n[l] * kl[l] for l in range(1, p.L + 1))
    packed = np.zeros((BH, tot), np.int32)
    cp = p.c()

    def run(s):
        q = _pack(pyrQ, s, np.float64)
        k = _pack(pyrK, s, np.float64)
        _load().oracle_select(ctypes.byref(cp), q.ctypes.data, k.ctypes.data, packed[s].ctypes.data)

    _map(run, BH)
    return _unpack_idx(p, packed)


def select_level(p: Problem, level: int, pyrQ, pyrK, idx: Sequence[np.ndarray], R: int = 0):
    """Level ``level`` only, with the parent lists taken from ``idx`` (teacher
    forcing).  Returns (idx_l [BH, n_l, K_l], ranked_id [BH, n_l, R],
    ranked_score [BH, n_l, R])."""
    n, kl = p.levels()
    BH = pyrQ[0].shape[0]
    tot = sum(n[l] * kl[l] for l in range(1, p.L + 1))
    ids = np.full((BH, n[level], max(R, 1)), -1, np.int32)
    scs = np.full((BH, n[level], max(R, 1)), -np.inf, np.float64)
    packed = np.zeros((BH, tot), np.int32)
    cp = p.c()

    def run(s):
        q = _pack(pyrQ, s, np.float64)
        k = _pack(pyrK, s, np.float64)
        buf = _pack(idx, s, np.int32)
        _load().oracle_select_level(ctypes.byref(cp), level, q.ctypes.data, k.ctypes.data, buf.ctypes.data,
                                    R, ids[s].ctypes.data, scs[s].ctypes.data)
        packed[s] = buf

    _map(run, BH)
    return _unpack_idx(p, packed)[level - 1], ids[:, :, :R], scs[:, :, :R]


def attn_fwd(p: Problem, q, k, v, pyrK, pyrV, idx, rows: Optional[np.ndarray] = None):
    """O [BH, N, d] and LSE [BH, N] (natural log).  With ``rows`` given, only
    those query rows are computed (others are NaN)."""
    qs, ks, vs = _as_slices(q, 2), _as_slices(k, 2), _as_slices(v, 2)
    BH = qs.shape[0]
    o = np.full_like(qs, np.nan)
    lse = np.full(qs.shape[:2], np.nan)
    cp = p.c()
    r = None if rows is None else np.ascontiguousarray(rows, dtype=np.int64)

    def run(s):
        pk = _pack(pyrK, s, np.float64)
        pv = _pack(pyrV, s, np.float64)
        ix = _pack(idx, s, np.int32)
        _load().oracle_attn_fwd_rows(ctypes.byref(cp), qs[s].ctypes.data, ks[s].ctypes.data, vs[s].ctypes.data,
                                     pk.ctypes.data, pv.ctypes.data, ix.ctypes.data,
                                     None if r is None else r.ctypes.data, 0 if r is None else len(r),
                                     o[s].ctypes.data, lse[s].ctypes.data)

    _map(run, BH)
    return o, lse


def attn_bwd(p: Problem, q, k, v, pyrK, pyrV, idx, dO, rows: Optional[np.ndarray] = None):
    """(dQ, dK, dV, dPK, dPV): token gradients [BH, N, d] and the pooled-level
    gradients (lists over l = 1..L) before they are sent back to the tokens.
    With ``rows`` given only those queries contribute (a timing sample)."""
    n, _ = p.levels()
    qs, ks, vs, gs = (_as_slices(a, 2) for a in (q, k, v, dO))
    BH = qs.shape[0]
    dq, dk, dv = np.empty_like(qs), np.empty_like(qs), np.empty_like(qs)
    tot = sum(n[l] for l in range(1, p.L + 1)) * p.d
    dpk = np.empty((BH, tot))
    dpv = np.empty((BH, tot))
    cp = p.c()

    r = None if rows is None else np.ascontiguousarray(rows, dtype=np.int64)

    def run(s):
        pk = _pack(pyrK, s, np.float64)
        pv = _pack(pyrV, s, np.float64)
        ix = _pack(idx, s, np.int32)
        _load().oracle_attn_bwd_rows(ctypes.byref(cp), qs[s].ctypes.data, ks[s].ctypes.data, vs[s].ctypes.data,
                                     pk.ctypes.data, pv.ctypes.data, ix.ctypes.data, gs[s].ctypes.data,
                                     None if r is None else r.ctypes.data, 0 if r is None else len(r),
                                     dq[s].ctypes.data, dk[s].ctypes.data, dv[s].ctypes.data,
                                     dpk[s].ctypes.data, dpv[s].ctypes.data)

    _map(run, BH)
    lk, lv, o = [], [], 0
    for l in range(1, p.L + 1):
        lk.append(dpk[:, o:o + n[l] * p.d].reshape(BH, n[l], p.d))
        lv.append(dpv[:, o:o + n[l] * p.d].reshape(BH, n[l], p.d))
        o += n[l] * p.d
    return dq, dk, dv, lk, lv


def attn_dq_rows(p: Problem, q, k, v, pyrK, pyrV, idx, dO, rows: np.ndarray):
    """dQ [BH, N, d] for the listed query rows only (others NaN)."""
    qs, ks, vs, gs = (_as_slices(a, 2) for a in (q, k, v, dO))
    BH = qs.shape[0]
    dq = np.full_like(qs, np.nan)
    cp = p.c()
    r = np.ascontiguousarray(rows, dtype=np.int64)

    def run(s):
        pk = _pack(pyrK, s, np.float64)
        pv = _pack(pyrV, s, np.float64)
        ix = _pack(idx, s, np.int32)
        _load().oracle_attn_dq_rows(ctypes.byref(cp), qs[s].ctypes.data, ks[s].ctypes.data, vs[s].ctypes.data,
                                    pk.ctypes.data, pv.ctypes.data, ix.ctypes.data, gs[s].ctypes.data,
                                    r.ctypes.data, len(r), dq[s].ctypes.data)

    _map(run, BH)
    return dq


def index_transpose(p: Problem, idx: Sequence[np.ndarray]):
    """(offsets, qlists), each a list over levels."""
    n, kl = p.levels()
    BH = idx[0].shape[0]
    totq = sum(n[l] * kl[l] for l in range(1, p.L + 1))
    toto = sum(n[l] + 1 for l in range(1, p.L + 1))
    offs = np.zeros((BH, toto), np.int32)
    ql = np.zeros((BH, totq), np.int32)
    cp = p.c()

    def run(s):
        ix = _pack(idx, s, np.int32)
        _load().oracle_index_transpose(ctypes.byref(cp), ix.ctypes.data, offs[s].ctypes.data, ql[s].ctypes.data)

    _map(run, BH)
    lo, lq, a, b = [], [], 0, 0
    for l in range(1, p.L + 1):
        lo.append(offs[:, a:a + n[l] + 1].copy())
        lq.append(ql[:, b:b + n[l] * kl[l]].copy())
        a += n[l] + 1
        b += n[l] * kl[l]
    return lo, lq


def dense_attention(q, k, v, scale: float, dO=None, rows=None, keys=None, chunk: int = 1024):
    """Plain softmax attention of every query over every key of its slice, the
    closed form that LLSA reduces to when every block is selected at every
    level and no pooled token joins ("Trainable Log-linear Sparse Attention"
    summary, §一: the method restricts dense attention to the selected
    blocks).  fp64, with library matrix products and exponentials (torch CPU
    ops) over chunks of query rows; nothing else is reordered.

      z_ij = scale * q_i . k_j,  lse_i = log sum_j exp z_ij,  P_ij = exp(z_ij - lse_i)
      o_i = sum_j P_ij v_j
      dP_ij = dO_i . v_j,  D_i = dO_i . o_i,  dz_ij = P_ij (dP_ij - D_i)
      dq_i = scale * sum_j dz_ij k_j,  dk_j = scale * sum_i dz_ij q_i,  dv_j = sum_i P_ij dO_i

    q, k, v, dO: [BH, N, d].  ``rows`` (query positions, default all) selects
    the rows of o, lse and dq that are returned ([BH, len(rows), ...]);
    ``keys`` (key positions) asks for dk and dv of those keys, which need every
    query row of the slice.  Returns a dict with o, lse and, when dO is given,
    dq (and dk, dv when keys are given)."""
    import torch
    qs, ks, vs = (torch.from_numpy(_as_slices(a, 2)) for a in (q, k, v))
    gs = None if dO is None else torch.from_numpy(_as_slices(dO, 2))
    BH, N, d = qs.shape
    rows_t = torch.arange(N) if rows is None else torch.from_numpy(np.asarray(rows, dtype=np.int64))
    keys_t = None if keys is None else torch.from_numpy(np.asarray(keys, dtype=np.int64))
    out = {"o": np.empty((BH, len(rows_t), d)), "lse": np.empty((BH, len(rows_t)))}
    if gs is not None:
        out["dq"] = np.empty((BH, len(rows_t), d))
        if keys_t is not None:
            out["dk"] = np.zeros((BH, len(keys_t), d))
            out["dv"] = np.zeros((BH, len(keys_t), d))

    def block(s, r):
        z = (qs[s, r] @ ks[s].T) * scale
        lse = torch.logsumexp(z, dim=1)
        P = torch.exp(z - lse[:, None])
        o = P @ vs[s]
        return z, lse, P, o

    for s in range(BH):
        for c0 in range(0, len(rows_t), chunk):
            r = rows_t[c0:c0 + chunk]
            _, lse, P, o = block(s, r)
            out["o"][s, c0:c0 + len(r)] = o.numpy()
            out["lse"][s, c0:c0 + len(r)] = lse.numpy()
            if gs is not None:
                dP = gs[s, r] @ vs[s].T
                D = (gs[s, r] * o).sum(dim=1)
                dz = P * (dP - D[:, None])
                out["dq"][s, c0:c0 + len(r)] = (scale * (dz @ ks[s])).numpy()
        if gs is not None and keys_t is not None:
            dk = torch.zeros((len(keys_t), d), dtype=torch.float64)
            dv = torch.zeros((len(keys_t), d), dtype=torch.float64)
            for c0 in range(0, N, chunk):
                r = torch.arange(c0, min(N, c0 + chunk))
                _, lse, P, o = block(s, r)
                PJ = P[:, keys_t]
                dPJ = gs[s, r] @ vs[s, keys_t].T
                D = (gs[s, r] * o).sum(dim=1)
                dzJ = PJ * (dPJ - D[:, None])
                dk += scale * (dzJ.T @ qs[s, r])
                dv += PJ.T @ gs[s, r]
            out["dk"][s] = dk.numpy()
            out["dv"][s] = dv.numpy()
    return out


def forward(p: Problem, q_hier, k_hier, v_hier):
    """pool -> select -> attend, all in hierarchical order.
    Returns dict(pyrQ, pyrK, pyrV, idx, o, lse)."""
    pq, pk, pv = pool(p, q_hier), pool(p, k_hier), pool(p, v_hier)
    idx = select(p, pq, pk)
    o, lse = attn_fwd(p, q_hier, k_hier, v_hier, pk, pv, idx)
    return dict(pyrQ=pq, pyrK=pk, pyrV=pv, idx=idx, o=o, lse=lse)
