"""Thin Python binding of the C ABI in include/llsa.h (ctypes).

Argument marshalling only: every step runs in the CUDA kernels of
libllsa.so.  PyTorch provides device memory and streams.  There is no CPU
fallback: if the library is missing or a call fails, an exception is raised.

The functions keep the C names without the ``llsa_`` prefix and take torch
CUDA tensors (or raw device addresses as ints):

    pool(problem, x, pyramid)            select(problem, pyrQ, pyrK, idx)
    reorder(problem, x_in, x_out, to_hier)
    select_level(problem, level, pyrQ, pyrK, idx)
    attn_fwd(problem, q, k, v, pyrK, pyrV, idx, o, lse)
    index_transpose(problem, idx, offs, qlist, scratch)
    attn_bwd(problem, q, k, v, o, dO, lse, pyrK, pyrV, idx, offs, qlist, dq, dk, dv, workspace)

``Pipeline`` allocates the buffers of one problem once and runs the whole
path (pool -> select -> attend -> transpose -> backward) through these calls.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass
from math import sqrt
from typing import Optional

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libllsa.so")

BF16, FP32 = 0, 1
MAX_LEVELS = 12

STATUS = {0: "ok", 1: "invalid argument", 2: "shape", 3: "alignment", 4: "workspace", 5: "cuda error",
          6: "device wait timed out", 7: "unsupported"}

EXPORTS = ("llsa_status_string", "llsa_validate", "llsa_level_sizes", "llsa_query_sizes", "llsa_reorder",
           "llsa_pool", "llsa_select", "llsa_select_level", "llsa_attn_fwd", "llsa_index_transpose",
           "llsa_attn_bwd", "llsa_device_error", "llsa_kernel_launches", "llsa_index_transpose_noalloc",
           "llsa_selftest_wait_timeout", "llsa_attn_paths")


class LLSAError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what}: {status_string(status)} (status {status})")
        self.status = status


class CProblem(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int), ("heads", ctypes.c_int), ("height", ctypes.c_int),
                ("width", ctypes.c_int), ("d", ctypes.c_int), ("B", ctypes.c_int), ("L", ctypes.c_int),
                ("K", ctypes.c_int), ("enrich_mask", ctypes.c_uint), ("scale", ctypes.c_float),
                ("dtype", ctypes.c_int)]


class CSizes(ctypes.Structure):
    _fields_ = [(n, ctypes.c_size_t) for n in ("tokens_bytes", "lse_bytes", "pyramid_bytes", "idx_bytes",
                                                "offs_bytes", "qlist_bytes", "transpose_scratch_bytes",
                                                "bwd_workspace_bytes")]


_lib = None


def lib() -> ctypes.CDLL:
    """Loads libllsa.so (built by __graft_entry__.build() or build.py)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with `python __graft_entry__.py build` "
                               "(nvcc, sm_100a); there is no fallback path")
        L = ctypes.CDLL(LIB_PATH)
        P = ctypes.POINTER(CProblem)
        vp, i32 = ctypes.c_void_p, ctypes.c_int
        sig = {
            "llsa_status_string": ([i32], ctypes.c_char_p),
            "llsa_validate": ([P], i32),
            "llsa_level_sizes": ([P, vp, vp], i32),
            "llsa_query_sizes": ([P, ctypes.POINTER(CSizes)], i32),
            "llsa_reorder": ([P, vp, vp, i32, vp], i32),
            "llsa_pool": ([P, vp, vp, vp], i32),
            "llsa_select": ([P, vp, vp, vp, vp], i32),
            "llsa_select_level": ([P, i32, vp, vp, vp, vp], i32),
            "llsa_attn_fwd": ([P, vp, vp, vp, vp, vp, vp, vp, vp, vp], i32),
            "llsa_index_transpose": ([P, vp, vp, vp, vp, vp], i32),
            "llsa_index_transpose_noalloc": ([P, vp, vp, vp, vp], i32),
            "llsa_attn_bwd": ([P] + [vp] * 16, i32),
            "llsa_device_error": ([vp, ctypes.POINTER(i32)], i32),
            "llsa_kernel_launches": ([], ctypes.c_uint64),
            "llsa_selftest_wait_timeout": ([ctypes.c_uint, i32, i32, vp], i32),
            "llsa_attn_paths": ([P, ctypes.POINTER(i32), ctypes.POINTER(i32)], i32),
        }
        for name, (args, res) in sig.items():
            fn = getattr(L, name)
            fn.argtypes = args
            fn.restype = res
        _lib = L
    return _lib


def status_string(s: int) -> str:
    try:
        return lib().llsa_status_string(s).decode()
    except Exception:
        return STATUS.get(s, "unknown")


@dataclass
class Problem:
    """Fields of llsa_problem.  enrich_mask defaults to every level; scale to 1/sqrt(d)."""
    batch: int
    heads: int
    height: int
    width: int
    d: int = 64
    B: int = 16
    L: int = 4
    K: int = 8
    enrich_mask: Optional[int] = None
    scale: Optional[float] = None
    dtype: int = BF16

    def __post_init__(self):
        if self.enrich_mask is None:
            self.enrich_mask = (1 << self.L) - 1
        if self.scale is None:
            self.scale = 1.0 / sqrt(self.d)

    @property
    def N(self) -> int:
        return self.height * self.width

    @property
    def BH(self) -> int:
        return self.batch * self.heads

    def c(self) -> CProblem:
        return CProblem(self.batch, self.heads, self.height, self.width, self.d, self.B, self.L, self.K,
                        self.enrich_mask, float(self.scale), self.dtype)


def _ptr(x) -> Optional[int]:
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(st: int, what: str):
    if st != 0:
        raise LLSAError(st, what)


def validate(p: Problem) -> int:
    return lib().llsa_validate(ctypes.byref(p.c()))


def level_sizes(p: Problem):
    n = (ctypes.c_int64 * (p.L + 1))()
    k = (ctypes.c_int64 * (p.L + 1))()
    _check(lib().llsa_level_sizes(ctypes.byref(p.c()), ctypes.addressof(n), ctypes.addressof(k)), "level_sizes")
    return list(n), list(k)


def query_sizes(p: Problem) -> dict:
    s = CSizes()
    _check(lib().llsa_query_sizes(ctypes.byref(p.c()), ctypes.byref(s)), "query_sizes")
    return {name: getattr(s, name) for name, _ in CSizes._fields_}


def reorder(p: Problem, x_in, x_out, to_hier: bool, stream=None):
    _check(lib().llsa_reorder(ctypes.byref(p.c()), _ptr(x_in), _ptr(x_out), int(bool(to_hier)), _stream(stream)),
           "reorder")


def pool(p: Problem, x, pyramid, stream=None):
    _check(lib().llsa_pool(ctypes.byref(p.c()), _ptr(x), _ptr(pyramid), _stream(stream)), "pool")


def select(p: Problem, pyrQ, pyrK, idx, stream=None):
    _check(lib().llsa_select(ctypes.byref(p.c()), _ptr(pyrQ), _ptr(pyrK), _ptr(idx), _stream(stream)), "select")


def select_level(p: Problem, level: int, pyrQ, pyrK, idx, stream=None):
    _check(lib().llsa_select_level(ctypes.byref(p.c()), level, _ptr(pyrQ), _ptr(pyrK), _ptr(idx), _stream(stream)),
           "select_level")


def attn_fwd(p: Problem, q, k, v, pyrK, pyrV, idx, o, lse, stream=None):
    _check(lib().llsa_attn_fwd(ctypes.byref(p.c()), _ptr(q), _ptr(k), _ptr(v), _ptr(pyrK), _ptr(pyrV), _ptr(idx),
                               _ptr(o), _ptr(lse), _stream(stream)), "attn_fwd")


def index_transpose(p: Problem, idx, offs, qlist, scratch, stream=None):
    _check(lib().llsa_index_transpose(ctypes.byref(p.c()), _ptr(idx), _ptr(offs), _ptr(qlist), _ptr(scratch),
                                      _stream(stream)), "index_transpose")


def index_transpose_noalloc(p: Problem, idx, offs, qlist, stream=None):
    """index_transpose with the library's own fixed scratch array: for callers
    that cannot allocate device memory.  Calls whose GPU work overlaps share
    that array and must be serialized."""
    _check(lib().llsa_index_transpose_noalloc(ctypes.byref(p.c()), _ptr(idx), _ptr(offs), _ptr(qlist),
                                              _stream(stream)), "index_transpose_noalloc")


def attn_bwd(p: Problem, q, k, v, o, dO, lse, pyrK, pyrV, idx, offs, qlist, dq, dk, dv, workspace, stream=None):
    _check(lib().llsa_attn_bwd(ctypes.byref(p.c()), *[_ptr(t) for t in (q, k, v, o, dO, lse, pyrK, pyrV, idx, offs,
                                                                          qlist, dq, dk, dv, workspace)],
                               _stream(stream)), "attn_bwd")


def attn_paths(p: Problem) -> dict:
    """Which kernels attn_fwd / attn_bwd run for p: "tensor" or "cuda-core"."""
    f, b = ctypes.c_int(0), ctypes.c_int(0)
    _check(lib().llsa_attn_paths(ctypes.byref(p.c()), ctypes.byref(f), ctypes.byref(b)), "attn_paths")
    name = {1: "tensor", 0: "cuda-core"}
    return {"fwd": name[f.value], "bwd": name[b.value]}


def kernel_launches() -> int:
    """Kernels launched by libllsa.so in this process so far."""
    return int(lib().llsa_kernel_launches())


def device_error(stream=None) -> int:
    code = ctypes.c_int(0)
    st = lib().llsa_device_error(_stream(stream), ctypes.byref(code))
    if st not in (0, 6):
        raise LLSAError(st, "device_error")
    return code.value


def selftest_wait_timeout(limit_us: int, code: int, arrive: bool = False, stream=None):
    """Launches the timeout-path self-test (llsa_selftest_wait_timeout)."""
    _check(lib().llsa_selftest_wait_timeout(int(limit_us), int(code), int(bool(arrive)), _stream(stream)),
           "selftest_wait_timeout")


# ------------------------------------------------------------------ layouts

def level_views(p: Problem, buf, per_token: int):
    """Per-level views [BH, n_l, per_token] of a level-packed buffer (per_token = d
    for pyramids, or -1 to use K_l for index lists)."""
    n, kl = level_sizes(p)
    out, o = [], 0
    for l in range(1, p.L + 1):
        w = kl[l] if per_token < 0 else per_token
        cnt = p.BH * n[l] * w
        out.append(buf[o:o + cnt].view(p.BH, n[l], w))
        o += cnt
    return out


def offs_views(p: Problem, buf):
    n, _ = level_sizes(p)
    out, o = [], 0
    for l in range(1, p.L + 1):
        cnt = p.BH * (n[l] + 1)
        out.append(buf[o:o + cnt].view(p.BH, n[l] + 1))
        o += cnt
    return out


class Pipeline:
    """Device buffers of one problem, allocated once, and the path run through the C ABI."""

    def __init__(self, p: Problem, device="cuda", backward: bool = True):
        import torch
        self.p = p
        _check(validate(p), "validate")
        self.sizes = query_sizes(p)
        self.n, self.Kl = level_sizes(p)
        dt = torch.bfloat16 if p.dtype == BF16 else torch.float32
        shape = (p.batch, p.heads, p.N, p.d)
        f32 = torch.float32
        nel_pyr = self.sizes["pyramid_bytes"] // 4
        self.pyrQ = torch.empty(nel_pyr, dtype=f32, device=device)
        self.pyrK = torch.empty(nel_pyr, dtype=f32, device=device)
        self.pyrV = torch.empty(nel_pyr, dtype=f32, device=device)
        self.idx = torch.empty(self.sizes["idx_bytes"] // 4, dtype=torch.int32, device=device)
        self.o = torch.empty(shape, dtype=dt, device=device)
        self.lse = torch.empty((p.batch, p.heads, p.N), dtype=f32, device=device)
        self.backward = backward
        if backward:
            self.offs = torch.empty(self.sizes["offs_bytes"] // 4, dtype=torch.int32, device=device)
            self.qlist = torch.empty(self.sizes["qlist_bytes"] // 4, dtype=torch.int32, device=device)
            self.tscratch = torch.empty(self.sizes["transpose_scratch_bytes"], dtype=torch.uint8, device=device)
            self.work = torch.empty(self.sizes["bwd_workspace_bytes"], dtype=torch.uint8, device=device)
            self.dq = torch.empty(shape, dtype=dt, device=device)
            self.dk = torch.empty(shape, dtype=dt, device=device)
            self.dv = torch.empty(shape, dtype=dt, device=device)

    def forward(self, q, k, v, stream=None):
        p = self.p
        pool(p, q, self.pyrQ, stream)
        pool(p, k, self.pyrK, stream)
        pool(p, v, self.pyrV, stream)
        select(p, self.pyrQ, self.pyrK, self.idx, stream)
        attn_fwd(p, q, k, v, self.pyrK, self.pyrV, self.idx, self.o, self.lse, stream)
        return self.o, self.lse

    def backward_pass(self, q, k, v, dO, stream=None):
        p = self.p
        index_transpose(p, self.idx, self.offs, self.qlist, self.tscratch, stream)
        attn_bwd(p, q, k, v, self.o, dO, self.lse, self.pyrK, self.pyrV, self.idx, self.offs, self.qlist,
                 self.dq, self.dk, self.dv, self.work, stream)
        return self.dq, self.dk, self.dv

    def step(self, q, k, v, dO=None, stream=None):
        """One pass of the whole path; backward too when dO is given."""
        self.forward(q, k, v, stream)
        if dO is not None:
            self.backward_pass(q, k, v, dO, stream)
