"""The C ABI without a GPU: the library loads, exports every declared entry
point, and rejects bad problems and buffers on the host before any launch."""
import ctypes
import os
import re

import pytest

import oracle
from hierarchical_top_sparse_b200 import llsa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    if not os.path.exists(llsa.LIB_PATH):
        import __graft_entry__
        __graft_entry__.build()
    return llsa.lib()


def declared_symbols():
    text = open(os.path.join(ROOT, "include", "llsa.h")).read()
    return sorted(set(re.findall(r"\b(llsa_[a-z_0-9]+)\s*\(", text)))


def test_every_declared_symbol_is_exported(L):
    names = declared_symbols()
    assert "llsa_attn_fwd" in names and "llsa_index_transpose" in names
    for n in names:
        assert hasattr(L, n), n
    assert set(llsa.EXPORTS) <= set(names)


def px256(**kw):
    base = dict(batch=2, heads=6, height=256, width=256, d=64, B=16, L=4, K=8)
    base.update(kw)
    return llsa.Problem(**base)


def test_level_sizes_agree_with_the_oracle(L):
    for kw in (dict(), dict(height=128, width=128, L=3, batch=8), dict(K=10 ** 6), dict(B=4, L=3, height=64, width=64)):
        p = px256(**kw)
        n, kl = llsa.level_sizes(p)
        on, okl = oracle.Problem(H=p.height, W=p.width, d=p.d, B=p.B, L=p.L, K=p.K).levels()
        assert n == on and kl == okl


def test_query_sizes(L):
    p = px256()
    s = llsa.query_sizes(p)
    assert s["tokens_bytes"] == 2 * 6 * 65536 * 64 * 2
    assert s["lse_bytes"] == 2 * 6 * 65536 * 4
    assert s["pyramid_bytes"] == 12 * (4096 + 256 + 16 + 1) * 64 * 4
    assert s["idx_bytes"] == 12 * (4096 * 8 + 256 * 8 + 16 * 8 + 1 * 1) * 4
    assert s["offs_bytes"] == 12 * (4097 + 257 + 17 + 2) * 4
    assert s["qlist_bytes"] == s["idx_bytes"]
    p32 = px256(dtype=llsa.FP32)
    assert llsa.query_sizes(p32)["tokens_bytes"] == 2 * s["tokens_bytes"]


@pytest.mark.parametrize("kw,status", [
    (dict(height=250), 2),            # does not tile into 4^4 squares
    (dict(B=15), 1),                  # not a perfect square
    (dict(B=9), 7),                   # square, but not a supported block size
    (dict(d=60), 7),
    (dict(d=256), 7),
    (dict(K=0), 1),
    (dict(L=0), 1),
    (dict(L=13), 7),
    (dict(enrich_mask=1 << 4), 1),    # level 5 does not exist
    (dict(batch=0), 1),
    (dict(dtype=5), 1),
    (dict(scale=-1.0), 1),
])
def test_validation_errors(L, kw, status):
    assert llsa.validate(px256(**kw)) == status


def test_valid_problems(L):
    for kw in (dict(), dict(K=1), dict(K=10 ** 6, enrich_mask=0), dict(B=64, L=2), dict(B=4, L=4, height=64, width=64),
               dict(L=1, K=32), dict(dtype=llsa.FP32, d=128)):
        assert llsa.validate(px256(**kw)) == 0, kw


def test_entry_points_reject_null_and_misaligned_buffers_before_launch(L):
    p = px256().c()
    good = 1 << 20          # never dereferenced: the calls must return before any launch
    bad = good + 4
    assert L.llsa_pool(ctypes.byref(p), None, good, None) == 1
    assert L.llsa_pool(ctypes.byref(p), bad, good, None) == 3
    assert L.llsa_select(ctypes.byref(p), good, good, None, None) == 1
    assert L.llsa_select_level(ctypes.byref(p), 0, good, good, good, None) == 1
    assert L.llsa_select_level(ctypes.byref(p), 5, good, good, good, None) == 1
    assert L.llsa_attn_fwd(ctypes.byref(p), good, good, good, good, good, good, good, bad, None) == 3
    assert L.llsa_index_transpose(ctypes.byref(p), good, good, good, None, None) == 1
    args = [good] * 15
    args[14] = None
    assert L.llsa_attn_bwd(ctypes.byref(p), *args, None) == 1
    assert L.llsa_reorder(ctypes.byref(p), good, good, 1, None) == 1      # in == out overlaps
    bad_p = px256(height=250).c()
    assert L.llsa_pool(ctypes.byref(bad_p), good, good, None) == 2


def test_timeout_selftest_rejects_bad_arguments_before_launch(L):
    # limit_us in [1, 1e6], code != 0, arrive in {0, 1}: LLSA_ERR_ARG, no CUDA call
    for args in ((0, 5, 0), (1000001, 5, 0), (10, 0, 0), (10, 5, 2), (10, 5, -1)):
        assert L.llsa_selftest_wait_timeout(*args, None) == 1, args


def test_status_strings(L):
    for s in range(8):
        assert llsa.status_string(s)


@pytest.mark.parametrize("kw, fwd, bwd", [
    # the metric's workload, and K = all at 256^2 (K_1 = 4096): tensor cores
    (dict(batch=2, heads=6, height=256, width=256, L=4, K=8), "tensor", "tensor"),
    (dict(batch=2, heads=6, height=256, width=256, L=1, K=10 ** 6, enrich_mask=0), "tensor", "tensor"),
    # K = all at 512^2 (K_1 = 16384): above the tensor-core list limit
    (dict(batch=1, heads=1, height=512, width=512, L=1, K=10 ** 6, enrich_mask=0), "cuda-core", "cuda-core"),
    # fp32, B = 64 and d = 128 run on the CUDA cores
    (dict(batch=1, heads=2, height=64, width=64, L=3, K=8, dtype=llsa.FP32), "cuda-core", "cuda-core"),
    (dict(batch=1, heads=2, height=64, width=64, B=64, L=1, K=8), "cuda-core", "cuda-core"),
    (dict(batch=1, heads=2, height=64, width=64, d=128, L=3, K=8), "cuda-core", "cuda-core"),
    # more than 32 pooled keys of levels >= 2 per query block
    (dict(batch=1, heads=1, height=256, width=256, L=4, K=16), "cuda-core", "cuda-core"),
])
def test_attention_dispatch(L, kw, fwd, bwd):
    """llsa_attn_paths (host only) reports the kernels the problem runs on."""
    base = dict(d=64, B=16)
    base.update(kw)
    p = llsa.Problem(**base)
    assert llsa.validate(p) == 0
    assert llsa.attn_paths(p) == {"fwd": fwd, "bwd": bwd}
