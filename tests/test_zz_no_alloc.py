"""The transpose entry point that takes no scratch buffer.

Some callers cannot allocate device memory where they run the transpose (a
plug-in whose host framework owns all device allocations, or a loop that must
never call cudaMalloc).  llsa_index_transpose_noalloc serves them from a fixed
array inside the library.  This file is collected last on purpose: it checks,
through the C ABI, that two calls in a row give exactly what the ordinary
entry point gives with a caller-provided scratch buffer, both in a fresh
process and after every other test has run.
"""
import ctypes

import numpy as np
import pytest

torch = pytest.importorskip("torch")


def _problem():
    from hierarchical_top_sparse_b200 import llsa
    return llsa.Problem(batch=8, heads=6, height=128, width=128, d=64, B=16, L=3, K=8, dtype=llsa.BF16)


@pytest.mark.gpu
def test_noalloc_transpose_equals_the_scratch_version_twice():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import synthetic
    from hierarchical_top_sparse_b200 import llsa
    p = _problem()
    lib = llsa.lib()
    q, k, _ = synthetic.qkv(3, p.batch, p.heads, p.height, p.width, p.d, 4.0)
    qd = torch.from_numpy(q).cuda().to(torch.bfloat16)
    kd = torch.from_numpy(k).cuda().to(torch.bfloat16)
    pipe = llsa.Pipeline(p, backward=True)
    llsa.pool(p, qd, pipe.pyrQ)
    llsa.pool(p, kd, pipe.pyrK)
    llsa.select(p, pipe.pyrQ, pipe.pyrK, pipe.idx)
    llsa.index_transpose(p, pipe.idx, pipe.offs, pipe.qlist, pipe.tscratch)
    torch.cuda.synchronize()
    want_offs, want_q = pipe.offs.cpu().numpy(), pipe.qlist.cpu().numpy()
    stream = torch.cuda.current_stream().cuda_stream
    for call in range(2):
        offs = torch.full_like(pipe.offs, -7)
        ql = torch.full_like(pipe.qlist, -7)
        st = lib.llsa_index_transpose_noalloc(ctypes.byref(p.c()), pipe.idx.data_ptr(), offs.data_ptr(),
                                              ql.data_ptr(), stream)
        assert st == 0, llsa.status_string(st)
        torch.cuda.synchronize()
        np.testing.assert_array_equal(offs.cpu().numpy(), want_offs, err_msg=f"offsets, call {call + 1}")
        np.testing.assert_array_equal(ql.cpu().numpy(), want_q, err_msg=f"query lists, call {call + 1}")


def test_noalloc_transpose_rejects_problems_beyond_its_array():
    # host-side check, returned before anything is launched: a 1024 x 1024
    # image with 16 slices needs more than the 16 MiB array
    from hierarchical_top_sparse_b200 import llsa
    lib = llsa.lib()
    p = llsa.Problem(batch=1, heads=16, height=1024, width=1024, d=64, B=16, L=4, K=8)
    assert llsa.query_sizes(p)["transpose_scratch_bytes"] > 16 << 20
    buf = 1 << 20   # never dereferenced
    assert lib.llsa_index_transpose_noalloc(ctypes.byref(p.c()), buf, buf, buf, None) == 4
    assert lib.llsa_index_transpose_noalloc(ctypes.byref(p.c()), None, buf, buf, None) in (1, 4)
