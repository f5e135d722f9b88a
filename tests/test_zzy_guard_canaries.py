"""Out-of-bounds writes, caught with canaries (no memory checker runs on
these GPUs): every buffer the path writes -- pyramids, index lists, CSC
lists, transpose scratch, backward workspace, O, LSE, dQ, dK, dV -- is
placed inside a larger allocation whose 64 KB guard bands on both sides hold
a sentinel byte; after a full forward + backward step no guard byte may have
changed.  The buffers' interiors start as the sentinel too (the library never
relies on zeroed outputs), so O, LSE and the index lists must also equal
those of a plain run bit for bit."""
import numpy as np
import pytest

from parity_util import Case, to_dev

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

GUARD = 65536          # bytes on each side of every buffer
SENTINEL = 0xA5
WRITTEN = ("pyrQ", "pyrK", "pyrV", "idx", "o", "lse", "offs", "qlist", "tscratch", "work", "dq", "dk", "dv")

CASES = {
    # tensor-core kernels (bf16, d = 64, B = 16)
    "px64_bf16": Case(batch=2, heads=2, H=64, W=64, L=3, K=8),
    # CUDA-core kernels (fp32; B = 64)
    "tiny32_fp32": Case(batch=1, heads=1, H=32, W=32, L=2, K=4, dtype="fp32"),
    "B64": Case(batch=1, heads=2, H=64, W=64, B=64, L=2, K=3, d=32),
}


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def _guarded_like(t):
    nbytes = t.numel() * t.element_size()
    big = torch.full((nbytes + 2 * GUARD,), SENTINEL, dtype=torch.uint8, device=t.device)
    return big, big[GUARD:GUARD + nbytes].view(t.dtype).view(t.shape)


@pytest.mark.parametrize("name", sorted(CASES))
def test_no_write_lands_outside_its_buffer(name):
    from hierarchical_top_sparse_b200 import llsa
    case = CASES[name]
    p, _ = case.problems()
    bf = case.dtype == "bf16"
    q, k, v, g = (to_dev(x.reshape(p.batch, p.heads, p.N, p.d).astype(np.float32), bf) for x in case.inputs())

    plain = llsa.Pipeline(p)
    plain.step(q, k, v, g)

    pipe = llsa.Pipeline(p)
    bigs = {}
    for attr in WRITTEN:
        bigs[attr], view = _guarded_like(getattr(pipe, attr))
        setattr(pipe, attr, view)
    pipe.step(q, k, v, g)
    torch.cuda.synchronize()
    assert llsa.device_error() == 0

    for attr, big in bigs.items():
        head, tail = big[:GUARD], big[big.numel() - GUARD:]
        assert bool((head == SENTINEL).all()), f"{attr}: a write landed before the buffer"
        assert bool((tail == SENTINEL).all()), f"{attr}: a write landed after the buffer"
    for attr in ("idx", "o", "lse"):
        assert torch.equal(getattr(pipe, attr), getattr(plain, attr)), f"{attr} depends on the buffer's old contents"
    for attr in ("dq", "dk", "dv"):
        a, b = getattr(pipe, attr).float(), getattr(plain, attr).float()
        assert bool(torch.isfinite(a).all()), attr
        assert float((a - b).abs().max()) <= 1e-2 * max(1.0, float(b.abs().max())), attr
