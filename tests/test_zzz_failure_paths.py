"""The timeout path of the bounded device waits, exercised without a fault or
a hang: llsa_selftest_wait_timeout runs the same bounded mbarrier wait the
pipelined kernels use, on a phase nothing completes, with a short limit; the
host reads the code it leaves in the device error word, and the context stays
usable.  (This file sorts last, after the parity runs.)"""
import pytest

from parity_util import Case, GpuRun, assert_close

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def _llsa():
    from hierarchical_top_sparse_b200 import llsa
    return llsa


def test_a_wait_nothing_completes_gives_up_after_its_limit_and_reports_its_code():
    llsa = _llsa()
    llsa.device_error()                                   # start from a clear word
    s = torch.cuda.current_stream()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(s)
    llsa.selftest_wait_timeout(2000, 91)
    t1.record(s)
    assert llsa.device_error() == 91                      # reported (LLSA_ERR_TIMEOUT) ...
    assert llsa.device_error() == 0                       # ... and cleared by the read
    assert t0.elapsed_time(t1) >= 1.8                     # ms: the wait ran to its 2 ms limit


def test_a_wait_that_completes_reports_nothing():
    llsa = _llsa()
    llsa.device_error()
    llsa.selftest_wait_timeout(1000000, 92, arrive=True)
    assert llsa.device_error() == 0


def test_the_context_stays_usable_after_a_timeout():
    llsa = _llsa()
    llsa.selftest_wait_timeout(1000, 93)
    assert llsa.device_error() == 93
    import oracle
    run = GpuRun(Case(batch=1, heads=1, H=32, W=32, L=2, K=4))
    pk, pv = oracle.pool(run.op, run.kh), oracle.pool(run.op, run.vh)
    o, lse = oracle.attn_fwd(run.op, run.qh, run.kh, run.vh, pk, pv, run.idx)
    assert_close("O", run.o, o, run.case.dtype)
    assert_close("LSE", run.lse, lse, run.case.dtype)
