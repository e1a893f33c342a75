"""The failure path of the bounded device waits, made to run out on purpose.

Every wait in the library's kernels gives up after a time limit, raises a bit
in a status word and lets its kernel return; the host reads the word
(qlora_ws_status, qlora_quantize_status, qlora_static_ws_status).  Here a
test-only kernel runs one wait that nothing completes -- on an mbarrier without
arrivals, and on a workspace counter that nothing advances -- with a limit of
a few tens of microseconds.  No copy or tensor-core work is in flight, nothing
faults or hangs, and the context stays usable afterwards (a forward call
right after still matches the oracle)."""

import pytest
import torch

import quantized_rank_fine_b200 as q
from oracle import linear
from tests.helpers import assert_close, layer_on_gpu, oracle_weight, require_gpu

pytestmark = pytest.mark.gpu

QLORA_ERR_TIMEOUT = 7


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    require_gpu()


@pytest.mark.parametrize("kind", [0, 1])
def test_bounded_wait_runs_out_and_reports(kind):
    ws = q.Workspace()
    assert ws.status() == 0
    q.qlora_selftest_wait_timeout(ws, kind, limit_us=50)
    assert ws.status() == QLORA_ERR_TIMEOUT      # the wait gave up and said so
    assert ws.status() == 0                      # reading clears the word
    # the context is intact: a forward on the same workspace is still right
    t, w = layer_on_gpu(256, 320, 40, 16, tag="after-timeout")
    Y, V = q.qlora_linear_fwd(w, t["X"], t["A"], t["B"], ws)
    torch.cuda.synchronize()
    assert ws.status() == 0
    Yr, Vr = linear.forward(t["X"], t["A"], t["B"], oracle_weight(w))
    assert_close(Y, Yr, "Y")
    assert_close(V, Vr, "V")


def test_bounded_wait_limit_is_honoured():
    """A 20 ms limit keeps the kernel for about 20 ms, not the 2 s default."""
    ws = q.Workspace()
    ws.get(1280)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    q.qlora_selftest_wait_timeout(ws, 0, limit_us=20000)
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1)
    assert 19.0 <= ms < 200.0, ms
    assert ws.status() == QLORA_ERR_TIMEOUT


def test_selftest_argument_checks():
    ws = q.Workspace()
    buf = ws.get(1280)
    lib = q.lib()
    s = torch.cuda.current_stream().cuda_stream
    assert lib.qlora_selftest_wait_timeout(buf.data_ptr(), buf.numel(), 2, 50, s) == 1
    assert lib.qlora_selftest_wait_timeout(buf.data_ptr(), buf.numel(), 0, 0, s) == 1
    assert lib.qlora_selftest_wait_timeout(buf.data_ptr(), buf.numel(), 0, 2000000, s) == 1
    assert lib.qlora_selftest_wait_timeout(buf.data_ptr(), 1024, 0, 50, s) == 4
    torch.cuda.synchronize()
    assert ws.status() == 0                      # nothing was launched


def test_quantize_status_clean_after_quantize():
    """The quantiser's own status word stays clear on a normal quantisation."""
    W0 = torch.randn(512, 768, device="cuda") * 0.02
    q.qlora_quantize_nf4(W0)
    assert q.qlora_quantize_status() == 0
