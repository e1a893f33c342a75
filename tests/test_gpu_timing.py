"""The measurement helpers of the library on the GPU: per-kernel event timing
(eagerly and inside a captured CUDA graph) and the launch counter."""

import pytest
import torch

import quantized_rank_fine_b200 as q
from tests.helpers import layer_on_gpu, require_gpu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    require_gpu()


def test_kernel_timer_eager_and_launch_count():
    t, w = layer_on_gpu(512, 512, 512, 16)
    ws = q.Workspace()
    q.qlora_linear_fwd(w, t["X"], t["A"], t["B"], ws)
    torch.cuda.synchronize()
    n0 = q.qlora_launch_count()
    tm = q.KernelTimer(q.KERNEL_FWD_GEMM, 3)
    for _ in range(3):
        q.qlora_linear_fwd(w, t["X"], t["A"], t["B"], ws)
    torch.cuda.synchronize()
    times = tm.times_ms()
    tm.disarm()
    assert all(x > 0 for x in times)
    assert q.qlora_launch_count() - n0 >= 6          # V = X A and the GEMM per call


def test_kernel_timer_inside_graph():
    t, w = layer_on_gpu(4096, 4096, 4, 16, tag="graph")
    ws = q.Workspace()
    Y, V = q.qlora_linear_fwd(w, t["X"], t["A"], t["B"], ws)
    torch.cuda.synchronize()
    tm = q.KernelTimer(q.KERNEL_GEMV, 2)
    g = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        with torch.cuda.graph(g, stream=side, capture_error_mode="relaxed"):
            for _ in range(2):
                q.qlora_linear_fwd(w, t["X"], t["A"], t["B"], ws, Y=Y, V=V)
    torch.cuda.current_stream().wait_stream(side)
    tm.disarm()
    g.replay()
    torch.cuda.synchronize()
    assert all(x > 0 for x in tm.times_ms())
    Y2, _ = q.qlora_linear_fwd(w, t["X"], t["A"], t["B"], ws)
    torch.cuda.synchronize()
    assert torch.equal(Y, Y2)
