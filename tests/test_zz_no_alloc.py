"""The allocation-free forward (qlora_linear_fwd_static_ws) against the
workspace forward (qlora_linear_fwd).

Callers that cannot allocate device memory (a host program using only the C
ABI with no device allocator, a plugin inside a runtime that owns all device
memory, a path that cannot afford cudaMalloc's possible synchronisation) call
the static-workspace entry point instead; it must give the same result as the
forward that takes a caller-allocated workspace.  The array inside the library
keeps the previous call's contents, so every case is called twice in a row, and
the cases themselves follow one another (small-M dequant-GEMV path and the
tcgen05 GEMM path share the array).  This file is collected last."""

import ctypes

import pytest
import torch

import quantized_rank_fine_b200 as q
from tests.helpers import assert_close, layer_on_gpu, require_gpu

pytestmark = pytest.mark.gpu


def _static_fwd(w, X, A, B, Y, V):
    ws = w.c_struct()
    return q.lib().qlora_linear_fwd_static_ws(ctypes.byref(ws), X.data_ptr(), X.shape[0], A.data_ptr(),
                                              B.data_ptr(), A.shape[1], Y.data_ptr(), V.data_ptr(),
                                              torch.cuda.current_stream().cuda_stream)


@pytest.mark.parametrize("n_in,n_out,M,r", [(256, 256, 64, 8), (4096, 4096, 4, 16), (512, 768, 300, 24),
                                            (4096, 11008, 16, 16), (1024, 1024, 1, 64)])
def test_static_workspace_forward_matches_workspace_forward(n_in, n_out, M, r):
    require_gpu()
    t, w = layer_on_gpu(n_in, n_out, M, r, tag="static")
    Yref, Vref = q.qlora_linear_fwd(w, t["X"], t["A"], t["B"], q.Workspace())
    torch.cuda.synchronize()
    for _ in range(2):
        Y = torch.full_like(Yref, float("nan"))
        V = torch.full_like(Vref, float("nan"))
        assert _static_fwd(w, t["X"], t["A"], t["B"], Y, V) == 0
        torch.cuda.synchronize()
        assert q.lib().qlora_static_ws_status(torch.cuda.current_stream().cuda_stream) == 0
        assert_close(Y, Yref.double().cpu().numpy(), "Y")
        assert_close(V, Vref.double().cpu().numpy(), "V")


def _min_fwd_ws(M, r):
    """The smallest forward workspace (the 1280-byte prefix and V, M x r bf16
    rounded up to 256 bytes) that the entry point checks against its array."""
    return 1280 + (M * r * 2 + 255) // 256 * 256


def test_static_workspace_rejects_sizes_beyond_the_array():
    require_gpu()
    M, n_in, n_out, r = 262144, 4096, 4096, 64
    assert _min_fwd_ws(M, r) > (16 << 20)
    t, w = layer_on_gpu(256, 256, 64, 8, tag="static_big")
    big = q._Weight(w.codes.data_ptr(), w.dq_codes.data_ptr(), w.dq_scales.data_ptr(), n_in, n_out)
    rc = q.lib().qlora_linear_fwd_static_ws(ctypes.byref(big), t["X"].data_ptr(), M, t["A"].data_ptr(),
                                           t["B"].data_ptr(), r, t["X"].data_ptr(), None,
                                           torch.cuda.current_stream().cuda_stream)
    assert rc == 4   # QLORA_ERR_WORKSPACE, nothing launched


def test_static_workspace_boundary():
    """At r = 64 the largest token count whose smallest workspace still fits the
    16 MiB array runs (and matches the workspace forward); one more token is
    refused.  The full workspace (with the GEMM's split region) of the accepted
    size is larger than the array: the entry point keeps every GEMM tile whole."""
    require_gpu()
    r, n_in, n_out = 64, 64, 128
    M_ok = ((16 << 20) - 1280) // (2 * r)
    assert _min_fwd_ws(M_ok, r) <= (16 << 20) < _min_fwd_ws(M_ok + 1, r)
    t, w = layer_on_gpu(n_in, n_out, M_ok + 1, r, tag="static_edge")
    X = t["X"][:M_ok]
    Yref, Vref = q.qlora_linear_fwd(w, X, t["A"], t["B"], q.Workspace())
    torch.cuda.synchronize()
    Y = torch.full_like(Yref, float("nan"))
    V = torch.full_like(Vref, float("nan"))
    assert _static_fwd(w, X, t["A"], t["B"], Y, V) == 0
    torch.cuda.synchronize()
    assert q.lib().qlora_static_ws_status(torch.cuda.current_stream().cuda_stream) == 0
    assert_close(Y, Yref.double().cpu().numpy(), "Y")
    assert_close(V, Vref.double().cpu().numpy(), "V")
    Y1 = torch.empty((M_ok + 1, n_out), dtype=torch.bfloat16, device="cuda")
    V1 = torch.empty((M_ok + 1, r), dtype=torch.bfloat16, device="cuda")
    assert _static_fwd(w, t["X"], t["A"], t["B"], Y1, V1) == 4
