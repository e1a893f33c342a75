"""GPU parity of the adapted linear layer (forward and backward) against the
float64 oracle: relative Frobenius error <= 1e-2 and max-abs error <= 2e-2 of
max |ref| on Y, V, dX, dA, dB; exact invariants where the method fixes them."""

import pytest
import torch

import quantized_rank_fine_b200 as q
import synth
from oracle import linear
from tests.helpers import (assert_close, assert_guards, full_check, guarded, layer_on_gpu, oracle_weight, require_gpu,
                           run_fwd_bwd)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    require_gpu()


def test_linear_256_m64_r8_full():
    """The small configuration: in = out = 256, M = 64, r = 8, every output."""
    t, w = layer_on_gpu(256, 256, 64, 8)
    full_check(t, w, run_fwd_bwd(t, w))


@pytest.mark.parametrize("M,n_in,n_out,r", [
    (1, 64, 64, 8), (7, 192, 320, 16), (300, 320, 192, 24), (257, 512, 768, 64),
    (130, 256, 512, 72), (513, 128, 1024, 256), (64, 1024, 64, 8), (1000, 576, 704, 40),
])
def test_linear_ragged_shapes(M, n_in, n_out, r):
    """Ragged M and N tiles, K not a multiple of the tile, several adapter K-steps;
    every output sits between canary guard regions that must stay untouched."""
    t, w = layer_on_gpu(n_in, n_out, M, r, tag="ragged")
    shapes = {"Y": ((M, n_out), torch.bfloat16), "V": ((M, r), torch.bfloat16), "dX": ((M, n_in), torch.bfloat16),
              "dA": ((n_in, r), torch.float32), "dB": ((r, n_out), torch.float32)}
    bufs, out = {}, {}
    for k, (shape, dt) in shapes.items():
        bufs[k], out[k] = guarded(shape, dt)
    ws = q.Workspace()
    q.qlora_linear_fwd(w, t["X"], t["A"], t["B"], ws, Y=out["Y"], V=out["V"])
    q.qlora_linear_bwd(w, t["X"], out["V"], t["dY"], t["A"], t["B"], ws, dX=out["dX"], dA=out["dA"], dB=out["dB"])
    assert_guards(list(bufs.values()), "ragged fwd/bwd")
    assert ws.status() == 0
    full_check(t, w, out)


def test_B_zero_invariants():
    """B = 0: dA is exactly zero, and the forward output does not depend on A
    at all (the adapter adds exact zeros to the accumulator)."""
    t, w = layer_on_gpu(320, 448, 200, 16, zero_B=True)
    out = run_fwd_bwd(t, w)
    assert torch.count_nonzero(out["dA"]).item() == 0
    t2 = dict(t)
    t2["A"] = synth.normal("otherA", t["A"].shape, 0.5, torch.bfloat16, "cuda")
    out2 = run_fwd_bwd(t2, w)
    assert torch.equal(out["Y"], out2["Y"])
    full_check(t, w, out)


def test_frozen_weight_untouched_by_fwd_bwd():
    t, w = layer_on_gpu(256, 320, 96, 16)
    snap = [x.clone() for x in (w.codes, w.dq_codes, w.dq_scales)]
    run_fwd_bwd(t, w)
    assert all(torch.equal(a, b) for a, b in zip(snap, (w.codes, w.dq_codes, w.dq_scales)))


def test_bwd_without_saved_V_and_without_dX():
    """V = NULL recomputes X A inside the backward; dX = NULL skips the dX GEMM."""
    t, w = layer_on_gpu(256, 384, 120, 16)
    ws = q.Workspace()
    Y, V = q.qlora_linear_fwd(w, t["X"], t["A"], t["B"], ws)
    dX1, dA1, dB1 = q.qlora_linear_bwd(w, t["X"], V, t["dY"], t["A"], t["B"], ws)
    dX2, dA2, dB2 = q.qlora_linear_bwd(w, t["X"], None, t["dY"], t["A"], t["B"], ws, need_dX=False)
    torch.cuda.synchronize()
    assert dX2 is None
    assert torch.equal(dA1, dA2) and torch.equal(dB1, dB2)


@pytest.mark.parametrize("M", [1, 4, 16])
@pytest.mark.parametrize("n_in,n_out", [(4096, 4096), (4096, 11008)])
def test_linear_small_m_forward(M, n_in, n_out):
    """Small-M forward (token counts 1, 4, 16), every output."""
    t, w = layer_on_gpu(n_in, n_out, M, 16, tag="gemv")
    ws = q.Workspace()
    Y, V = q.qlora_linear_fwd(w, t["X"], t["A"], t["B"], ws)
    torch.cuda.synchronize()
    Yr, Vr = linear.forward(t["X"], t["A"], t["B"], oracle_weight(w))
    assert_close(Y, Yr, "Y")
    assert_close(V, Vr, "V")


@pytest.mark.parametrize("M,n_in,n_out,r", [
    (1, 64, 64, 8), (3, 192, 320, 16), (8, 128, 256, 8), (9, 1024, 704, 24),
    (16, 8192, 512, 256), (13, 11008, 1088, 8), (2, 4096, 11072, 16), (5, 2048, 256, 72),
    (12, 64, 192, 40),
])
def test_small_m_forward_shapes(M, n_in, n_out, r):
    """Small-M forward on ragged shapes: a partial last column tile, one to
    sixteen K-splits, both token-tile counts, the largest adapter rank."""
    t, w = layer_on_gpu(n_in, n_out, M, r, tag="gemv-ragged")
    ws = q.Workspace()
    (bY, Y), (bV, V) = guarded((M, n_out), torch.bfloat16), guarded((M, r), torch.bfloat16)
    q.qlora_linear_fwd(w, t["X"], t["A"], t["B"], ws, Y=Y, V=V)
    assert_guards([bY, bV], "small-M forward")
    assert ws.status() == 0
    Yr, Vr = linear.forward(t["X"], t["A"], t["B"], oracle_weight(w))
    assert_close(Y, Yr, "Y")
    assert_close(V, Vr, "V")


def test_small_m_forward_deterministic_and_graph():
    """The small-M forward is deterministic (fixed reduction order), also when
    captured in a CUDA graph together with the kernel that produces V."""
    t, w = layer_on_gpu(4096, 4096, 4, 16, tag="gemv-graph")
    ws = q.Workspace()
    Y1, V1 = q.qlora_linear_fwd(w, t["X"], t["A"], t["B"], ws)
    Y2, V2 = q.qlora_linear_fwd(w, t["X"], t["A"], t["B"], ws)
    Yg = torch.empty_like(Y1)
    Vg = torch.empty_like(V1)
    graph = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        with torch.cuda.graph(graph, stream=side):
            q.qlora_linear_fwd(w, t["X"], t["A"], t["B"], ws, Y=Yg, V=Vg)
    torch.cuda.current_stream().wait_stream(side)
    Yg.zero_()
    graph.replay()
    torch.cuda.synchronize()
    assert torch.equal(Y1, Y2) and torch.equal(V1, V2)
    assert torch.equal(Yg, Y1) and torch.equal(Vg, V1)
    del graph


@pytest.mark.parametrize("M,n_in,n_out,r", [(8, 512, 768, 16), (300, 320, 192, 24)])
def test_adapter_scale(M, n_in, n_out, r):
    """Y = X w' + s (X A) B and its backward with s = alpha / r = 2 ("Scaling
    Factor alpha"), on the small-M and the GEMM paths, against the oracle."""
    t, w = layer_on_gpu(n_in, n_out, M, r, tag="scale")
    s = 2.0
    ws = q.Workspace()
    Y, V = q.qlora_linear_fwd(w, t["X"], t["A"], t["B"], ws, adapter_scale=s)
    dX, dA, dB = q.qlora_linear_bwd(w, t["X"], V, t["dY"], t["A"], t["B"], ws, adapter_scale=s)
    torch.cuda.synchronize()
    assert ws.status() == 0
    Wq = oracle_weight(w)
    Yr, Vr = linear.forward(t["X"], t["A"], t["B"], Wq, s)
    g = linear.backward(t["X"], t["A"], t["B"], Wq, t["dY"], s)
    for got, ref, name in ((Y, Yr, "Y"), (V, Vr, "V"), (dX, g["dX"], "dX"), (dA, g["dA"], "dA"), (dB, g["dB"], "dB")):
        assert_close(got, ref, name)


def test_accumulated_gradients():
    """QLORA_ACCUMULATE_GRADS adds into the given dA and dB (two micro-batches on
    top of a nonzero start) instead of overwriting them."""
    t, w = layer_on_gpu(256, 384, 96, 16, tag="acc")
    t2, _ = layer_on_gpu(256, 384, 96, 16, tag="acc2")
    ws = q.Workspace()
    dA0 = synth.normal("acc_dA0", (256, 16), 1.0, device="cuda")
    dB0 = synth.normal("acc_dB0", (16, 384), 1.0, device="cuda")
    dA, dB = dA0.clone(), dB0.clone()
    for tt in (t, t2):
        _, V = q.qlora_linear_fwd(w, tt["X"], t["A"], t["B"], ws)
        q.qlora_linear_bwd(w, tt["X"], V, tt["dY"], t["A"], t["B"], ws, need_dX=False, dA=dA, dB=dB,
                           accumulate=True)
    torch.cuda.synchronize()
    Wq = oracle_weight(w)
    g1 = linear.backward(t["X"], t["A"], t["B"], Wq, t["dY"])
    g2 = linear.backward(t2["X"], t["A"], t["B"], Wq, t2["dY"])
    assert_close(dA, dA0.double().cpu().numpy() + g1["dA"] + g2["dA"], "dA accumulated")
    assert_close(dB, dB0.double().cpu().numpy() + g1["dB"] + g2["dB"], "dB accumulated")


@pytest.mark.parametrize("M,n_in,n_out,r,p", [
    (300, 320, 192, 24, 0.05), (1000, 576, 704, 40, 0.5), (4, 512, 768, 16, 0.3), (16, 4096, 4096, 16, 0.05),
])
def test_dropout(M, n_in, n_out, r, p):
    """Dropout on X A ("LoRA & QLoRA", "Dropout") with adapter scale 2: a keep mask
    drawn with torch on the device, the same bytes to both sides; every output of
    the forward and backward against the oracle (M <= 16 takes the small-M
    forward), and the backward that recomputes V matches the one given V."""
    t, w = layer_on_gpu(n_in, n_out, M, r, tag="drop")
    gen = torch.Generator(device="cuda")
    gen.manual_seed(5)
    keep = q.dropout_mask(M, r, p, generator=gen)
    s = 2.0
    ws = q.Workspace()
    Y, V = q.qlora_linear_fwd(w, t["X"], t["A"], t["B"], ws, adapter_scale=s, dropout_keep=keep, dropout_p=p)
    dX, dA, dB = q.qlora_linear_bwd(w, t["X"], V, t["dY"], t["A"], t["B"], ws, adapter_scale=s,
                                    dropout_keep=keep, dropout_p=p)
    dX2, dA2, dB2 = q.qlora_linear_bwd(w, t["X"], None, t["dY"], t["A"], t["B"], ws, adapter_scale=s,
                                       dropout_keep=keep, dropout_p=p)
    torch.cuda.synchronize()
    assert ws.status() == 0
    assert torch.equal(dX, dX2) and torch.equal(dA, dA2) and torch.equal(dB, dB2)
    k = keep.cpu().numpy()
    assert 0 < k.sum() < k.size or p < 0.1
    Wq = oracle_weight(w)
    Yr, Vr = linear.forward(t["X"], t["A"], t["B"], Wq, s, k, p)
    g = linear.backward(t["X"], t["A"], t["B"], Wq, t["dY"], s, k, p)
    assert_close(Y, Yr, "Y")
    assert_close(V, Vr, "V")
    assert_close(dX, g["dX"], "dX")
    assert_close(dA, g["dA"], "dA")
    assert_close(dB, g["dB"], "dB")
    # dropped elements of V are exact zeros
    assert torch.count_nonzero(V[keep == 0]).item() == 0


@pytest.mark.parametrize("M", [8, 300])
def test_dropout_drop_all(M):
    """A mask that drops every element leaves the frozen base alone: Y is the
    forward with B = 0, bit for bit, and dA = dB = 0 exactly."""
    n_in, n_out, r = 512, 320, 16
    t, w = layer_on_gpu(n_in, n_out, M, r, tag="dropall")
    ws = q.Workspace()
    keep = torch.zeros((M, r), dtype=torch.uint8, device="cuda")
    Y, V = q.qlora_linear_fwd(w, t["X"], t["A"], t["B"], ws, dropout_keep=keep, dropout_p=0.5)
    dX, dA, dB = q.qlora_linear_bwd(w, t["X"], V, t["dY"], t["A"], t["B"], ws, dropout_keep=keep, dropout_p=0.5)
    Y0, _ = q.qlora_linear_fwd(w, t["X"], t["A"], torch.zeros_like(t["B"]), ws)
    torch.cuda.synchronize()
    assert torch.equal(Y, Y0)
    assert torch.count_nonzero(dA).item() == 0 and torch.count_nonzero(dB).item() == 0
