"""GPU parity of the symmetric uniform INT quantiser with one scale per 16
weights (2-bit ternary, 3 and 4 bits): codes and scales bit for bit against the
oracle, and the dense dequantisation bit for bit (fp32 and bf16)."""

import numpy as np
import pytest
import torch

import quantized_rank_fine_b200 as q
import synth
from oracle import intq, linear, nf4
from tests.helpers import assert_close, require_gpu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    require_gpu()


def _check(W, bits):
    n_in, n_out = W.shape
    codes, scales = q.qlora_quantize_int(torch.from_numpy(np.ascontiguousarray(W)).cuda(), bits)
    torch.cuda.synchronize()
    rc, rs = intq.quantize_int(W, bits)
    gc, gs = codes.cpu().numpy(), scales.cpu().numpy()
    bad = np.flatnonzero(gc != rc)
    assert bad.size == 0, f"bits {bits}: {bad.size} code bytes differ, first {bad[:4]}"
    assert np.array_equal(gs.view(np.uint32), rs.view(np.uint32)), f"bits {bits}: scales differ"
    want = intq.dequantize_int(rc, rs, n_in, n_out)
    got32 = q.qlora_dequantize_int(codes, scales, n_in, n_out, torch.float32).cpu().numpy()
    got16 = q.qlora_dequantize_int(codes, scales, n_in, n_out, torch.bfloat16).float().cpu().numpy()
    assert np.array_equal(got32.view(np.uint32), want.view(np.uint32))
    assert np.array_equal(got16.view(np.uint32), nf4.round_bf16(want).view(np.uint32))


@pytest.mark.parametrize("bits", [2, 3, 4])
@pytest.mark.parametrize("shape", [(256, 256), (7, 48), (4096, 4096)])
def test_int_quantize_bitexact(bits, shape):
    W = synth.normal(f"intq{shape}", shape, 0.02).numpy()
    _check(W, bits)


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_int_quantize_edge_cases(bits):
    """Exact half-steps (ties to even), all-zero groups, a lone non-zero,
    subnormal and huge magnitudes, and negative group maxima."""
    Qm = intq.qmax(bits)
    rng = np.random.default_rng(bits)
    G = np.asarray(rng.normal(0, 0.02, (64, 16)), dtype=np.float32)
    G[0] = 0.0
    G[1] = -0.0
    G[2] = 0.0
    G[2, 9] = 0.3
    for r in range(3, 3 + Qm):
        # group max Q (s = 1): every half-step k + 1/2 below it, both signs
        row = np.zeros(16, np.float32)
        row[0] = Qm
        halves = [k + 0.5 for k in range(Qm)]
        row[1:1 + len(halves)] = halves
        row[8:8 + len(halves)] = [-h for h in halves]
        G[r] = row
    G[10] *= np.float32(1e30)
    G[11] = np.asarray(rng.normal(0, 1, 16), dtype=np.float32) * np.float32(1e-41)
    G[12] = -np.abs(G[12])
    _check(G.reshape(16, 64), bits)


def _int_layer(n_in, n_out, M, r, bits, tag):
    t = synth.layer_inputs(n_in, n_out, M, r, device="cuda", tag=tag)
    codes, scales = q.qlora_quantize_int(t["W0"], bits)
    return t, q.int_weight(codes, scales, n_in, n_out)


def _int_oracle_weight(w):
    return nf4.round_bf16(intq.dequantize_int(w.codes.cpu().numpy(), w.dq_scales.cpu().numpy(), w.n_in, w.n_out))


@pytest.mark.parametrize("bits", [2, 4])
def test_int_weight_dequantize_and_merge(bits):
    """The INT weight through the layer's descriptor: qlora_dequantize equals
    qlora_dequantize_int bit for bit, and the merge matches the oracle's."""
    t, w = _int_layer(320, 192, 1, 24, bits, "intm")
    a = q.qlora_dequantize(w, torch.float32)
    b = q.qlora_dequantize_int(w.codes, w.dq_scales, 320, 192, torch.float32)
    assert torch.equal(a, b)
    ref = linear.merge(intq.dequantize_int(w.codes.cpu().numpy(), w.dq_scales.cpu().numpy(), 320, 192),
                       t["A"], t["B"])
    assert_close(q.qlora_merge(w, t["A"], t["B"], torch.float32), ref, "merge int", rel_fro=1e-6, max_abs=1e-5)


@pytest.mark.parametrize("bits", [2, 3, 4])
@pytest.mark.parametrize("M,n_in,n_out,r", [(300, 320, 192, 24), (8, 512, 768, 16), (1100, 2048, 1536, 40)])
def test_linear_int_weight(bits, M, n_in, n_out, r):
    """Forward and backward of the adapted layer on an INT (group 16) base,
    through the fused GEMMs (small M included), against the oracle."""
    t, w = _int_layer(n_in, n_out, M, r, bits, "intlin")
    ws = q.Workspace()
    Y, V = q.qlora_linear_fwd(w, t["X"], t["A"], t["B"], ws)
    dX, dA, dB = q.qlora_linear_bwd(w, t["X"], V, t["dY"], t["A"], t["B"], ws)
    torch.cuda.synchronize()
    assert ws.status() == 0
    Wq = _int_oracle_weight(w)
    Yr, Vr = linear.forward(t["X"], t["A"], t["B"], Wq)
    g = linear.backward(t["X"], t["A"], t["B"], Wq, t["dY"])
    for name, got, ref in (("Y", Y, Yr), ("V", V, Vr), ("dX", dX, g["dX"]), ("dA", dA, g["dA"]),
                           ("dB", dB, g["dB"])):
        assert_close(got, ref, name)
