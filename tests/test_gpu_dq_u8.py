"""GPU parity of the linear-uint8 double quantisation (dq_format = QLORA_DQ_U8):
per group s = fl32(max / 255), absmax code = min(255, rint(fl32(a / s))) with
ties to even, a' = fl32(code s).  Codes, absmax codes, scales and the dense
dequantised weight bit for bit against the oracle; merge and the adapted layer
(fused GEMM and small-M paths) within the layer tolerance."""

import numpy as np
import pytest
import torch

import quantized_rank_fine_b200 as q
import synth
from oracle import linear, nf4
from tests.helpers import assert_close, assert_quant_equal, full_check, layer_on_gpu, oracle_weight, require_gpu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    require_gpu()


def quantize_u8(W0):
    w = q.qlora_quantize_nf4(W0.cuda().contiguous(), dq_format=q.QLORA_DQ_U8)
    torch.cuda.synchronize()
    gpu = (w.codes.cpu().numpy(), w.dq_codes.cpu().numpy(), w.dq_scales.cpu().numpy())
    ref = nf4.quantize_nf4(W0.cpu().numpy(), dq_format="u8")
    return w, gpu, ref


@pytest.mark.parametrize("shape", [(256, 256), (7, 640), (512, 4160), (4096, 4096)])
def test_quantize_u8_bitexact(shape):
    """Several groups, a partial last group, a full-size weight."""
    W0 = synth.normal(f"u8{shape}", shape, 0.02)
    w, gpu, ref = quantize_u8(W0)
    assert w.dq_format == q.QLORA_DQ_U8
    assert_quant_equal(gpu, ref, f"u8 {shape}")
    # the NF4 codes do not depend on the absmax format
    w8 = q.qlora_quantize_nf4(W0.cuda())
    assert torch.equal(w8.codes, w.codes)


def test_quantize_u8_ties_and_zero_groups():
    """Blocks whose absmax sits exactly half-way between two codes (group max
    63.75, so s = 0.25 and a = (k + 1/2) / 4 rounds to the even k), an all-zero
    group, and a group whose maximum is a subnormal."""
    rng = np.random.default_rng(4)
    nblk = 3 * 256
    W = nf4.fl32(rng.uniform(-0.01, 0.01, (nblk, 64)))
    W[0, 3] = np.float32(63.75)
    for k in range(1, 200):
        W[k] = nf4.fl32(rng.uniform(-0.1, 0.1, 64)) * np.float32(min(1.0, (k + 0.5) * 0.25 / 0.1))
        W[k, 7] = np.float32((k + 0.5) * 0.25)
        np.clip(W[k], -(k + 0.5) * 0.25, (k + 0.5) * 0.25, out=W[k])
    W[256:512] = 0.0
    W[512:] = nf4.fl32(rng.normal(0, 1, (256, 64))) * np.float32(1e-41)
    W0 = torch.from_numpy(np.ascontiguousarray(W.reshape(nblk * 64 // 256, 256)))
    _, gpu, ref = quantize_u8(W0)
    assert_quant_equal(gpu, ref, "u8 ties")
    assert not np.any(gpu[1][256:512]) and gpu[2][1] == 0.0


@pytest.mark.parametrize("shape", [(320, 192), (4096, 11008)])
def test_dequantize_u8_bitexact(shape):
    W0 = synth.normal(f"u8deq{shape}", shape, 0.02)
    w, gpu, _ = quantize_u8(W0)
    want = nf4.dequantize(*gpu, *shape, dq_format="u8")
    got32 = q.qlora_dequantize(w, torch.float32).cpu().numpy()
    got16 = q.qlora_dequantize(w, torch.bfloat16).float().cpu().numpy()
    assert np.array_equal(got32.view(np.uint32), want.view(np.uint32))
    assert np.array_equal(got16.view(np.uint32), nf4.round_bf16(want).view(np.uint32))


def test_merge_u8():
    t = synth.layer_inputs(320, 192, 1, 24, tag="u8m")
    w, gpu, _ = quantize_u8(t["W0"])
    ref = linear.merge(nf4.dequantize(*gpu, 320, 192, dq_format="u8"), t["A"], t["B"])
    assert_close(q.qlora_merge(w, t["A"].cuda(), t["B"].cuda(), torch.float32), ref, "merge u8", rel_fro=1e-6,
                 max_abs=1e-5)


def _u8_layer(n_in, n_out, M, r, tag):
    t = synth.layer_inputs(n_in, n_out, M, r, device="cuda", tag=tag)
    w = q.qlora_quantize_nf4(t["W0"], dq_format=q.QLORA_DQ_U8)
    return t, w


def _u8_oracle_weight(w):
    return nf4.dequantize_bf16(w.codes.cpu().numpy(), w.dq_codes.cpu().numpy(), w.dq_scales.cpu().numpy(),
                               w.n_in, w.n_out, dq_format="u8")


@pytest.mark.parametrize("M,n_in,n_out,r", [(300, 320, 192, 24), (1100, 2048, 1536, 40)])
def test_linear_u8(M, n_in, n_out, r):
    """Forward and backward through the fused GEMMs with a uint8-absmax weight."""
    t, w = _u8_layer(n_in, n_out, M, r, "u8lin")
    ws = q.Workspace()
    Y, V = q.qlora_linear_fwd(w, t["X"], t["A"], t["B"], ws)
    dX, dA, dB = q.qlora_linear_bwd(w, t["X"], V, t["dY"], t["A"], t["B"], ws)
    torch.cuda.synchronize()
    assert ws.status() == 0
    Wq = _u8_oracle_weight(w)
    Yr, Vr = linear.forward(t["X"], t["A"], t["B"], Wq)
    g = linear.backward(t["X"], t["A"], t["B"], Wq, t["dY"])
    for name, got, ref in (("Y", Y, Yr), ("V", V, Vr), ("dX", dX, g["dX"]), ("dA", dA, g["dA"]),
                           ("dB", dB, g["dB"])):
        assert_close(got, ref, name)


@pytest.mark.parametrize("M", [1, 16])
def test_small_m_forward_u8(M):
    """The small-M forward (dequant-GEMV) with a uint8-absmax weight."""
    t, w = _u8_layer(4096, 4096, M, 16, "u8gemv")
    Y, _ = q.qlora_linear_fwd(w, t["X"], t["A"], t["B"], q.Workspace())
    Yr, _ = linear.forward(t["X"], t["A"], t["B"], _u8_oracle_weight(w))
    assert_close(Y, Yr, "Y")
