"""GPU parity of the merge -> re-quantize round trip and of the LoftQ-style
adapter initialisation against the float64 oracle."""

import numpy as np
import pytest
import torch

import quantized_rank_fine_b200 as q
import synth
from oracle import loftq, nf4
from tests.helpers import assert_close, layer_on_gpu, require_gpu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    require_gpu()


def _f64(t):
    return t.detach().double().cpu().numpy()


def test_round_trip_with_zero_adapters_keeps_every_byte():
    """Merging zero adapters and quantising again reproduces the weight's codes,
    absmax codes and scales bit for bit."""
    t, w = layer_on_gpu(512, 768, 8, 8, zero_B=True, tag="rt0")
    w2 = q.requantize_merged(w, t["A"], t["B"])
    torch.cuda.synchronize()
    assert torch.equal(w2.codes, w.codes)
    assert torch.equal(w2.dq_codes, w.dq_codes)
    assert torch.equal(w2.dq_scales, w.dq_scales)


@pytest.mark.parametrize("scale", [1.0, 30.0])
def test_round_trip_matches_oracle(scale):
    """The re-quantized merge against the oracle's round trip of the same
    weight and adapters: the dequantised results agree, and so does the share
    of A B the round trip loses (about 0.7 at the configs' adapter scale)."""
    t, w = layer_on_gpu(512, 512, 8, 16, tag="rt1")
    B = (t["B"].float() * scale).to(torch.bfloat16)
    w2 = q.requantize_merged(w, t["A"], B)
    W_gpu = _f64(q.qlora_dequantize(w2, torch.float32))
    # the merge adds A B to the fp32 w' (not to its bf16 rounding)
    Wq32 = nf4.dequantize(w.codes.cpu().numpy(), w.dq_codes.cpu().numpy(), w.dq_scales.cpu().numpy(), 512, 512)
    W_ref, _ = loftq.requantize_merged(Wq32, t["A"], B)
    assert_close(W_gpu, W_ref, "re-quantized merge")
    lost_gpu = loftq.lost_fraction(Wq32, t["A"], B, W_gpu)
    lost_ref = loftq.lost_fraction(Wq32, t["A"], B, W_ref)
    assert abs(lost_gpu - lost_ref) < 0.02, (lost_gpu, lost_ref)


@pytest.mark.parametrize("n_in,n_out,r", [(512, 384, 8), (1024, 1024, 16)])
def test_loftq_init_matches_oracle(n_in, n_out, r):
    """A B from the device SVD against the oracle's float64 SVD of the same
    residual, and the residual after initialisation is smaller than before."""
    W0 = synth.normal("loftqW0", (n_in, n_out), 0.02, device="cuda")
    w, A, B = q.loftq_init(W0, r)
    torch.cuda.synchronize()
    A_ref, B_ref = loftq.loftq_init(W0.cpu().numpy(), r)
    assert_close(_f64(A.float() @ B.float()), A_ref @ B_ref, "A B")
    R = _f64(W0) - _f64(q.qlora_dequantize(w, torch.float32))
    assert np.linalg.norm(R - _f64(A.float() @ B.float())) < np.linalg.norm(R)


@pytest.mark.parametrize("shape,fmt", [((512, 384), "nf4"), ((4096, 11008), "nf4"), ((320, 192), "u8"),
                                       ((256, 512), "int16")])
def test_loftq_residual_bitexact(shape, fmt):
    """R = fl32(W0 - w') from the library kernel equals the oracle's residual
    (exact in float64) rounded once to fp32, bit for bit, for NF4 weights with
    either absmax code format and for the INT (one scale per 16) format."""
    from oracle import intq
    W0 = synth.normal(f"resid{shape}", shape, 0.02, device="cuda")
    W0h = W0.cpu().numpy()
    if fmt == "int16":
        codes, scales = q.qlora_quantize_int(W0, 4)
        w = q.int_weight(codes, scales, *shape)
        ref = W0h.astype(np.float64) - intq.dequantize_int(codes.cpu().numpy(), scales.cpu().numpy(), *shape)
    else:
        w = q.qlora_quantize_nf4(W0, dq_format=q.QLORA_DQ_U8 if fmt == "u8" else q.QLORA_DQ_E4M3)
        deq = nf4.dequantize(w.codes.cpu().numpy(), w.dq_codes.cpu().numpy(), w.dq_scales.cpu().numpy(), *shape,
                             dq_format="u8" if fmt == "u8" else "e4m3")
        ref = W0h.astype(np.float64) - deq.astype(np.float64)
        if fmt == "nf4":
            np.testing.assert_array_equal(ref, loftq.residual(W0h))
    R = q.qlora_loftq_residual(W0, w)
    torch.cuda.synchronize()
    assert np.array_equal(R.cpu().numpy().view(np.uint32), nf4.fl32(ref).view(np.uint32))


@pytest.mark.parametrize("n_in,n_out,k,r", [(512, 384, 384, 8), (1024, 1024, 1024, 16), (4096, 11008, 64, 64)])
def test_loftq_split_bitexact(n_in, n_out, k, r):
    """A and B from given fp32 factors (U with k > r columns, Vh with k rows)
    equal the oracle's stored-precision split bit for bit."""
    U = synth.normal(f"splitU{n_in}", (n_in, k), 1.0 / np.sqrt(n_in), device="cuda")
    S = synth.normal(f"splitS{k}", (k,), 1.0, device="cuda").abs().sort(descending=True).values.contiguous()
    Vh = synth.normal(f"splitV{n_out}", (k, n_out), 1.0 / np.sqrt(n_out), device="cuda")
    A, B = q.qlora_loftq_split(U, S, Vh, r)
    torch.cuda.synchronize()
    Ar, Br = loftq.split_adapters(U.cpu().numpy(), S.cpu().numpy(), Vh.cpu().numpy(), r)
    assert np.array_equal(A.float().cpu().numpy().view(np.uint32), Ar.view(np.uint32))
    assert np.array_equal(B.float().cpu().numpy().view(np.uint32), Br.view(np.uint32))
