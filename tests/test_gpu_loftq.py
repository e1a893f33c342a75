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
