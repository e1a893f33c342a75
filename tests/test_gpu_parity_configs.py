"""GPU parity at the benchmark configurations, in the launch configuration
`bench.py` times (default workspace with the GEMM's split region, every SM).

* Attention projection 4096 x 4096, r = 16, M = 4096, and the two MLP
  projections 4096 -> 11008 and 11008 -> 4096 at r = 64, M = 8192: every row of
  Y, V and dX and all of dA, dB against the float64 oracle (row blocks of the
  oracle's own forward and backward; the same tolerances as everywhere).
* The Llama-7B stack (32 layers x q, k, v, o, gate, up, down; M = 2048, r = 16),
  drawn with the benchmark's own per-linear tags on the device: the quantiser
  bit-exact on all seven projections of layers 0 and 31 and of 8 further layers
  chosen at random (seeded), and every output of the forward and backward of all
  seven projections of layers 0 and 31.

Pages: "QLoRA (low-rank adapters on a quantized model)", "How it works" steps 1-4
and "What QLoRA adds over LoRA" (the quantised frozen base, the adapters on
every linear of the model).
"""

import numpy as np
import pytest
import torch

import bench
import quantized_rank_fine_b200 as q
from oracle import nf4
from tests.helpers import (assert_quant_equal, full_check_blocked, layer_on_gpu, oracle_pool, require_gpu,
                           run_fwd_bwd)

pytestmark = pytest.mark.gpu

STACK = bench.WORKLOADS["llama7b_stack_m2048_r16"]


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    require_gpu()


def test_attn4096_m4096_r16_every_row():
    """4096 x 4096, r = 16, M = 4096: all 4096 rows of Y, V, dX; dA, dB."""
    t, w = layer_on_gpu(4096, 4096, 4096, 16)
    full_check_blocked(t, w, run_fwd_bwd(t, w))


@pytest.mark.parametrize("n_in,n_out", [(4096, 11008), (11008, 4096)])
def test_mlp_m8192_r64_every_row(n_in, n_out):
    """The MLP projections at M = 8192, r = 64: all 8192 rows of Y, V, dX; dA, dB."""
    t, w = layer_on_gpu(n_in, n_out, 8192, 64)
    full_check_blocked(t, w, run_fwd_bwd(t, w))


def stack_sample_layers():
    """Layers 0 and 31 and 8 more drawn without replacement from 1..30 (seed 8)."""
    rng = np.random.default_rng(8)
    return [0, STACK["layers"] - 1] + sorted(int(x) for x in rng.choice(np.arange(1, STACK["layers"] - 1), 8,
                                                                       replace=False))


def test_stack_quantize_sample_bitexact():
    """Codes, absmax codes and group scales of all seven projections of ten layers
    of the stack, drawn as the benchmark draws them, equal the oracle's bit for bit."""
    layers = stack_sample_layers()
    assert len(set(layers)) == 10
    with oracle_pool() as pool:
        for li in layers:
            gpu, mats = [], []
            for name, n_in, n_out, _ in STACK["layer"]:
                W0 = bench.stack_weight(li, name, n_in, n_out, seed=0)
                w = q.qlora_quantize_nf4(W0)
                torch.cuda.synchronize()
                gpu.append((w.codes.cpu().numpy(), w.dq_codes.cpu().numpy(), w.dq_scales.cpu().numpy()))
                mats.append(W0.cpu().numpy())
                del W0, w
            for (name, _, _, _), g, ref in zip(STACK["layer"], gpu, pool.map(nf4.quantize_nf4, mats, chunksize=1)):
                assert_quant_equal(g, ref, f"layer {li} {name}")


@pytest.mark.parametrize("li", [0, STACK["layers"] - 1])
def test_stack_layer_fwd_bwd_every_output(li):
    """All seven projections of one layer of the stack, on the benchmark's tensors
    (q, k, v share one input X, gate and up another): every output against the
    oracle, whose weight comes from the oracle's own quantiser of the same W0
    (and equals the GPU's codes bit for bit)."""
    M, r = STACK["M"], STACK["r"]
    acts = {}
    for name, n_in, n_out, x_key in STACK["layer"]:
        W0, t = bench.stack_linear(li, name, n_in, n_out, x_key, M, r, 0, acts)
        w = q.qlora_quantize_nf4(W0)
        out = run_fwd_bwd(t, w)
        ref = nf4.quantize_nf4(W0.cpu().numpy())
        gpu = (w.codes.cpu().numpy(), w.dq_codes.cpu().numpy(), w.dq_scales.cpu().numpy())
        assert_quant_equal(gpu, ref, f"layer {li} {name}")
        del W0
        full_check_blocked(t, w, out, Wq=nf4.dequantize_bf16(*ref, n_in, n_out))
