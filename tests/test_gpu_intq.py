"""GPU parity of the symmetric uniform INT quantiser with one scale per 16
weights (2-bit ternary, 3 and 4 bits): codes and scales bit for bit against the
oracle, and the dense dequantisation bit for bit (fp32 and bf16)."""

import numpy as np
import pytest
import torch

import quantized_rank_fine_b200 as q
import synth
from oracle import intq, nf4
from tests.helpers import require_gpu

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
