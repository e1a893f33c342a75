"""GPU parity of the quantiser, dequantiser and merge against the float64 oracle.
NF4 codes, E4M3 absmax codes and fp32 group scales must be bit-exact; the
dequantised weight too (plain binary32 products)."""

import numpy as np
import pytest
import torch

import quantized_rank_fine_b200 as q
import synth
from oracle import linear, nf4
from tests.helpers import assert_close, assert_guards, assert_quant_equal, guarded, quantize_both, require_gpu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    require_gpu()


@pytest.mark.parametrize("shape", [(256, 256), (64, 64), (1, 64), (128, 320), (320, 192), (7, 640), (512, 4160)])
def test_quantize_bitexact_shapes(shape):
    """Several tiles, partial last group (blocks not a multiple of 256), odd rows;
    the three outputs sit between canary guard regions that must stay untouched."""
    W0 = synth.normal(f"qshape{shape}", shape, 0.02)
    n = shape[0] * shape[1]
    (b0, codes), (b1, dqc), (b2, dqs) = (guarded((n // 2,), torch.uint8), guarded((n // 64,), torch.uint8),
                                         guarded(((n // 64 + 255) // 256,), torch.float32))
    w = q.qlora_quantize_nf4(W0.cuda(), out=q.NF4Weight(codes, dqc, dqs, *shape))
    assert_guards([b0, b1, b2], "quantize")
    assert q.qlora_quantize_status() == 0
    gpu = (w.codes.cpu().numpy(), w.dq_codes.cpu().numpy(), w.dq_scales.cpu().numpy())
    assert_quant_equal(gpu, nf4.quantize_nf4(W0.numpy()), str(shape))
    (b3, deq) = guarded(shape, torch.float32)
    q.qlora_dequantize(w, torch.float32, out=deq)
    assert_guards([b3], "dequantize")
    assert np.array_equal(deq.cpu().numpy().view(np.uint32), nf4.dequantize(*gpu, *shape).view(np.uint32))


@pytest.mark.parametrize("dq_format", [q.QLORA_DQ_E4M3, q.QLORA_DQ_U8])
def test_batch_quantize_equals_single(dq_format):
    """The batch quantiser (one launch per 32 weights, the weights' groups walked
    as one sequence) gives the bytes of one call per weight: 40 weights of mixed
    shapes (short last groups, a single block, 4096 x 11008), so a batch spans
    two launches; the outputs sit between canary guard regions."""
    shapes = [(4096, 11008), (64, 96), (1, 64), (512, 768), (7, 640), (320, 192)] * 6 + [(256, 256)] * 4
    W0s = [synth.normal(f"qbatch{i}", shp, 0.02, device="cuda") for i, shp in enumerate(shapes)]
    outs, guards = [], []
    for shp in shapes:
        n = shp[0] * shp[1]
        (b0, codes), (b1, dqc), (b2, dqs) = (guarded((n // 2,), torch.uint8), guarded((n // 64,), torch.uint8),
                                             guarded(((n // 64 + 255) // 256,), torch.float32))
        outs.append(q.NF4Weight(codes, dqc, dqs, *shp))
        guards += [b0, b1, b2]
    q.qlora_quantize_nf4_batch(W0s, outs=outs, dq_format=dq_format)
    assert q.qlora_quantize_status() == 0
    assert_guards(guards, "batch quantize")
    for i, (W0, w) in enumerate(zip(W0s, outs)):
        one = q.qlora_quantize_nf4(W0, dq_format=dq_format)
        for a, b in ((w.codes, one.codes), (w.dq_codes, one.dq_codes), (w.dq_scales, one.dq_scales)):
            assert torch.equal(a, b), f"job {i} {shapes[i]}"
        assert w.dq_format == dq_format
    # and the oracle on a few of them
    for i in (1, 3, 4):
        gpu = (outs[i].codes.cpu().numpy(), outs[i].dq_codes.cpu().numpy(), outs[i].dq_scales.cpu().numpy())
        assert_quant_equal(gpu, nf4.quantize_nf4(W0s[i].cpu().numpy(),
                                                 dq_format="u8" if dq_format == q.QLORA_DQ_U8 else "e4m3"),
                           f"batch job {i}")


def test_quantize_edge_cases():
    """All-zero blocks, -0.0, a single non-zero, dominant +-values, huge and tiny
    magnitudes, a subnormal absmax, and values at / next to every decision
    threshold (the division fast path's fallback)."""
    rng = np.random.default_rng(11)
    nblk = 256 * 3 + 40
    W = nf4.fl32(rng.normal(0, 0.02, (nblk, 64)))
    W[0] = 0.0
    W[1] = -0.0
    W[2] = 0.0
    W[2, 17] = 0.3
    W[3, 5] = -1.5
    W[4] *= 1e30
    W[5] *= 1e-30
    W[6] = nf4.fl32(rng.normal(0, 1, 64)) * np.float32(1e-40)      # subnormal values and absmax
    W[7, :] = np.float32(3e-39)
    W[7, 1] = -np.float32(1e-45)
    lv = nf4.nf4_codebook().astype(np.float64)
    mids = (lv[:-1] + lv[1:]) / 2
    b = 8
    for j, m in enumerate(mids):
        for a in (np.float32(0.05), np.float32(0.0371), np.float32(1.7e-3), np.float32(0.123456)):
            row = nf4.fl32(rng.normal(0, 0.01, 64))
            row[0] = a
            c = np.float32(m * float(a))
            vals = [c, np.nextafter(c, np.float32(-1)), np.nextafter(c, np.float32(1)),
                    np.nextafter(np.nextafter(c, np.float32(1)), np.float32(1)),
                    np.nextafter(np.nextafter(c, np.float32(-1)), np.float32(-1))]
            for i, v in enumerate(vals):
                row[1 + i] = v
                row[10 + i] = -v
            W[b] = row
            b += 1
    assert b < nblk
    W0 = torch.from_numpy(W.reshape(-1, 128).copy())
    _, gpu, ref = quantize_both(W0)
    assert_quant_equal(gpu, ref, "edge")


@pytest.mark.parametrize("shape", [(4096, 4096), (4096, 11008), (11008, 4096)])
def test_quantize_bitexact_full_sizes(shape):
    """The projection shapes of the benchmarks, every code compared."""
    W0 = synth.normal(f"full{shape}", shape, 0.02, device="cuda").cpu()
    _, gpu, ref = quantize_both(W0)
    assert_quant_equal(gpu, ref, str(shape))


@pytest.mark.parametrize("shape", [(256, 256), (320, 192), (4096, 11008)])
def test_dequantize_bitexact(shape):
    W0 = synth.normal(f"deq{shape}", shape, 0.02)
    w, gpu, ref = quantize_both(W0)
    want = nf4.dequantize(*gpu, *shape)
    got32 = q.qlora_dequantize(w, torch.float32).cpu().numpy()
    got16 = q.qlora_dequantize(w, torch.bfloat16).float().cpu().numpy()
    assert np.array_equal(got32.view(np.uint32), want.view(np.uint32))
    assert np.array_equal(got16.view(np.uint32), nf4.round_bf16(want).view(np.uint32))


@pytest.mark.parametrize("n_in,n_out,r", [(256, 256, 8), (320, 192, 24), (128, 320, 72), (4096, 4096, 16)])
def test_merge_matches_oracle(n_in, n_out, r):
    t = synth.layer_inputs(n_in, n_out, 1, r)
    w, gpu, _ = quantize_both(t["W0"])
    A, B = t["A"].cuda(), t["B"].cuda()
    ref = linear.merge(nf4.dequantize(*gpu, n_in, n_out), t["A"], t["B"])
    got32 = q.qlora_merge(w, A, B, torch.float32)
    got16 = q.qlora_merge(w, A, B, torch.bfloat16)
    assert_close(got32, ref, "merge fp32", rel_fro=1e-6, max_abs=1e-5)
    assert_close(got16, ref, "merge bf16")


def test_frozen_weight_untouched_by_merge_and_dequant():
    t = synth.layer_inputs(256, 256, 1, 8)
    w, _, _ = quantize_both(t["W0"])
    snap = [x.clone() for x in (w.codes, w.dq_codes, w.dq_scales)]
    q.qlora_merge(w, t["A"].cuda(), t["B"].cuda())
    q.qlora_dequantize(w, torch.bfloat16)
    torch.cuda.synchronize()
    assert all(torch.equal(a, b) for a, b in zip(snap, (w.codes, w.dq_codes, w.dq_scales)))
