"""Pins of the NF4 / double-quantisation oracle against what the pages and the
mathematics fix (CPU only).  Each test names what it would catch."""

import math

import numpy as np
import pytest
import torch
from scipy.special import ndtr, ndtri

from oracle import nf4
from tests.conftest import read_golden


# ---------------------------------------------------------------- codebook

def test_codebook_shape_and_invariants():
    """16 levels, strictly ascending, ends exactly -1 and +1, an exact zero at code 7
    ("What QLoRA adds over LoRA": 16 levels at normal quantiles; "LoRA & QLoRA":
    table 0000 = -1.0, 0111 = 0.0)."""
    lv = nf4.nf4_codebook()
    assert lv.dtype == np.float32 and lv.shape == (16,)
    assert np.all(np.diff(lv.astype(np.float64)) > 0)
    assert lv[0] == -1.0 and lv[15] == 1.0 and lv[7] == 0.0
    assert np.sum(lv < 0) == 7 and np.sum(lv > 0) == 8


def test_codebook_matches_printed_table():
    """The legible rows of the page's NF4 value table ("LoRA & QLoRA",
    "4-bit NormalFloat (NF4)") to the 3 printed decimals; catches a wrong
    quantile offset, a swapped half or an off-by-one in the level order."""
    lv = nf4.nf4_codebook().astype(np.float64)
    checked = 0
    for code, value, status in read_golden("nf4_table_codewithdark.txt"):
        v = float(value)
        if status == "ok":
            assert abs(lv[int(code, 2)] - v) <= 5e-4 + 1e-9, (code, lv[int(code, 2)], v)
            checked += 1
        elif status == "value":
            assert np.min(np.abs(lv - v)) <= 5e-4 + 1e-9, (code, v)
            checked += 1
    assert checked == 8


def test_codebook_levels_are_normal_quantiles():
    """Each level times the top quantile maps back, through the normal CDF of a
    second library (scipy), onto the evenly spaced probabilities of the
    construction: 8 on the positive side, 7 on the negative side."""
    lv = nf4.nf4_codebook().astype(np.float64)
    top = ndtri(nf4.DELTA)
    p_pos = ndtr(lv[8:] * top)
    p_neg = ndtr(-lv[:7] * top)
    assert np.allclose(np.sort(p_pos)[::-1], np.linspace(nf4.DELTA, 0.5, 9)[:-1], atol=2e-7)
    assert np.allclose(np.sort(p_neg)[::-1], np.linspace(nf4.DELTA, 0.5, 8)[:-1], atol=2e-7)


def test_codebook_levels_unambiguous_in_fp32():
    """Every level sits well inside its fp32 rounding interval, so the float32
    codebook does not depend on the inverse-CDF routine's last bits."""
    from statistics import NormalDist
    nd = NormalDist()
    top = nd.inv_cdf(nf4.DELTA)
    exact = sorted([nd.inv_cdf(p) / top for p in np.linspace(nf4.DELTA, 0.5, 9)[:-1]]
                   + [0.0] + [-nd.inv_cdf(p) / top for p in np.linspace(nf4.DELTA, 0.5, 8)[:-1]])
    lv = nf4.nf4_codebook()
    for e, f in zip(exact, lv):
        if f == 0 or abs(f) == 1:
            continue
        ulp = float(np.spacing(np.float32(abs(f))))
        assert abs(e - float(f)) / ulp < 0.49


# ---------------------------------------------------------------- encode

def test_nearest_level_brute_force_random():
    """Counting midpoints equals a direct argmin in exact rationals (ties low)."""
    rng = np.random.default_rng(1)
    lv = nf4.nf4_codebook()
    x = nf4.fl32(rng.uniform(-1, 1, 3000))
    got = nf4.nearest_level(x, lv)
    want = [nf4.nearest_level_exact(float(v), lv) for v in x]
    assert np.array_equal(got, np.array(want, dtype=np.uint8))


def test_nearest_level_adversarial_midpoints():
    """Values on, just below and just above every midpoint: a tie keeps the lower
    level (argmin returns the first minimum, "LLMs · QLoRA" ``quantise``)."""
    lv = nf4.nf4_codebook()
    l64 = lv.astype(np.float64)
    xs = []
    for j in range(15):
        m = (l64[j] + l64[j + 1]) / 2
        f = np.float32(m)
        xs += [f, np.nextafter(f, np.float32(-2)), np.nextafter(f, np.float32(2))]
        if float(f) == m:                       # midpoint exactly representable
            xs += [f]
    xs += [np.float32(-1), np.float32(1), np.float32(0), np.float32(-0.0)]
    xs = np.array(xs, dtype=np.float32)
    got = nf4.nearest_level(xs, lv)
    want = [nf4.nearest_level_exact(float(v), lv) for v in xs]
    assert np.array_equal(got, np.array(want, dtype=np.uint8))


def test_blockwise_special_values():
    """The absmax element codes to 0 or 15, zeros (and -0.0) code to 7, an
    all-zero block codes to 7 everywhere; absmax is the exact max |w|."""
    rng = np.random.default_rng(2)
    w = nf4.fl32(rng.normal(0, 0.02, (8, 64)))
    w[0, 5] = 0.0
    w[1, 9] = -0.0
    w[2, :] = 0.0
    w[3, :] = -0.0
    w[4, 17] = 0.5                   # dominant positive element
    w[5, 33] = -0.5                  # dominant negative element
    a = nf4.block_absmax(w)
    assert np.array_equal(a, np.max(np.abs(w), axis=1))
    codes = nf4.nearest_level(nf4.scaled(w, a), nf4.nf4_codebook()).reshape(8, 64)
    assert codes[0, 5] == 7 and codes[1, 9] == 7
    assert np.all(codes[2] == 7) and np.all(codes[3] == 7)
    assert codes[4, 17] == 15 and codes[5, 33] == 0
    big = np.argmax(np.abs(w), axis=1)
    for b in (0, 1, 6, 7):
        assert codes[b, big[b]] in (0, 15)


def test_blog_experiment_reproduces_printed_errors():
    """The experiment of "LLMs · QLoRA" on a numpy stream: mean-abs
    reconstruction errors within 3% of the printed 1.71e-3 (uniform) and
    1.46e-3 (NF4-style), least-used level shares within 0.1 percentage point of
    1.13% / 1.98% (the page's torch stream is not reproduced)."""
    gold = {k: float(v) for k, v in read_golden("blog_quantiser_output.txt")}
    rng = np.random.default_rng(0)
    w = nf4.fl32(rng.standard_normal(4096 * 64) * 0.02)
    for name, lv in (("uniform4", nf4.uniform4_codebook()), ("nf4style", nf4.blog_codebook())):
        deq, codes = nf4.quantise_blockwise(w, lv)
        err = float(np.mean(np.abs(deq.astype(np.float64) - w.astype(np.float64))))
        use = np.bincount(codes, minlength=16)
        share = use.min() / use.sum()
        assert math.isclose(err, gold[name + ".mean_abs_error"], rel_tol=0.03), (name, err)
        assert abs(share - gold[name + ".least_used_share"]) < 1e-3, (name, share)


def test_blog_codebooks_shape():
    """The approximate codebook is symmetric with no zero level; the uniform grid
    has step 2/15 ("LLMs · QLoRA" listing)."""
    b = nf4.blog_codebook().astype(np.float64)
    assert np.allclose(b, -b[::-1], atol=1e-7) and np.min(np.abs(b)) > 0 and b.max() == 1.0
    u = nf4.uniform4_codebook().astype(np.float64)
    assert np.allclose(np.diff(u), 2 / 15, atol=1e-7)


def test_weight_memory_arithmetic():
    """7e9 weights at 16 / 8 / 4 bits: the printed 14.0 / 7.0 / 3.5 GB."""
    gold = {k: float(v) for k, v in read_golden("blog_quantiser_output.txt")}
    for bits in (16, 8, 4):
        assert round(7e9 * bits / 8 / 1e9, 1) == gold[f"weights_7b_{bits}bit_gb"]


# ---------------------------------------------------------------- E4M3

def test_e4m3_exhaustive_roundtrip_and_midpoints():
    """All 127 finite non-negative codes decode and re-encode to themselves; each
    midpoint between neighbours goes to the even code; above 448 saturates."""
    codes = np.arange(0x7F)
    vals = nf4.e4m3_decode(codes)
    assert vals[0] == 0 and vals[0x7E] == 448.0 and vals[1] == 2.0 ** -9
    assert np.all(np.diff(vals) > 0)
    assert np.array_equal(nf4.e4m3_encode(vals), codes.astype(np.uint8))
    mids = (vals[:-1] + vals[1:]) / 2
    enc = nf4.e4m3_encode(mids)
    lower = codes[:-1]
    want = np.where(lower % 2 == 0, lower, lower + 1)
    assert np.array_equal(enc, want.astype(np.uint8))
    assert np.all(nf4.e4m3_encode(np.array([448.0, 460.0, 464.0, 1e6])) == 0x7E)
    assert np.isnan(nf4.e4m3_decode(0x7F)) and nf4.e4m3_decode(0xB8) == -1.0


def test_e4m3_matches_torch_float8():
    """Against torch's float8_e4m3fn cast (RNE) on random and tie values below the
    saturation range."""
    rng = np.random.default_rng(3)
    vals = nf4.e4m3_decode(np.arange(0x7F))
    mids = (vals[:-1] + vals[1:]) / 2
    y = np.concatenate([rng.uniform(0, 460, 20000), np.exp(rng.uniform(-14, 6, 20000)), mids])
    y = nf4.fl32(y)
    y = y[y < 464]
    ref = torch.from_numpy(y).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(nf4.e4m3_encode(y.astype(np.float64)), ref)


# ---------------------------------------------------------------- double quant

def test_double_quant_bits_per_weight():
    """4 + 8/64 + 32/(64*256) = 4.127 bits; saving against an fp32 absmax per
    block is 0.373 bit ("about 0.37 bits per weight", "What QLoRA adds over LoRA")."""
    b = nf4.bits_per_weight()
    assert math.isclose(b, 4.126953125)
    saving = (4 + 32 / 64) - b
    assert round(saving, 2) == 0.37


def test_double_quant_properties():
    """Group max codes to 448 (0x7E); relative absmax error <= 2^-4 on normal
    weights; a zero group stores zero scale and codes; partial last group."""
    rng = np.random.default_rng(4)
    w = nf4.fl32(rng.normal(0, 0.02, 64 * (256 * 3 + 100)))
    a = nf4.block_absmax(w)
    a[256:512] = 0.0                                  # second group all zero
    c, s = nf4.double_quant(a)
    assert s.shape == (4,) and c.shape == a.shape
    assert s[1] == 0 and np.all(c[256:512] == 0)
    for g in (0, 2, 3):
        seg = slice(256 * g, 256 * (g + 1))
        assert c[seg][np.argmax(a[seg])] == 0x7E
        assert s[g] == np.float32(np.float64(a[seg].max()) / 448.0)
    a2 = nf4.absmax_dequant(c, s).astype(np.float64)
    nz = a > 0
    rel = np.abs(a2[nz] - a[nz]) / a[nz]
    assert rel.max() <= 2 ** -4 * (1 + 1e-6)


def test_double_quant_hand_example():
    """A hand-worked group: absmax {448, 1, 0.3} with scale 1 -> codes 0x7E, 0x38,
    and 0.3 -> nearest E4M3 0.3125 (0x2A)."""
    a = np.array([448.0, 1.0, 0.3], dtype=np.float32)
    c, s = nf4.double_quant(a)
    assert s[0] == 1.0
    assert list(c) == [0x7E, 0x38, 0x2A]


# ---------------------------------------------------------------- full quantize + dequantize

def test_quantize_roundtrip_error_bound_and_packing():
    """Dequantised weights stay within half the widest level gap times absmax
    plus the absmax error; packing puts element 2k in the low nibble."""
    rng = np.random.default_rng(5)
    W = nf4.fl32(rng.normal(0, 0.02, (128, 192)))
    codes, dqc, dqs = nf4.quantize_nf4(W)
    assert codes.shape == (128 * 192 // 2,) and dqc.shape == (384,) and dqs.shape == (2,)
    Wd = nf4.dequantize(codes, dqc, dqs, 128, 192).astype(np.float64)
    lv = nf4.nf4_codebook().astype(np.float64)
    gap = np.max(np.diff(lv)) / 2
    a = nf4.block_absmax(W).astype(np.float64)
    a2 = nf4.absmax_dequant(dqc, dqs).astype(np.float64)
    err = np.abs(Wd.reshape(-1, 64) - W.reshape(-1, 64).astype(np.float64))
    bound = a[:, None] * gap + np.abs(a - a2)[:, None] + 1e-7
    assert np.all(err <= bound)
    flat = nf4.unpack_nibbles(codes)
    x = nf4.scaled(W, nf4.block_absmax(W))
    assert np.array_equal(flat, nf4.nearest_level(x, lv).reshape(-1))
    assert codes[0] == (flat[0] | (flat[1] << 4))


def test_dequantize_hand_built():
    """Hand-built codes and constants: code byte 0x2F puts level 15 then level 2;
    E4M3 0x38 = 1.0 times scale 0.5 gives absmax' 0.5."""
    lv = nf4.nf4_codebook().astype(np.float64)
    codes = np.zeros(32, dtype=np.uint8)
    codes[0] = 0x2F
    dqc = np.array([0x38], dtype=np.uint8)
    dqs = np.array([0.5], dtype=np.float32)
    Wd = nf4.dequantize(codes, dqc, dqs, 1, 64).reshape(-1).astype(np.float64)
    assert Wd[0] == 0.5 and Wd[1] == np.float32(lv[2] * 0.5) and np.all(Wd[2:] == -0.5)


def test_round_bf16_matches_torch():
    """Bit-pattern RNE to bfloat16 equals torch's cast, ties included."""
    rng = np.random.default_rng(6)
    x = nf4.fl32(np.concatenate([rng.normal(0, 1, 50000), rng.normal(0, 1e-3, 50000)]))
    u = x.view(np.uint32)
    ties = ((u & np.uint32(0xFFFF0000)) | np.uint32(0x8000)).view(np.float32)
    x = np.concatenate([x, ties])
    ref = torch.from_numpy(x).to(torch.bfloat16).float().numpy()
    assert np.array_equal(nf4.round_bf16(x), ref)


def test_quantize_rejects_bad_input():
    with pytest.raises(ValueError):
        nf4.quantize_nf4(np.full((2, 64), np.nan, dtype=np.float32))
    with pytest.raises(ValueError):
        nf4.quantize_nf4(np.zeros((3, 7), dtype=np.float32))


# ---------------------------------------------------------------------------
# the linear-uint8 reading of the 8-bit double quantisation


def test_u8_double_quant_grid_points_and_ends():
    """Values on the grid k * s come back as code k; the group maximum is code
    255 and zero is code 0; the scale is fl32(max / 255)."""
    top = np.float32(3.0)
    s = np.float32(np.float64(top) / 255.0)
    ks = np.array([0, 1, 2, 17, 128, 200, 254], dtype=np.int64)
    vals = (ks.astype(np.float64) * np.float64(s)).astype(np.float32)
    a = np.concatenate([vals, [top]]).astype(np.float32)
    codes, scales = nf4.double_quant(a, dq_format="u8")
    assert scales[0] == s
    assert list(codes[:-1]) == list(ks) and codes[-1] == 255


def test_u8_double_quant_ties_to_even():
    """Half-way values (k + 1/2) s, exactly representable, round to the even
    neighbour (a round-half-up coder would give k + 1 for every even k)."""
    s = np.float32(0.25)                       # max = 63.75 -> s = 0.25 exactly
    top = np.float32(63.75)
    a = np.array([top] + [(k + 0.5) * 0.25 for k in range(0, 20)], dtype=np.float32)
    codes, scales = nf4.double_quant(a, dq_format="u8")
    assert scales[0] == s
    for k in range(20):
        assert codes[1 + k] == (k if k % 2 == 0 else k + 1), k


def test_u8_double_quant_error_bound_and_monotone():
    """Decoded absmax within half a step (plus rounding) of the exact value, and
    codes non-decreasing in the absmax, on a group of random values."""
    rng = np.random.default_rng(11)
    a = np.sort(rng.uniform(0.0, 0.07, 256)).astype(np.float32)
    codes, scales = nf4.double_quant(a, dq_format="u8")
    dec = nf4.absmax_dequant(codes, scales, dq_format="u8").astype(np.float64)
    s = float(scales[0])
    assert np.all(np.abs(dec - a.astype(np.float64)) <= 0.5 * s * (1 + 1e-6) + 1e-9)
    assert np.all(np.diff(codes.astype(int)) >= 0)


def test_u8_zero_group_and_weight_codes_independent_of_format():
    """An all-zero group has scale 0 and codes 0; the packed NF4 weight codes are
    the same in both formats (they use the exact absmax), only the stored absmax
    differs."""
    codes, scales = nf4.double_quant(np.zeros(300, np.float32), dq_format="u8")
    assert not np.any(codes) and not np.any(scales)
    W = np.random.default_rng(2).standard_normal((64, 512)).astype(np.float32) * 0.02
    c8, q8, s8 = nf4.quantize_nf4(W, dq_format="e4m3")
    cu, qu, su = nf4.quantize_nf4(W, dq_format="u8")
    assert np.array_equal(c8, cu)
    assert not np.array_equal(q8, qu)


def test_u8_more_precise_for_large_blocks():
    """Where a group's absmax values all lie in [max/2, max] the linear code's
    relative error (<= 1/255) is below E4M3's worst case (2^-4), and on such a
    group it is smaller on average."""
    rng = np.random.default_rng(5)
    a = rng.uniform(0.5, 1.0, 256).astype(np.float32)
    cu, su = nf4.double_quant(a, dq_format="u8")
    ce, se = nf4.double_quant(a, dq_format="e4m3")
    eu = np.abs(nf4.absmax_dequant(cu, su, dq_format="u8") - a) / a
    ee = np.abs(nf4.absmax_dequant(ce, se) - a) / a
    assert eu.max() <= 1 / 255 * (1 + 1e-6) and ee.max() <= 2 ** -4
    assert eu.mean() < ee.mean()


def test_unknown_dq_format_rejected():
    with pytest.raises(ValueError):
        nf4.double_quant(np.ones(4, np.float32), dq_format="fp16")
