"""Pins of the symmetric uniform INT quantiser with one scale per 16 weights
(CPU only): grid points, ties to even, the half-step error bound, the ternary
values of the 2-bit case, the code ranges per bit width, zero groups, and the
error ordering of the 2/3/4-bit workloads."""

import numpy as np
import pytest

from oracle import intq, nf4


def _group(values):
    return np.asarray(values, dtype=np.float32).reshape(1, 16)


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_grid_points_come_back_exactly(bits):
    """w = k s for every k in -Q .. Q (group max Q s) is coded as k and
    reconstructed exactly."""
    Q = intq.qmax(bits)
    s = np.float32(0.125)                                   # max Q s / Q = s exactly
    ks = np.array(list(range(-Q, Q + 1)) + [Q] * (16 - (2 * Q + 1)), dtype=np.int64)
    W = _group(ks * 0.125)
    codes, scales = intq.quantize_int(W, bits)
    assert scales[0] == s
    assert np.array_equal(nf4.unpack_nibbles(codes).astype(int) - 8, ks)
    assert np.array_equal(intq.dequantize_int(codes, scales, 1, 16), W)


def test_ties_to_even():
    """4 bits, s = 1: w = k + 1/2 rounds to the even neighbour."""
    vals = [7.0, 0.5, 1.5, 2.5, 3.5, -0.5, -1.5, -2.5, -3.5, 4.5, 5.5, 6.5, -4.5, -5.5, -6.5, 0.0]
    codes, scales = intq.quantize_int(_group(vals), 4)
    assert scales[0] == 1.0
    q = nf4.unpack_nibbles(codes).astype(int) - 8
    want = [7, 0, 2, 2, 4, 0, -2, -2, -4, 4, 6, 6, -4, -6, -6, 0]
    assert list(q) == want


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_error_bound_and_code_range(bits):
    """Every reconstruction within half a step of the weight; codes confined to
    8 - Q .. 8 + Q; the 2-bit case produces only {-s, 0, s}."""
    rng = np.random.default_rng(bits)
    W = rng.normal(0, 0.02, (32, 64)).astype(np.float32)
    codes, scales = intq.quantize_int(W, bits)
    deq = intq.dequantize_int(codes, scales, 32, 64).reshape(-1, 16).astype(np.float64)
    s = scales.astype(np.float64)[:, None]
    err = np.abs(deq - W.reshape(-1, 16).astype(np.float64))
    assert np.all(err <= 0.5 * s * (1 + 1e-6) + 1e-12)
    c = nf4.unpack_nibbles(codes).astype(int)
    Q = intq.qmax(bits)
    assert c.min() >= 8 - Q and c.max() <= 8 + Q
    if bits == 2:
        r = deq / np.where(s > 0, s, 1.0)
        assert set(np.unique(np.round(r, 12))) <= {-1.0, 0.0, 1.0}


def test_zero_group_and_group_max():
    """An all-zero group has scale 0 and codes 8 (q = 0); the group's largest
    magnitude maps to +-Q."""
    W = np.zeros((2, 16), np.float32)
    W[1] = np.linspace(-0.3, 0.2, 16, dtype=np.float32)
    codes, scales = intq.quantize_int(W, 3)
    q = nf4.unpack_nibbles(codes).astype(int) - 8
    assert scales[0] == 0.0 and not np.any(q[:16])
    assert q[16] == -3                                      # -0.3 is the group's absmax


def test_more_bits_less_error():
    """On N(0, 0.02) weights the mean reconstruction error falls with the bit
    width, and at 4 bits with group 16 it is below NF4's with block 64 (the
    finer scales of the pages' simulation)."""
    rng = np.random.default_rng(0)
    W = rng.normal(0, 0.02, (128, 256)).astype(np.float32)
    errs = []
    for b in (2, 3, 4):
        c, s = intq.quantize_int(W, b)
        errs.append(np.mean(np.abs(intq.dequantize_int(c, s, 128, 256) - W)))
    assert errs[0] > errs[1] > errs[2]
    codes, dqc, dqs = nf4.quantize_nf4(W)
    e_nf4 = np.mean(np.abs(nf4.dequantize(codes, dqc, dqs, 128, 256) - W))
    assert errs[2] < e_nf4


def test_bad_arguments():
    with pytest.raises(ValueError):
        intq.qmax(5)
    with pytest.raises(ValueError):
        intq.quantize_int(np.ones(24, np.float32), 4)
