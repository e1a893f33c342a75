"""Pins of the merge -> re-quantize round trip and the LoftQ-style initialisation
oracle (CPU only): the Eckart-Young optimum, exact reconstruction at full rank,
idempotence of the quantiser on its own grid, and the pages' claim that small
adapter corrections are mostly lost by re-quantization."""

import numpy as np
import pytest

import synth
from oracle import loftq, nf4


def _w0(n_in=128, n_out=192, seed=0, tag="loftq"):
    return synth.layer_inputs(n_in, n_out, 8, 8, seed=seed, tag=tag)["W0"].numpy()


@pytest.mark.parametrize("r", [1, 4, 16])
def test_init_reaches_the_eckart_young_optimum(r):
    """A B is the best rank-r approximation of the residual: the remaining error
    is the root sum of the discarded squared singular values (computed here from
    numpy's singular values, not from the oracle's factors)."""
    W0 = _w0()
    R = loftq.residual(W0)
    A, B = loftq.loftq_init(W0, r)
    s = np.linalg.svd(R, compute_uv=False)
    assert np.isclose(np.linalg.norm(R - A @ B), np.sqrt(np.sum(s[r:] ** 2)), rtol=1e-10)
    # and it never does worse than starting from zero adapters
    assert np.linalg.norm(R - A @ B) < np.linalg.norm(R)


def test_full_rank_init_reconstructs_W0():
    """With r = min(in, out) the adapters absorb the whole residual:
    deq(Q(W0)) + A B = W0 up to float64 rounding."""
    W0 = _w0(64, 96)
    A, B = loftq.loftq_init(W0, 64)
    codes, dqc, dqs = nf4.quantize_nf4(W0)
    Wq = nf4.dequantize(codes, dqc, dqs, 64, 96).astype(np.float64)
    np.testing.assert_allclose(Wq + A @ B, W0.astype(np.float64), rtol=0, atol=1e-12)


def test_symmetric_split():
    """A = U_r S^1/2 and B = S^1/2 V_r^T: A^T A = B B^T = diag(S_r)."""
    W0 = _w0()
    A, B = loftq.loftq_init(W0, 6)
    s = np.linalg.svd(loftq.residual(W0), compute_uv=False)[:6]
    np.testing.assert_allclose(A.T @ A, np.diag(s), atol=1e-12 * s[0])
    np.testing.assert_allclose(B @ B.T, np.diag(s), atol=1e-12 * s[0])


def test_round_trip_with_zero_adapters_is_idempotent():
    """Re-quantizing an unchanged NF4 weight gives back the same codes, absmax
    codes and scales: every block keeps its absmax at a +-1 level and every
    group its maximum at E4M3's 448."""
    W0 = _w0(256, 256)
    codes, dqc, dqs = nf4.quantize_nf4(W0)
    Wq = nf4.dequantize(codes, dqc, dqs, 256, 256)
    W_round, (c2, q2, s2) = loftq.requantize_merged(Wq, np.zeros((256, 4)), np.zeros((4, 256)))
    assert np.array_equal(c2, codes) and np.array_equal(q2, dqc) and np.array_equal(s2.view(np.uint32),
                                                                                   dqs.view(np.uint32))
    assert np.array_equal(W_round, Wq.astype(np.float64))


def test_small_corrections_are_mostly_lost():
    """The page's warning: adapters at the scale of the configs (B ~ 0.01 N(0,1),
    A ~ N(0,1)/sqrt(in)) change the weight by much less than one quantization
    step, so the round trip keeps little of A B; a correction the size of a step
    survives far better."""
    t = synth.layer_inputs(256, 256, 8, 16, seed=1, tag="round")
    codes, dqc, dqs = nf4.quantize_nf4(t["W0"].numpy())
    Wq = nf4.dequantize(codes, dqc, dqs, 256, 256)
    A, B = t["A"].double().numpy(), t["B"].double().numpy()
    W_round, _ = loftq.requantize_merged(Wq, A, B)
    small = loftq.lost_fraction(Wq, A, B, W_round)
    W_big, _ = loftq.requantize_merged(Wq, A, 30 * B)
    big = loftq.lost_fraction(Wq, A, 30 * B, W_big)
    assert small > 0.5          # most of a small correction is lost
    assert big < small / 2      # a larger one is kept much better


def test_split_adapters_exact_on_representable_values():
    """Square roots and products that are exact in fp32 and bf16 (singular values
    16, 4, 2.25, 0.25; factors with a few significant bits): the split gives
    U s and s Vt exactly, as computed here with rationals."""
    from fractions import Fraction
    S = np.array([16.0, 4.0, 2.25, 0.25, 9.0], np.float32)
    roots = [Fraction(4), Fraction(2), Fraction(3, 2), Fraction(1, 2)]
    rng = np.random.default_rng(3)
    vals = np.array([1.0, -1.0, 0.5, -0.75, 0.125, 1.5, -0.375, 0.0], np.float32)
    U = vals[rng.integers(0, len(vals), (6, 5))]
    Vt = vals[rng.integers(0, len(vals), (5, 7))]
    A, B = loftq.split_adapters(U, S, Vt, 4)
    for i in range(6):
        for j in range(4):
            assert Fraction(float(A[i, j])) == Fraction(float(U[i, j])) * roots[j]
    for j in range(4):
        for o in range(7):
            assert Fraction(float(B[j, o])) == roots[j] * Fraction(float(Vt[j, o]))
    assert A.shape == (6, 4) and B.shape == (4, 7)


def test_split_adapters_product_and_gram_within_bf16_rounding():
    """On an exact SVD of a random matrix (fp32 factors), A B equals the rank-r
    truncation U_r diag(S_r) Vt_r, and A^T A equals diag(S_r), each within the
    rounding of bf16 storage (relative 2^-8 per factor)."""
    rng = np.random.default_rng(4)
    R = rng.normal(size=(96, 80))
    U, S, Vt = np.linalg.svd(R, full_matrices=False)
    U32, S32, Vt32 = U.astype(np.float32), S.astype(np.float32), Vt.astype(np.float32)
    r = 12
    A, B = loftq.split_adapters(U32, S32, Vt32, r)
    ref = (U32[:, :r].astype(np.float64) * S32[:r].astype(np.float64)) @ Vt32[:r].astype(np.float64)
    bound = 2 * 2.0 ** -8 * (np.abs(U32[:, :r]) * S32[:r]) @ np.abs(Vt32[:r])
    assert np.all(np.abs(A.astype(np.float64) @ B.astype(np.float64) - ref) <= bound + 1e-12)
    gram = A.astype(np.float64).T @ A.astype(np.float64)
    np.testing.assert_allclose(np.diag(gram), S[:r], rtol=2 * 2.0 ** -8)


def test_split_adapters_agrees_with_the_float64_split():
    """The stored-precision split of the oracle's own SVD is the float64 split of
    loftq_init rounded: within 2^-7 relative, element by element."""
    W0 = _w0()
    R = loftq.residual(W0)
    U, S, Vt = np.linalg.svd(R, full_matrices=False)
    A, B = loftq.split_adapters(U.astype(np.float32), S.astype(np.float32), Vt.astype(np.float32), 8)
    A64, B64 = loftq.loftq_init(W0, 8)
    assert np.all(np.abs(A - A64) <= 2.0 ** -7 * np.abs(A64) + 1e-30)
    assert np.all(np.abs(B - B64) <= 2.0 ** -7 * np.abs(B64) + 1e-30)
