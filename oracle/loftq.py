"""Merge -> re-quantize round trip, and the LoftQ-style initialisation of the
adapters (float64 oracle).

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

* "QLoRA (low-rank adapters on a quantized model)", "What the simulations show":
  the merged Wq + A B is a dense float matrix, off the quantization grid; to keep
  the memory savings one either keeps the adapters separate or re-quantizes the
  merged weight and accepts some loss ("When it breaks": re-quantizing can throw
  away much of what the adapters learned, their corrections often being smaller
  than one quantization step).  ``requantize_merged`` is that round trip:
  W' = deq(Q(deq(Wq) + A B)), with the same NF4 + double-quant quantiser.
* Same page, "Going further": LoftQ and similar methods start A and B from an SVD
  of W0 - Q(W0) instead of zero.  Reading: the rank-r truncated SVD of the
  residual R = W0 - deq(Q(W0)) = U S V^T, split symmetrically, A = U_r S_r^1/2,
  B = S_r^1/2 V_r^T (the page fixes the product A B, not the split).
  ``split_adapters`` restates that split in the precision of stored adapters
  (fp32 square roots and products, bf16 results), the step a GPU kernel takes
  from a given decomposition.
"""

from __future__ import annotations

import numpy as np

from oracle import linear, nf4


def _f64(a) -> np.ndarray:
    if hasattr(a, "detach"):
        a = a.detach().double().cpu().numpy()
    return np.asarray(a, dtype=np.float64)


def residual(W0):
    """R = W0 - deq(Q(W0)) with the oracle's own quantiser (fp32 W0)."""
    W0 = np.asarray(W0, dtype=np.float32)
    n_in, n_out = W0.shape
    codes, dqc, dqs = nf4.quantize_nf4(W0)
    return W0.astype(np.float64) - nf4.dequantize(codes, dqc, dqs, n_in, n_out).astype(np.float64)


def loftq_init(W0, r: int):
    """Returns (A (in x r), B (r x out)) in float64: the rank-r truncated SVD of
    the quantisation residual, split symmetrically."""
    R = residual(W0)
    U, S, Vt = np.linalg.svd(R, full_matrices=False)
    root = np.sqrt(S[:r])
    return U[:, :r] * root[None, :], root[:, None] * Vt[:r, :]


def split_adapters(U, S, Vt, r: int):
    """The symmetric split in the library's precision: each of the r largest
    singular values is square-rooted in fp32 (s = fl32(sqrt(S_j)), the correctly
    rounded square root), A[i][j] = bf16(fl32(U[i][j] s_j)) and
    B[j][o] = bf16(fl32(s_j Vt[j][o])) (adapters are stored in bf16).  U, S, Vt
    are fp32 values; returns (A, B) as float32 arrays holding bf16 values.  Every
    fl32 is one exact float64 operation rounded once (exact products of two fp32
    values; for the square root the float64 double rounding is innocuous)."""
    U = np.asarray(U, np.float32).astype(np.float64)
    S = np.asarray(S, np.float32).astype(np.float64)
    Vt = np.asarray(Vt, np.float32).astype(np.float64)
    s = nf4.fl32(np.sqrt(S[:r])).astype(np.float64)
    A = nf4.round_bf16(nf4.fl32(U[:, :r] * s[None, :]))
    B = nf4.round_bf16(nf4.fl32(s[:, None] * Vt[:r, :]))
    return A, B


def requantize_merged(Wq, A, B):
    """The round trip: quantise the fp32 merge deq(Wq) + A B again; returns the
    dequantised result (float64) and the (codes, dq codes, scales) triple."""
    M = linear.merge(Wq, A, B).astype(np.float32)
    n_in, n_out = M.shape
    codes, dqc, dqs = nf4.quantize_nf4(M)
    return nf4.dequantize(codes, dqc, dqs, n_in, n_out).astype(np.float64), (codes, dqc, dqs)


def lost_fraction(Wq, A, B, W_round) -> float:
    """|| W_round - (Wq + A B) ||_F / || A B ||_F: how much of the adapters' product
    the round trip fails to keep (0 = all kept)."""
    AB = _f64(A) @ _f64(B)
    return float(np.linalg.norm(_f64(W_round) - (_f64(Wq) + AB)) / np.linalg.norm(AB))
