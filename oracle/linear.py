"""Forward, backward and merge of the QLoRA adapted linear layer (float64 oracle).

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

Layout follows "QLoRA (low-rank adapters on a quantized model)", "How it works":
the weight is stored as (in, out), A is (in x r), B is (r x out), so a row of
tokens X (M x in) maps to X @ W.

* Forward: Y = X Wq + (X A) B, with Wq the dequantised frozen base in bf16
  ("How it works", steps 1-2: W = Wq + A B; "What QLoRA adds over LoRA": the
  frozen weights are dequantised to bf16 for each matmul; "LoRA & QLoRA",
  "Mathematical Formulation": h = W0 x + B(A x), the transposed notation).
* Backward: dL/dA = dL/dW B^T and dL/dB = A^T dL/dW with dL/dW = X^T dY
  ("How it works", step 4; "The code, line by line": dA = dW B^T, dB = A^T dW).
  Written here in the factored form that never forms the (in x out) dW:
  U = dY B^T, dA = X^T U, dB = (X A)^T dY.  The input gradient,
  dX = dY Wq^T + U A^T, is what "Forward and backward as usual" (step 3) implies
  for a layer inside a network; Wq receives no update ("What QLoRA adds over
  LoRA", last paragraph).
* Dropout on the low-rank intermediate ("LoRA & QLoRA", "Dropout": dropout is
  applied to A x during training).  Reading: inverted dropout with a given keep
  mask (1 = keep) and drop probability p, V = s (X A) * keep / (1 - p), so that
  E[V] = s X A; the same mask enters the backward, U = (s keep / (1 - p)) *
  (dY B^T), and dB = V^T dY uses the dropped V.  The mask is an input: both the
  oracle and the CUDA path receive the same bytes.
* Merge: W = Wq + A B as a dense float matrix ("How it works", step 5).
* Adapter size r (in + out) per layer ("How it works", paragraph after step 5).

All arithmetic is float64 on the exact values of the (bf16 / fp32) inputs: no
rounding of the intermediate V = X A or U = dY B^T.
"""

from __future__ import annotations

import numpy as np


def _f64(a) -> np.ndarray:
    if hasattr(a, "detach"):            # a torch tensor from the input generator
        a = a.detach().float().cpu().numpy()
    return np.asarray(a, dtype=np.float64)


def _factor(scale: float, keep, p: float):
    """The factor each element of X A (and of dY B^T) is multiplied by: the
    adapter scale s, times keep / (1 - p) under dropout."""
    if keep is None:
        return scale
    if not 0.0 <= p < 1.0:
        raise ValueError("the drop probability must lie in [0, 1)")
    return scale * _f64(keep) / (1.0 - p)


def forward(X, A, B, Wq, scale: float = 1.0, keep=None, p: float = 0.0):
    """Returns (Y, V) with V = s X A and Y = X Wq + V B (float64); s is the
    adapter scale alpha / r of "LoRA & QLoRA", "Scaling Factor alpha"
    (h = W0 x + (alpha / r) B (A x)); 1 is the plain layer.  With a keep mask
    (M x r, 1 = keep) V is dropped out: V = s (X A) * keep / (1 - p)."""
    X, A, B, Wq = _f64(X), _f64(A), _f64(B), _f64(Wq)
    V = _factor(scale, keep, p) * (X @ A)
    Y = X @ Wq + V @ B
    return Y, V


def forward_rows(X, A, B, Wq, rows):
    """Y and V restricted to the given token rows (each row is independent)."""
    X = _f64(X)[np.asarray(rows)]
    return forward(X, A, B, Wq)


def backward(X, A, B, Wq, dY, scale: float = 1.0, keep=None, p: float = 0.0):
    """Returns dict(dX, dA, dB, U) for L with dL/dY = dY (float64), for the layer
    with adapter scale s: U = s dY B^T, dX = dY Wq^T + U A^T, dA = X^T U,
    dB = s (X A)^T dY.  Under dropout with keep mask `keep` the factor
    f = s keep / (1 - p) replaces s elementwise: U = f * (dY B^T), dB = V^T dY
    with V = f * (X A)."""
    X, A, B, Wq, dY = _f64(X), _f64(A), _f64(B), _f64(Wq), _f64(dY)
    f = _factor(scale, keep, p)
    U = f * (dY @ B.T)
    dX = dY @ Wq.T + U @ A.T
    dA = X.T @ U
    dB = (f * (X @ A)).T @ dY
    return {"dX": dX, "dA": dA, "dB": dB, "U": U}


def adapter_grads(X, A, B, dY):
    """dA = X^T (dY B^T) and dB = (X A)^T dY alone (no dX), for large token counts."""
    X, A, B, dY = _f64(X), _f64(A), _f64(B), _f64(dY)
    U = dY @ B.T
    return {"dA": X.T @ U, "dB": (X @ A).T @ dY}


def backward_dense(X, A, B, dY):
    """The pages' own route: dW = X^T dY, dA = dW B^T, dB = A^T dW."""
    X, A, B, dY = _f64(X), _f64(A), _f64(B), _f64(dY)
    dW = X.T @ dY
    return {"dA": dW @ B.T, "dB": A.T @ dW}


def dX_rows(A, B, Wq, dY, rows):
    """dX restricted to the given token rows."""
    A, B, Wq = _f64(A), _f64(B), _f64(Wq)
    dY = _f64(dY)[np.asarray(rows)]
    return dY @ Wq.T + (dY @ B.T) @ A.T


def merge(Wq, A, B):
    """W = Wq + A B (float64, (in, out))."""
    return _f64(Wq) + _f64(A) @ _f64(B)


def adapter_params(n_in: int, n_out: int, r: int) -> int:
    """Trainable adapter parameters of one layer: r (in + out)."""
    return r * (n_in + n_out)


def loss_inner(Y, dY) -> float:
    """L = <dY, Y>, whose gradient with respect to Y is dY (finite-difference pins)."""
    return float(np.sum(_f64(Y) * _f64(dY)))


def rel_fro(got, ref) -> float:
    """||got - ref||_F / ||ref||_F (0 when both are 0)."""
    got, ref = _f64(got), _f64(ref)
    den = np.linalg.norm(ref)
    num = np.linalg.norm(got - ref)
    if den == 0.0:
        return 0.0 if num == 0.0 else float("inf")
    return float(num / den)


def max_abs_ratio(got, ref) -> float:
    """max |got - ref| / max |ref| (0 when both are 0)."""
    got, ref = _f64(got), _f64(ref)
    den = np.max(np.abs(ref)) if ref.size else 0.0
    num = np.max(np.abs(got - ref)) if ref.size else 0.0
    if den == 0.0:
        return 0.0 if num == 0.0 else float("inf")
    return float(num / den)
