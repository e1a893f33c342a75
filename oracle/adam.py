"""Adam / AdamW step on the adapters only (float64 oracle).

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

"QLoRA (low-rank adapters on a quantized model)", "The code, line by line":
``opt = Adam(A + B, lr=lr)`` hands the optimizer only the adapter matrices, and
``opt.step(...)`` is given dA = dW B^T and dB = A^T dW; the frozen base never
changes.  "LoRA and QLoRA: Efficient Fine-Tuning Explained", "A real run",
trains the same way with ``torch.optim.AdamW(..., lr=1e-3)``.  Neither page
prints the update rule, so the reading is Adam (Kingma & Ba) with bias
correction, in the form torch uses, and AdamW's decoupled weight decay applied
before the moment step:

    theta <- theta * (1 - lr * wd)                    (wd = 0: plain Adam)
    m     <- beta1 m + (1 - beta1) g
    v     <- beta2 v + (1 - beta2) g^2
    theta <- theta - lr * (m / (1 - beta1^t)) / (sqrt(v / (1 - beta2^t)) + eps)

with t the 1-based step number.  Everything is float64 on the exact values of
the inputs.
"""

from __future__ import annotations

import numpy as np


def _f64(a) -> np.ndarray:
    if hasattr(a, "detach"):
        a = a.detach().double().cpu().numpy()
    return np.asarray(a, dtype=np.float64)


def adam_step(theta, g, m, v, t: int, lr: float, beta1: float = 0.9, beta2: float = 0.999,
              eps: float = 1e-8, weight_decay: float = 0.0):
    """One step on one parameter array; returns (theta', m', v') as new arrays."""
    if t < 1:
        raise ValueError("the step number t is 1-based")
    theta, g, m, v = _f64(theta), _f64(g), _f64(m), _f64(v)
    theta = theta * (1.0 - lr * weight_decay)
    m = beta1 * m + (1.0 - beta1) * g
    v = beta2 * v + (1.0 - beta2) * g * g
    m_hat = m / (1.0 - beta1 ** t)
    v_hat = v / (1.0 - beta2 ** t)
    theta = theta - lr * m_hat / (np.sqrt(v_hat) + eps)
    return theta, m, v


def adapter_adam_step(A, B, dA, dB, state: dict, t: int, **hp):
    """The adapters' step: A with dA and B with dB, each with its own moments
    (state keys mA, vA, mB, vB).  Returns (A', B', state')."""
    A1, mA, vA = adam_step(A, dA, state["mA"], state["vA"], t, **hp)
    B1, mB, vB = adam_step(B, dB, state["mB"], state["vB"], t, **hp)
    return A1, B1, {"mA": mA, "vA": vA, "mB": mB, "vB": vB}
