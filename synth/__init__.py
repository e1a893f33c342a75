"""Seeded synthetic inputs for the QLoRA linear layer.

Both the CUDA path's tests/benchmark and the float64 oracle take their inputs
from here; this module holds none of the method's arithmetic (no quantisation,
no matmul), only random draws.  Every tensor comes from its own stream keyed by
(seed, name), so a tensor's bytes do not depend on which other tensors were
drawn.  A stream on the CPU and one on a GPU differ; a test that compares the
two paths draws once and hands the same bytes to both.

Distributions follow the workloads the pages describe:

* W0 = fp32(0.02 * N(0, 1)): "LLMs · QLoRA", ``w = torch.randn(...) * 0.02``.
* X, dY = bf16(N(0, 1)).
* A = bf16(N(0, 1) / sqrt(in)): "QLoRA (low-rank adapters on a quantized
  model)", "The code, line by line" (A = standard normal / sqrt(in)).
* B = bf16(0.01 * N(0, 1)), non-zero so that dA is exercised; the B = 0 start
  of "How it works" step 2 is a separate case (``zeros``).
"""

from __future__ import annotations

import math
import zlib

import torch


def stream_seed(name: str, seed: int = 0) -> int:
    return (int(seed) * 1_000_003 + zlib.crc32(name.encode("utf-8"))) & 0x7FFF_FFFF_FFFF


def normal(name: str, shape, std: float = 1.0, dtype=torch.float32, device="cpu",
           seed: int = 0) -> torch.Tensor:
    """std * N(0, 1) drawn in float32 on ``device``, then cast to ``dtype``."""
    g = torch.Generator(device=device)
    g.manual_seed(stream_seed(name, seed))
    t = torch.randn(tuple(shape), generator=g, device=device, dtype=torch.float32)
    if std != 1.0:
        t.mul_(std)
    return t.to(dtype)


def layer_inputs(n_in: int, n_out: int, M: int, r: int, device="cpu", seed: int = 0,
                 tag: str = "", zero_B: bool = False) -> dict:
    """All inputs of one adapted linear: W0 (in, out) fp32, X (M, in), A (in, r),
    B (r, out), dY (M, out) in bf16."""
    p = f"{tag}{n_in}x{n_out}:"
    W0 = normal(p + "W0", (n_in, n_out), 0.02, torch.float32, device, seed)
    X = normal(p + "X", (M, n_in), 1.0, torch.bfloat16, device, seed)
    A = normal(p + "A", (n_in, r), 1.0 / math.sqrt(n_in), torch.bfloat16, device, seed)
    if zero_B:
        B = torch.zeros((r, n_out), dtype=torch.bfloat16, device=device)
    else:
        B = normal(p + "B", (r, n_out), 0.01, torch.bfloat16, device, seed)
    dY = normal(p + "dY", (M, n_out), 1.0, torch.bfloat16, device, seed)
    return {"W0": W0, "X": X, "A": A, "B": B, "dY": dY}


# The five workloads of the benchmark plan, by name and sizes.
CONFIGS = {
    "linear256_m64_r8": dict(shapes=[(256, 256)], M=64, r=8, bwd=True),
    "attn4096_m4096_r16": dict(shapes=[(4096, 4096)], M=4096, r=16, bwd=True),
    "mlp4096x11008_m8192_r64": dict(shapes=[(4096, 11008), (11008, 4096)], M=8192, r=64, bwd=True),
    "gemv4096_r16": dict(shapes=[(4096, 4096), (4096, 11008)], M=(1, 4, 16), r=16, bwd=False),
    "llama7b_stack_m2048_r16": dict(
        shapes=[(4096, 4096)] * 4 + [(4096, 11008)] * 2 + [(11008, 4096)],
        layers=32, M=2048, r=16, bwd=True),
}
