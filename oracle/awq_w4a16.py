"""CPU oracle of the W4A16 consumer of the packed artifact — TEST INFRASTRUCTURE ONLY.

Pages: "AWQ：为什么 4-bit 权重量化要先观察 Activation" (AWQ-P1) §7: the search's output feeds
a W4A16 kernel, and the alignment check decodes the artifact, compares it with the
search's own quantize/dequantize, then compares the kernel's output with a reference;
§8: W4A16 means 4-bit weights with 16-bit activations, the accumulation precision being
a separate choice; §6: the scales are folded into the operation that produces the
activations, so the linear layer receives X / s. "model-quantization / 05 core modules"
(QUANT-P4) §5.3: int4 codes packed eight per int32 with separate fp16 scale tensors.

Readings:
* activations: A = fp16(fl32(X / s)) — 16-bit activations already divided by the scales;
* dequantized weight: w16[k][n] = fp16((q[k][n] - z[g][n]) * step[g][n]) with the
  artifact's fp16 step and zero (q - z is an integer of magnitude at most 15, so the
  product is exact before its one rounding to fp16);
* output: Y = A w16, every product exact (11 + 11 significant bits), sums exact in fp64
  here (the kernels accumulate in fp32).

Pins: tests/test_oracle_w4a16_pins.py.
"""
from __future__ import annotations

import numpy as np

from .awq_oracle import unpack_codes

__all__ = ["fp16_activations", "dequant_operand", "w4a16_matmul"]


def fp16_activations(X, s) -> np.ndarray:
    """A = fp16(fl32(X / s)) as float16 (AWQ-P1 §6: the scales divide the activations)."""
    X = np.asarray(X, dtype=np.float32)
    s = np.asarray(s, dtype=np.float32)
    return (X / s[None, :]).astype(np.float32).astype(np.float16)


def dequant_operand(codes, steps_f16, zeros_f16, group: int, N: int) -> np.ndarray:
    """w16[k][n] = fp16((q - z) * step), K x N float16."""
    q = unpack_codes(codes, N).astype(np.float64)
    K = q.shape[0]
    if K % group:
        raise ValueError("group must divide K")
    st = np.repeat(np.asarray(steps_f16, dtype=np.float16).astype(np.float64), group, axis=0)
    zr = np.repeat(np.asarray(zeros_f16, dtype=np.float16).astype(np.float64), group, axis=0)
    exact = (q - zr) * st          # exact in fp64 (4-bit integer times an 11-bit significand)
    return exact.astype(np.float16)


def w4a16_matmul(A_f16, codes, steps_f16, zeros_f16, group: int) -> np.ndarray:
    """Y = A w16 in fp64 (exact products, fp64 sums), M x N."""
    A = np.asarray(A_f16, dtype=np.float16).astype(np.float64)
    N = np.asarray(steps_f16).shape[1]
    W = dequant_operand(codes, steps_f16, zeros_f16, group, N).astype(np.float64)
    return A @ W
