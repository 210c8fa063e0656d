"""CPU oracle of the module-level objective for an MLP block — TEST INFRASTRUCTURE ONLY.

Page: "AWQ：为什么 4-bit 权重量化要先观察 Activation" (AWQ-P1) §4: a candidate is scored by
running the module it belongs to with the candidate's weights and comparing the module
output with the original one; the module may hold several projections, up to a whole
MLP block. Here the searched projections are the gate and up projections of a
Llama-shaped MLP, which read the same input and share one scale vector; the block
output is down(act(X W_gate) * (X W_up)).

Readings:
* W_gu = [W_gate | W_up] (K x 2F) is searched jointly, as the gate+up layers are;
* act = SiLU, x / (1 + exp(-x)) (the activation of the Llama-shaped blocks);
* the down projection keeps its original weights during the search;
* operands as the search's GEMMs consume them: bf16 X, bf16 candidate weights, bf16
  W_down; the intermediate h = silu(G) * U is rounded to fp32 and then to bf16 (the
  operand of the second GEMM); products and sums exact in fp64 here;
* loss_i = mean over M x K_out of (Y_i - Y_ref)^2, Y_ref the block with the original
  (bf16) weights; the first minimum wins.

Pins: tests/test_oracle_module_pins.py.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np

from .awq_oracle import (activation_statistic, bf16_rne, candidate_scales, candidate_what, first_argmin,
                         squared_error_mean)

__all__ = ["silu", "mlp_forward", "ModuleResult", "mlp_search"]


def silu(x) -> np.ndarray:
    """SiLU in fp64: x / (1 + exp(-x))."""
    x = np.asarray(x, dtype=np.float64)
    return x / (1.0 + np.exp(-x))


def mlp_forward(X_b, Wgu_b, Wd_b) -> np.ndarray:
    """down(silu(X W_gate) * (X W_up)) with bf16 operands given as fp64 arrays, the
    intermediate rounded to fp32 and then to bf16."""
    F = Wgu_b.shape[1] // 2
    H = X_b @ Wgu_b                                   # exact products, fp64 sums
    h = (silu(H[:, :F]) * H[:, F:]).astype(np.float32)
    h_b = bf16_rne(h).astype(np.float64)
    return h_b @ Wd_b


@dataclass
class ModuleResult:
    a: np.ndarray          # statistic, K
    S: np.ndarray          # candidate scales, n_grid x K
    losses: np.ndarray     # fp64, n_grid
    best: int
    scales: np.ndarray     # S[best]


def mlp_search(X, W_gu, W_down, group: int = 128, n_grid: int = 20, *, quantizer: str = "asym") -> ModuleResult:
    """The scale search of the gate and up projections scored on the block output."""
    X = np.asarray(X, dtype=np.float32)
    W_gu = np.asarray(W_gu, dtype=np.float32)
    W_down = np.asarray(W_down, dtype=np.float32)
    if W_gu.shape[1] % 2 or W_down.shape[0] != W_gu.shape[1] // 2:
        raise ValueError("W_gu is K x 2F and W_down is F x K_out")
    a = activation_statistic(X)
    S = candidate_scales(a, n_grid)
    X_b = bf16_rne(X).astype(np.float64)
    Wd_b = bf16_rne(W_down).astype(np.float64)
    Y_ref = mlp_forward(X_b, bf16_rne(W_gu).astype(np.float64), Wd_b)
    losses = np.empty(n_grid, dtype=np.float64)
    for i in range(n_grid):
        what_b = bf16_rne(candidate_what(W_gu, S[i], group, quantizer)).astype(np.float64)
        losses[i] = squared_error_mean(mlp_forward(X_b, what_b, Wd_b), Y_ref)
    best = first_argmin(losses)
    return ModuleResult(a=a, S=S, losses=losses, best=best, scales=S[best].copy())
