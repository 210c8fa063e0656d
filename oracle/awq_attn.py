"""CPU oracle of the module-level objective for an attention block — TEST INFRASTRUCTURE ONLY.

Page: "AWQ：为什么 4-bit 权重量化要先观察 Activation" (AWQ-P1) §4: a candidate is scored by
running the module it belongs to with the candidate's weights and comparing the module
output with the original one; the inspected module may be an attention block holding
several projections rather than one linear layer. Here the searched projections are the
query, key and value projections, which read the same input X and share one scale
vector, and the module output is their causal multi-head attention.

Readings (the page names the module and nothing of its inside):
* W_qkv = [W_q | W_k | W_v] (K x 3D, D = heads * head_dim) is searched jointly, with one
  scale vector, as the joint gate+up layers are;
* X (M x K) holds n_seq calibration sequences of T = M / n_seq tokens each, sequence b
  in rows b T .. b T + T - 1; tokens attend within their own sequence only;
* head h is columns h d .. h d + d - 1 (d = head_dim) of each of Q, K and V;
* causal scaled dot-product attention, no position encoding (the page names none) and no
  output projection (W_o is a linear layer with its own input, the attention output):
    s_ij = q_i . k_j for j <= i;   m_i = max_j s_ij;   e_ij = exp((s_ij - m_i) / sqrt(d));
    l_i = sum_j e_ij;   p_ij = bf16(e_ij);   o_i = (sum_j p_ij v_j) / l_i;
* operands as the module's products consume them: bf16 X, bf16 candidate weights; Q, K
  and V rounded to fp32 and then to bf16 (the attention's operands); the weights p_ij
  rounded to fp32 and then to bf16 (the operand of the second product); the normaliser
  l_i sums the unrounded e_ij; products and sums exact (fp64) here;
* loss_i = mean over M x D of (O_i - O_ref)^2, O_ref the module with the original
  (bf16) weights; the first minimum wins.

Pins: tests/test_oracle_attn_pins.py.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np

from .awq_oracle import (activation_statistic, bf16_rne, candidate_scales, candidate_what, first_argmin,
                         squared_error_mean)

__all__ = ["causal_attention", "attn_forward", "AttnResult", "attn_search"]


def causal_attention(Q_b, K_b, V_b, n_seq: int, n_heads: int) -> np.ndarray:
    """Causal multi-head attention of bf16 Q, K, V (given as fp64 arrays, M x D each),
    the sequences stacked along the rows; returns O (M x D) in fp64."""
    M, D = Q_b.shape
    if M % n_seq or D % n_heads:
        raise ValueError("M must hold n_seq whole sequences and D n_heads whole heads")
    T, d = M // n_seq, D // n_heads
    inv_sqrt_d = 1.0 / np.sqrt(float(d))
    causal = np.tril(np.ones((T, T), dtype=bool))
    O = np.empty((M, D), dtype=np.float64)
    for b in range(n_seq):
        rows = slice(b * T, (b + 1) * T)
        for h in range(n_heads):
            cols = slice(h * d, (h + 1) * d)
            s = Q_b[rows, cols] @ K_b[rows, cols].T           # T x T dot products
            s = np.where(causal, s, -np.inf)
            m = s.max(axis=1, keepdims=True)
            e = np.exp((s - m) * inv_sqrt_d)                  # 0 where masked
            l = e.sum(axis=1, keepdims=True)
            p = bf16_rne(e.astype(np.float32)).astype(np.float64)
            O[rows, cols] = (p @ V_b[rows, cols]) / l
    return O


def attn_forward(X_b, Wqkv_b, n_seq: int, n_heads: int) -> np.ndarray:
    """The module output for bf16 X and bf16 [W_q | W_k | W_v] given as fp64 arrays."""
    D = Wqkv_b.shape[1] // 3
    QKV = X_b @ Wqkv_b                                         # exact products, fp64 sums
    QKV_b = bf16_rne(QKV.astype(np.float32)).astype(np.float64)
    return causal_attention(QKV_b[:, :D], QKV_b[:, D:2 * D], QKV_b[:, 2 * D:], n_seq, n_heads)


@dataclass
class AttnResult:
    a: np.ndarray          # statistic, K
    S: np.ndarray          # candidate scales, n_grid x K
    losses: np.ndarray     # fp64, n_grid
    best: int
    scales: np.ndarray     # S[best]


def attn_search(X, W_qkv, n_seq: int, n_heads: int, group: int = 128, n_grid: int = 20, *,
                quantizer: str = "asym") -> AttnResult:
    """The scale search of the query, key and value projections scored on the causal
    attention output of the calibration sequences."""
    X = np.asarray(X, dtype=np.float32)
    W_qkv = np.asarray(W_qkv, dtype=np.float32)
    if W_qkv.shape[1] % 3:
        raise ValueError("W_qkv is K x 3D")
    a = activation_statistic(X)
    S = candidate_scales(a, n_grid)
    X_b = bf16_rne(X).astype(np.float64)
    O_ref = attn_forward(X_b, bf16_rne(W_qkv).astype(np.float64), n_seq, n_heads)
    losses = np.empty(n_grid, dtype=np.float64)
    for i in range(n_grid):
        what_b = bf16_rne(candidate_what(W_qkv, S[i], group, quantizer)).astype(np.float64)
        losses[i] = squared_error_mean(attn_forward(X_b, what_b, n_seq, n_heads), O_ref)
    best = first_argmin(losses)
    return AttnResult(a=a, S=S, losses=losses, best=best, scales=S[best].copy())
