"""CPU oracle of AWQ's clipping search — TEST INFRASTRUCTURE ONLY.

Source: the AWQ walk-through page "AWQ：为什么 4-bit 权重量化要先观察 Activation"
(AWQ-P1), §5: after the channel scaling, a group can still hold a few large weights that
widen its range; clipping gives up those end points for a finer step. For every output
channel and every input group separately, the search tries thresholds of 1, 0.95, ...,
0.55 times the group's absolute maximum (10 candidates, 0.5 excluded), clamps the group
to [-threshold, threshold], quantizes it, and scores the candidate by the mean squared
error of the group's partial dot product over sampled tokens; the lowest error wins.

Readings:
* the weights searched are the scaled ones, W' = fl32(s * W), with the scales the
  scale search chose, and the partial outputs use the scaled activations
  X' = fl32(X / s) — the layer as it stands once the scales are folded in (AWQ-P1 §6);
* sampled tokens: every (M // 512)-th row of X, at most 512 rows;
* threshold c_i = fl32(absmax * fl32(1 - i/20)), i = 0..9;
* the quantizer is the search's own (the asymmetric 4-bit one of AWQ-P1 §7, fp32), or the
  symmetric teaching quantizer of AWQ-P1 §2 for the page's worked counterexample;
* error_i = mean over sampled tokens t of (sum_{k in group} X'[t,k] (Q(clamp(W'))[k] - W'[k]))^2,
  in fp64 from the fp32 values; the first minimum wins (as in the scale search).

Pins: tests/test_oracle_clip_pins.py (the page's counterexample 0.5 -> 0.5 - 4/175, an
independently written Gram-form error, factor 1 reproducing the unclipped quantizer,
brute force of the argmin, planted mistakes).
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np

from .awq_oracle import asym_qdq, sym_teaching_qdq, sym_artifact, scale_weights, pack_codes, fp16_rne, first_argmin

__all__ = ["clip_factors", "sample_tokens", "ClipResult", "clip_search", "clipped_artifact", "N_SHRINK",
           "SHRINK_GRID", "MAX_TOKENS"]

N_SHRINK = 10      # candidates 1, 0.95, ..., 0.55
SHRINK_GRID = 20   # factor_i = 1 - i / 20
MAX_TOKENS = 512


def clip_factors(n_shrink: int = N_SHRINK, grid: int = SHRINK_GRID, dtype=np.float32) -> np.ndarray:
    return np.array([1.0 - i / grid for i in range(n_shrink)], dtype=np.float64).astype(dtype)


def sample_tokens(M: int, max_tokens: int = MAX_TOKENS) -> np.ndarray:
    stride = max(1, M // max_tokens)
    return np.arange(0, M, stride)[:max_tokens]


def _quantize(wc, group, quantizer):
    if quantizer == "asym":
        return asym_qdq(wc, group)[3]
    if quantizer == "sym_teaching":
        return sym_teaching_qdq(wc, group)[2]
    raise ValueError(quantizer)


@dataclass
class ClipResult:
    errors: np.ndarray      # [n_shrink][G][N] fp64
    best: np.ndarray        # [G][N] int: first argmin over the shrink candidates
    max_val: np.ndarray     # [G][N] chosen threshold (dtype of the arithmetic)
    thresholds: np.ndarray  # [n_shrink][G][N]


def clip_search(X, W, s, group: int, n_shrink: int = N_SHRINK, *, quantizer: str = "asym",
                arith_dtype=np.float32, max_tokens: int = MAX_TOKENS) -> ClipResult:
    X = np.asarray(X, dtype=arith_dtype)
    W = np.asarray(W, dtype=arith_dtype)
    s = np.asarray(s, dtype=arith_dtype)
    M, K = X.shape
    N = W.shape[1]
    G = K // group
    Wp = scale_weights(W, s)                                        # W' = s * W
    rows = sample_tokens(M, max_tokens)
    Xp = (X[rows] / s[None, :]).astype(arith_dtype)                 # X' = X / s, sampled tokens
    factors = clip_factors(n_shrink, dtype=arith_dtype)
    errors = np.empty((n_shrink, G, N), dtype=np.float64)
    thresholds = np.empty((n_shrink, G, N), dtype=arith_dtype)
    for g in range(G):
        wg = Wp[g * group:(g + 1) * group]                          # group x N
        xg = Xp[:, g * group:(g + 1) * group].astype(np.float64)   # T x group
        absmax = np.abs(wg).max(axis=0)
        for i, f in enumerate(factors):
            c = (absmax * f).astype(arith_dtype)
            thresholds[i, g] = c
            wc = np.minimum(np.maximum(wg, -c[None, :]), c[None, :]).astype(arith_dtype)
            rec = _quantize(wc, group, quantizer)
            delta = rec.astype(np.float64) - wg.astype(np.float64)
            partial = xg @ delta                                    # T x N partial output errors
            errors[i, g] = np.mean(partial ** 2, axis=0)
    best = np.empty((G, N), dtype=np.int64)
    for g in range(G):
        for n in range(N):
            best[g, n] = first_argmin(list(errors[:, g, n]))
    max_val = np.take_along_axis(thresholds, best[None], axis=0)[0]
    return ClipResult(errors=errors, best=best, max_val=max_val, thresholds=thresholds)


def clipped_artifact(W, s, group: int, max_val, quantizer: str = "asym"):
    """Codes (packed), fp16 steps and fp16 zeros of Q(clamp(s * W, -max_val, max_val))."""
    W = np.asarray(W, dtype=np.float32)
    Wp = scale_weights(W, np.asarray(s, dtype=np.float32))
    c = np.repeat(np.asarray(max_val, dtype=np.float32), group, axis=0)
    wc = np.minimum(np.maximum(Wp, -c), c).astype(np.float32)
    if quantizer == "asym":
        q, step, zero, _ = asym_qdq(wc, group)
    else:
        q, step, zero = sym_artifact(wc, group)
    return pack_codes(q), fp16_rne(step), zero.astype(np.float16)
