"""Plain CPU oracle of AWQ's activation-aware per-layer scale search.

TEST INFRASTRUCTURE ONLY: imported by tests/, __graft_entry__.smoke() and the CPU
baseline of bench.py; never by the product path.

Source pages (cited by title and section):

* [AWQ-P1] "AWQ：为什么 4-bit 权重量化要先观察 Activation" (charlestar.github.io) —
  §1 the activation statistic and the X^T X cross terms, §2 the symmetric teaching
  quantizer, §3 channel scaling and the two-channel worked example with its
  20-candidate search, §4 the scale family and the candidate loss, §7 the
  asymmetric zero-point quantizer of the real artifact and its orientation, §8 the
  bits-per-weight budget.
* [AWQ-P2] "AWQ salient weight / GGUF compilation" (dreamvfia.cn), §二: the scale
  family s_k = (mean_b |X_bk|)^alpha written out in LaTeX.
* [QUANT-P4] "model-quantization / 05 core modules" (ai-infra.cypggs.com), §5.3:
  int4 codes packed eight to an int32.

Notation (AWQ-P1 §1, §7): X is M x K (M calibration tokens, K input channels), W is
K x N (N output channels), groups run along K, a group is `group` consecutive rows
of one column of W.

Readings where the pages are silent or garbled:

* statistic: |X| summed in fp64, divided by M in fp64, rounded once to fp32;
* scales: alpha_i = i / n_grid; raw = max(a^alpha, 1e-4) (clamp BEFORE the
  normalisation, AWQ-P1 §4), s = raw / sqrt(max(raw) * min(raw)), all in fp64, then
  one rounding to fp32;
* asymmetric QDQ (AWQ-P1 §7) in fp32, in the order the page states: step =
  (max - min) / 15, an all-equal group (or an underflowed step) gets step 1;
  z = clamp(rint(-min / step), 0, 15); q = clamp(rint(w' / step) + z, 0, 15);
  reconstruction (q - z) * step; rint is round-half-even (AWQ-P1 §2 ties-to-even);
* fold-back: W_hat = reconstruction / s (AWQ-P1 §4: "scale, pseudo-quantize, divide
  back"), fp32, then rounded to bf16 because the candidate forward runs with bf16
  operands (W4A16 keeps FP16/BF16 activations, AWQ-P1 §8);
* loss: mean over all M*N outputs of (X_b W_hat_b - X_b W_b)^2, computed here in fp64
  from exact bf16 products (AWQ-P1 §4: output difference in FP32, squared, mean);
* argmin: the FIRST minimum (AWQ-P1 §3 uses Python's min);
* artifact: codes packed eight per int32 along N, nibble i of word (k, w) holding
  column 8w + i (QUANT-P4 §5.3); steps and zeros as fp16.

Pins (tests/test_oracle_pins.py): the worked example of AWQ-P1 §3 through `search`
with the teaching quantizer; the teaching quantizer's unit facts (AWQ-P1 §3 code
asserts); brute force over every 4-bit code vector of tiny groups; the exact
no-quantization fold-back invariant; power-of-two common-scale invariance; a rational
brute-force statistic; an independently written Gram-form loss (the X^T X form of
AWQ-P1 §1); zero loss for weights already on the grid; bf16 rounding against torch's
converter; packing round trip and the 4.25 bits/weight budget of AWQ-P1 §8.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

__all__ = [
    "bf16_rne", "fp16_rne", "activation_statistic", "candidate_alphas",
    "candidate_scales", "scale_weights", "asym_qdq", "sym_teaching_qdq", "fold_back",
    "candidate_what", "squared_error_mean", "output_loss", "block_squared_error", "first_argmin",
    "pack_codes", "unpack_codes", "decode_artifact", "bits_per_weight", "sym_artifact",
    "SearchResult", "search", "CLAMP_MIN", "Q_MAX",
]

CLAMP_MIN = 1e-4   # positive lower bound applied to a^alpha before normalising (AWQ-P1 §4)
Q_MAX = 15         # 4-bit unsigned codes 0..15 (AWQ-P1 §7)


# ----------------------------------------------------------------------------------
# Number formats
# ----------------------------------------------------------------------------------
def bf16_rne(x) -> np.ndarray:
    """Round float32 values to the nearest bfloat16 (ties to even), returned as float32.

    bfloat16 is the upper 16 bits of an IEEE binary32; rounding to nearest-even adds
    0x7FFF plus the lowest kept bit, then truncates. Finite inputs only.
    """
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    keep_lsb = (u >> np.uint64(16)) & np.uint64(1)
    u = ((u + np.uint64(0x7FFF) + keep_lsb) >> np.uint64(16)) << np.uint64(16)
    return u.astype(np.uint32).view(np.float32)


def fp16_rne(x) -> np.ndarray:
    """IEEE binary16 rounding (numpy's converter, round-to-nearest-even)."""
    return np.asarray(x, dtype=np.float32).astype(np.float16)


# ----------------------------------------------------------------------------------
# Step 1: activation statistic (AWQ-P1 §1; AWQ-P2 §二)
# ----------------------------------------------------------------------------------
def activation_statistic(X, out_dtype=np.float32) -> np.ndarray:
    """a_j = (1/M) * sum_m |X[m, j]|, accumulated in fp64 and rounded once.

    Non-finite inputs are rejected (AWQ-P1 §2: only finite reals take part).
    """
    X64 = np.asarray(X, dtype=np.float64)
    if X64.ndim != 2 or X64.shape[0] == 0:
        raise ValueError("X must be a non-empty M x K matrix")
    if not np.all(np.isfinite(X64)):
        raise ValueError("non-finite activation")
    total = np.abs(X64).sum(axis=0)
    return (total / X64.shape[0]).astype(out_dtype)


# ----------------------------------------------------------------------------------
# Step 2: candidate scales (AWQ-P1 §3 code, §4; AWQ-P2 §二)
# ----------------------------------------------------------------------------------
def candidate_alphas(n_grid: int) -> np.ndarray:
    """alpha_i = i / n_grid for i = 0..n_grid-1 (1 itself is excluded, AWQ-P1 §4)."""
    return np.array([i / n_grid for i in range(n_grid)], dtype=np.float64)


def candidate_scales(a, n_grid: int, out_dtype=np.float32) -> np.ndarray:
    """S[i, j] = raw_ij / sqrt(max_j raw_ij * min_j raw_ij), raw_ij = max(a_j^alpha_i, 1e-4)."""
    a64 = np.asarray(a, dtype=np.float64)
    S = np.empty((n_grid, a64.size), dtype=out_dtype)
    for i, alpha in enumerate(candidate_alphas(n_grid)):
        raw = np.maximum(np.power(a64, alpha), CLAMP_MIN)
        normaliser = np.sqrt(raw.max() * raw.min())
        S[i] = (raw / normaliser).astype(out_dtype)
    return S


# ----------------------------------------------------------------------------------
# Step 3: scaling and group-wise quantize/dequantize
# ----------------------------------------------------------------------------------
def scale_weights(W, s) -> np.ndarray:
    """W' = diag(s) W: row j of W (input channel j) times s_j (AWQ-P1 §3)."""
    W = np.asarray(W)
    return (np.asarray(s, dtype=W.dtype)[:, None] * W).astype(W.dtype)


def _groups(Wp, group):
    K, N = Wp.shape
    if group <= 0 or K % group:
        raise ValueError("group size must divide the input dimension K (AWQ-P1 §7)")
    return Wp.reshape(K // group, group, N)


def asym_qdq(Wp, group: int):
    """Asymmetric 4-bit zero-point pseudo-quantization along K (AWQ-P1 §7).

    Works in the dtype of ``Wp`` (fp32 for the search). Returns
    ``(q, step, zero, rec)``: codes q (int32, K x N), step and zero (G x N, zero
    integral in 0..15), and the reconstruction rec = (q - zero) * step (K x N).
    """
    Wp = np.asarray(Wp)
    dt = Wp.dtype.type
    if not np.all(np.isfinite(Wp)):
        raise ValueError("non-finite weight")
    Wg = _groups(Wp, group)
    mn = Wg.min(axis=1)
    mx = Wg.max(axis=1)
    step = ((mx - mn).astype(dt) / dt(Q_MAX)).astype(dt)
    step = np.where((mx == mn) | (step == 0), dt(1), step).astype(dt)
    # the zero point is an integer in 0..15: adding +0 turns a rounded -0 into 0
    zero = (np.clip(np.rint((-mn / step).astype(dt)), 0, Q_MAX).astype(dt) + dt(0)).astype(dt)
    q = np.clip(np.rint((Wg / step[:, None, :]).astype(dt)) + zero[:, None, :], 0, Q_MAX).astype(dt)
    rec = ((q - zero[:, None, :]) * step[:, None, :]).astype(dt)
    K, N = Wp.shape
    return (q.reshape(K, N).astype(np.int32), step, zero, rec.reshape(K, N))


def sym_teaching_qdq(Wp, group: int):
    """The symmetric [-7, 7] absmax teaching quantizer of AWQ-P1 §2 (ties-to-even).

    step = peak / 7 per group (peak = max |w|), an all-zero group gets step 1 and
    codes 0; non-finite values are rejected. Returns ``(q, step, rec)``.
    """
    Wp = np.asarray(Wp)
    dt = Wp.dtype.type
    if Wp.size == 0 or not np.all(np.isfinite(Wp)):
        raise ValueError("a group must contain finite values")
    Wg = _groups(Wp, group)
    peak = np.abs(Wg).max(axis=1)
    step = (peak / dt(7)).astype(dt)
    # an all-zero group gets step 1 (AWQ-P1 §2); so does a quotient that underflows to 0
    step = np.where((peak == 0) | (step == 0), dt(1), step).astype(dt)
    q = np.clip(np.rint((Wg / step[:, None, :]).astype(dt)), -7, 7).astype(dt)
    rec = (q * step[:, None, :]).astype(dt)
    K, N = Wp.shape
    return q.reshape(K, N).astype(np.int32), step, rec.reshape(K, N)


def fold_back(rec, s) -> np.ndarray:
    """W_hat = diag(s)^-1 Q(diag(s) W): divide row j by s_j again (AWQ-P1 §4)."""
    rec = np.asarray(rec)
    return (rec / np.asarray(s, dtype=rec.dtype)[:, None]).astype(rec.dtype)


def candidate_what(W, s, group: int, quantizer: str = "asym") -> np.ndarray:
    """diag(s)^-1 Q(diag(s) W) in the dtype of W, before any bf16 operand rounding."""
    Wp = scale_weights(W, s)
    if quantizer == "asym":
        rec = asym_qdq(Wp, group)[3]
    elif quantizer == "sym_teaching":
        rec = sym_teaching_qdq(Wp, group)[2]
    elif quantizer == "none":
        rec = Wp
    else:
        raise ValueError(f"unknown quantizer {quantizer!r}")
    return fold_back(rec, s)


# ----------------------------------------------------------------------------------
# Step 4: forward-output loss (AWQ-P1 §4)
# ----------------------------------------------------------------------------------
def squared_error_mean(Yhat, Y) -> float:
    """mean over all outputs of (Y_hat - Y)^2, in fp64."""
    return float(np.mean((np.asarray(Yhat, np.float64) - np.asarray(Y, np.float64)) ** 2))


def output_loss(X64, W64, What64) -> float:
    """mean over the M x N outputs of (X W_hat - X W)^2, in fp64."""
    return squared_error_mean(X64 @ What64, X64 @ W64)


def block_squared_error(X64, W64, What64) -> float:
    """Sum (not mean) of (X W_hat - X W)^2 over the given block of outputs, in fp64."""
    Y = X64 @ W64
    Yhat = X64 @ What64
    return float(np.sum((Yhat - Y) ** 2))


# ----------------------------------------------------------------------------------
# Step 5: argmin (AWQ-P1 §3: Python's min keeps the first minimum)
# ----------------------------------------------------------------------------------
def first_argmin(losses) -> int:
    best = 0
    for i in range(1, len(losses)):
        if losses[i] < losses[best]:
            best = i
    return best


# ----------------------------------------------------------------------------------
# Step 6: artifact (AWQ-P1 §7, §8; QUANT-P4 §5.3)
# ----------------------------------------------------------------------------------
def pack_codes(q) -> np.ndarray:
    """Pack 4-bit codes (K x N, N % 8 == 0) eight per int32 along N, column 8w+i in bits 4i..4i+3."""
    q = np.asarray(q, dtype=np.int64)
    K, N = q.shape
    if N % 8:
        raise ValueError("N must be a multiple of 8 to pack eight codes per int32")
    words = np.zeros((K, N // 8), dtype=np.int64)
    for i in range(8):
        words |= (q[:, i::8] & 0xF) << (4 * i)
    return words.astype(np.uint32).view(np.int32)


def unpack_codes(words, N: int) -> np.ndarray:
    w = np.asarray(words).view(np.uint32).astype(np.int64)
    K = w.shape[0]
    q = np.zeros((K, N), dtype=np.int32)
    for i in range(8):
        q[:, i::8] = (w >> (4 * i)) & 0xF
    return q


def decode_artifact(words, steps_f16, zeros_f16, group: int, N: int) -> np.ndarray:
    """Scaled-domain weights step * (q - zero) from the artifact (fp32)."""
    q = unpack_codes(words, N).astype(np.float32)
    st = np.repeat(np.asarray(steps_f16, dtype=np.float32), group, axis=0)
    zr = np.repeat(np.asarray(zeros_f16, dtype=np.float32), group, axis=0)
    return ((q - zr) * st).astype(np.float32)


def bits_per_weight(K: int, N: int, group: int) -> float:
    """Storage of codes + fp16 step + fp16 zero per weight, excluding the K scales."""
    return (4.0 * K * N + 32.0 * (K // group) * N) / (K * N)


# ----------------------------------------------------------------------------------
# The whole search
# ----------------------------------------------------------------------------------
@dataclass
class SearchResult:
    a: np.ndarray                  # statistic, K
    S: np.ndarray                  # candidate scales, n_grid x K
    losses: np.ndarray             # fp64, n_grid
    best: int                      # first argmin
    scales: np.ndarray             # S[best]
    q: np.ndarray | None = None    # codes K x N (asym only)
    step: np.ndarray | None = None
    zero: np.ndarray | None = None
    codes: np.ndarray | None = None        # packed int32, K x N/8
    steps_f16: np.ndarray | None = None    # G x N
    zeros_f16: np.ndarray | None = None    # G x N
    extra: dict = field(default_factory=dict)


def search(X, W, group: int = 128, n_grid: int = 20, *, quantizer: str = "asym",
           arith_dtype=np.float32, bf16_operands: bool = True) -> SearchResult:
    """Run the six steps on one layer.

    ``arith_dtype`` is the precision of the statistic rounding, the scales and the
    QDQ (fp32 for the product definition; fp64 reproduces AWQ-P1 §3's Python, which
    works in binary64). ``bf16_operands`` rounds X and every candidate W_hat to bf16
    before the fp64 forward, as the GEMM of the search consumes them.
    """
    X = np.asarray(X, dtype=arith_dtype)
    W = np.asarray(W, dtype=arith_dtype)
    M, K = X.shape
    K2, N = W.shape
    if K != K2:
        raise ValueError("X is M x K and W is K x N")
    if not np.all(np.isfinite(W)):
        raise ValueError("non-finite weight")
    a = activation_statistic(X, out_dtype=arith_dtype)
    S = candidate_scales(a, n_grid, out_dtype=arith_dtype)

    if bf16_operands:
        X64 = bf16_rne(X).astype(np.float64)
        W64 = bf16_rne(W).astype(np.float64)
    else:
        X64 = X.astype(np.float64)
        W64 = W.astype(np.float64)
    Y = X64 @ W64
    losses = np.empty(n_grid, dtype=np.float64)
    for i in range(n_grid):
        what = candidate_what(W, S[i], group, quantizer)
        what64 = (bf16_rne(what) if bf16_operands else what).astype(np.float64)
        losses[i] = squared_error_mean(X64 @ what64, Y)
    best = first_argmin(losses)
    res = SearchResult(a=a, S=S, losses=losses, best=best, scales=S[best].copy())
    res.extra["Y"] = Y
    if quantizer == "asym":
        q, step, zero, _ = asym_qdq(scale_weights(W, S[best]), group)
    elif quantizer == "sym_teaching":
        q, step, zero = sym_artifact(scale_weights(W, S[best]), group)
    else:
        return res
    res.q, res.step, res.zero = q, step, zero
    if N % 8 == 0:
        res.codes = pack_codes(q)
    res.steps_f16 = fp16_rne(step)
    res.zeros_f16 = zero.astype(np.float16)
    return res


def sym_artifact(Wp, group: int):
    """The teaching quantizer's codes in the unsigned 4-bit artifact: code = q + 7 in
    0..14 with zero point 7, so step * (code - zero) = q * step (AWQ-P1 §2 quantizer,
    §7 artifact)."""
    q, step, _ = sym_teaching_qdq(Wp, group)
    zero = np.full(step.shape, 7.0, dtype=np.asarray(Wp).dtype)
    return (q + 7).astype(np.int32), step, zero
