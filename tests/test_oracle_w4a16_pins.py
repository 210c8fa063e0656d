"""Pins of the W4A16 consumer oracle (CPU only).

Pages: "AWQ：为什么 4-bit 权重量化要先观察 Activation" (AWQ-P1) §6-§8 (the artifact's
consumer and its alignment check); "model-quantization / 05 core modules" §5.3.
"""
import struct
from fractions import Fraction

import numpy as np
import pytest

import oracle as O
import oracle.awq_w4a16 as Q


def _fp16(x: Fraction) -> float:
    """Round an exact rational to IEEE binary16 with CPython's own converter: the rational
    is first made a double (exact for the values used here), then struct's 'e' format
    rounds to half precision (round half to even)."""
    d = float(x)
    assert Fraction(d) == x, "the test values are exact in a double"
    return struct.unpack("<e", struct.pack("<e", d))[0]


def _artifact(q, steps, zeros):
    return O.pack_codes(np.asarray(q, dtype=np.int64)), np.asarray(steps, np.float16), np.asarray(zeros, np.float16)


def test_hand_built_artifact_decodes_to_the_definition():
    # K = 8 rows, N = 8 columns, groups of 4 rows; codes, steps and zeros chosen by hand
    rng = np.random.default_rng(0)
    q = rng.integers(0, 16, size=(8, 8))
    steps = np.array([[0.5, 0.25, 1 / 3, 0.1, 2.0 ** -14, 3.0, 0.007, 1.0]] * 2, dtype=np.float16)
    steps[1] *= np.float16(1.5)
    zeros = np.array([[0, 3, 7, 15, 8, 1, 12, 5], [2, 0, 15, 4, 9, 9, 0, 11]], dtype=np.float16)
    codes, st, zr = _artifact(q, steps, zeros)
    w = Q.dequant_operand(codes, st, zr, 4, 8)
    for k in range(8):
        for n in range(8):
            g = k // 4
            exact = (Fraction(int(q[k, n])) - Fraction(float(zeros[g, n]))) * Fraction(float(steps[g, n]))
            assert float(w[k, n]) == _fp16(exact), (k, n)
    # a code equal to the zero point decodes to +0
    assert np.all(w[q == np.repeat(zeros, 4, axis=0).astype(int)] == 0)


def test_matmul_is_the_exact_sum_of_exact_products():
    rng = np.random.default_rng(1)
    M, K, N, g = 3, 8, 8, 4
    q = rng.integers(0, 16, size=(K, N))
    steps = (rng.random((K // g, N)) * 0.1 + 0.01).astype(np.float16)
    zeros = rng.integers(0, 16, size=(K // g, N)).astype(np.float16)
    codes, st, zr = _artifact(q, steps, zeros)
    A = (rng.standard_normal((M, K)) * 3).astype(np.float16)
    Y = Q.w4a16_matmul(A, codes, st, zr, g)
    w = Q.dequant_operand(codes, st, zr, g, N)
    for m in range(M):
        for n in range(N):
            ref = sum(Fraction(float(A[m, k])) * Fraction(float(w[k, n])) for k in range(K))
            assert Y[m, n] == float(ref)  # fp64 sums of these products are exact here


def test_alignment_check_against_the_search():
    """AWQ-P1 §7: the decoded artifact matches the search's Q/DQ, and the consumer's output
    matches the search's folded-back layer up to the 16-bit roundings of the consumer."""
    rng = np.random.default_rng(2)
    M, K, N = 32, 256, 64
    X = (rng.standard_normal((M, K)) * np.exp(0.5 * rng.standard_normal(K))).astype(np.float32)
    W = (rng.standard_normal((K, N)) * 0.02).astype(np.float32)
    r = O.search(X, W, group=128, n_grid=20)
    w16 = Q.dequant_operand(r.codes, r.steps_f16, r.zeros_f16, 128, N).astype(np.float64)
    rec = O.asym_qdq(O.scale_weights(W, r.scales), 128)[3].astype(np.float64)
    st = np.repeat(r.step, 128, axis=0).astype(np.float64)
    # the fp16 rounding of the step (15 * 2^-11 step) and of the product (half an fp16 ulp)
    assert np.all(np.abs(w16 - rec) <= 15 * st * 2.0 ** -11 + np.abs(rec) * 2.0 ** -11 + 1e-30)
    Y = Q.w4a16_matmul(Q.fp16_activations(X, r.scales), r.codes, r.steps_f16, r.zeros_f16, 128)
    Wf = O.fold_back(rec, r.scales.astype(np.float64))
    ref = X.astype(np.float64) @ Wf
    assert np.linalg.norm(Y - ref) <= 2e-3 * np.linalg.norm(ref)


def test_activations_are_divided_by_the_scales():
    X = np.array([[1.0, 2.0, -3.0, 0.5]], np.float32)
    s = np.array([2.0, 0.5, 3.0, 0.25], np.float32)
    A = Q.fp16_activations(X, s)
    assert A.dtype == np.float16
    assert A.astype(np.float64).tolist() == [[0.5, 4.0, -1.0, 2.0]]


def test_group_boundaries_use_their_own_step():
    # one column, two groups of 2 rows with very different steps: the second group's rows
    # must use the second step
    q = np.array([[1], [2], [1], [2]] * 1)
    q = np.concatenate([q] * 8, axis=1)[:, :8]
    steps = np.array([[1.0] * 8, [100.0] * 8], np.float16)
    zeros = np.zeros((2, 8), np.float16)
    codes, st, zr = _artifact(q, steps, zeros)
    w = Q.dequant_operand(codes, st, zr, 2, 8)
    assert w[:, 0].astype(float).tolist() == [1.0, 2.0, 100.0, 200.0]
