"""Pins of the clipping-search oracle (CPU only).

Page: "AWQ：为什么 4-bit 权重量化要先观察 Activation" (AWQ-P1), §5.
"""
import json
import os

import numpy as np
import pytest

import oracle as O
import oracle.awq_clip as C


@pytest.fixture(scope="module")
def example(golden_dir):
    with open(os.path.join(golden_dir, "awq_p1_clipping_counterexample.json")) as f:
        return json.load(f)


def _example_layer(example):
    x = np.concatenate([np.array(g["x"]) for g in example["groups"]])[None, :]
    w = np.concatenate([np.array(g["w"]) for g in example["groups"]])[:, None]
    return x, w


def test_counterexample_local_gain_whole_loss(example):
    """Per-group clipping improves each group's error but breaks the cancellation (AWQ-P1 §5)."""
    x, w = _example_layer(example)
    grp = example["group"]
    r = C.clip_search(x, w, np.ones(x.shape[1]), grp, example["n_shrink"], quantizer="sym_teaching",
                      arith_dtype=np.float64)
    factors = C.clip_factors(dtype=np.float64)
    assert len(factors) == 10 and factors[0] == 1.0 and factors[-1] == pytest.approx(0.55)
    total_base = total_sel = 0.0
    for g in range(2):
        xg, wg = x[0, g * grp:(g + 1) * grp], w[g * grp:(g + 1) * grp, 0]
        base = O.sym_teaching_qdq(wg[:, None], grp)[2].ravel()
        c = np.abs(wg).max() * factors[r.best[g, 0]]
        sel = O.sym_teaching_qdq(np.clip(wg, -c, c)[:, None], grp)[2].ravel()
        ref = float(xg @ wg)
        assert abs(float(xg @ base) - ref) == pytest.approx(example["per_group_abs_error_before"], abs=1e-9)
        assert abs(float(xg @ sel) - ref) == pytest.approx(example["per_group_abs_error_after"], abs=1e-9)
        # the search's own error for the chosen factor is that squared output error
        assert r.errors[r.best[g, 0], g, 0] == pytest.approx((float(xg @ sel) - ref) ** 2, rel=1e-12)
        total_base += float(xg @ base)
        total_sel += float(xg @ sel)
    assert total_base == pytest.approx(example["baseline_total"], abs=1e-12)
    assert total_sel == pytest.approx(0.5 - 4 / 175, abs=1e-12)
    assert total_sel == pytest.approx(example["selected_total"], abs=1e-12)


def _gram_errors(Xp, delta):
    """sum_t (x_t . d)^2 / T written as d^T (X^T X) d / T with explicit loops."""
    T, G = len(Xp), len(Xp[0])
    H = [[sum(Xp[t][i] * Xp[t][j] for t in range(T)) for j in range(G)] for i in range(G)]
    return sum(delta[i] * H[i][j] * delta[j] for i in range(G) for j in range(G)) / T


def test_errors_match_an_independent_gram_form():
    rng = np.random.default_rng(2)
    M, K, N, group = 9, 16, 3, 8
    X = (rng.standard_normal((M, K)) * np.exp(rng.standard_normal(K))).astype(np.float32)
    W = (rng.standard_normal((K, N)) * 0.05).astype(np.float32)
    s = np.exp(0.3 * rng.standard_normal(K)).astype(np.float32)
    r = C.clip_search(X, W, s, group, max_tokens=512)
    Wp = O.scale_weights(W, s)
    Xp = (X / s).astype(np.float32).astype(np.float64)
    for i in (0, 3, 9):
        for g in range(K // group):
            for n in range(N):
                wg = Wp[g * group:(g + 1) * group, n]
                c = np.float32(np.abs(wg).max() * C.clip_factors()[i])
                rec = O.asym_qdq(np.clip(wg, -c, c).astype(np.float32)[:, None], group)[3].ravel()
                d = (rec.astype(np.float64) - wg.astype(np.float64)).tolist()
                ref = _gram_errors(Xp[:, g * group:(g + 1) * group].tolist(), d)
                assert r.errors[i, g, n] == pytest.approx(ref, rel=1e-9)


def test_factor_one_is_the_unclipped_quantizer_and_best_is_first_min():
    rng = np.random.default_rng(4)
    M, K, N, group = 40, 256, 16, 128
    X = (rng.standard_normal((M, K)) * np.exp(0.5 * rng.standard_normal(K))).astype(np.float32)
    W = (rng.standard_normal((K, N)) * 0.02).astype(np.float32)
    s = O.candidate_scales(O.activation_statistic(X), 20)[7]
    r = C.clip_search(X, W, s, group)
    Wp = O.scale_weights(W, s)
    rec = O.asym_qdq(Wp, group)[3]
    Xp = (X / s).astype(np.float32).astype(np.float64)
    for g in range(K // group):
        d = rec[g * group:(g + 1) * group].astype(np.float64) - Wp[g * group:(g + 1) * group].astype(np.float64)
        e0 = np.mean((Xp[:, g * group:(g + 1) * group] @ d) ** 2, axis=0)
        assert np.allclose(r.errors[0, g], e0, rtol=1e-12, atol=0)
    # brute force of the argmin and the chosen thresholds
    for g in range(K // group):
        for n in range(N):
            e = list(r.errors[:, g, n])
            b = min(range(10), key=lambda i: (e[i], i))
            assert r.best[g, n] == b and r.max_val[g, n] == r.thresholds[b, g, n]


def test_sampled_tokens_stride():
    assert C.sample_tokens(4096).tolist() == list(range(0, 4096, 8))
    assert C.sample_tokens(100).tolist() == list(range(100))
    assert len(C.sample_tokens(16384)) == 512 and C.sample_tokens(16384)[1] == 32


def test_clipped_artifact_with_factor_one_is_the_search_artifact():
    rng = np.random.default_rng(6)
    K, N, group = 256, 16, 128
    W = (rng.standard_normal((K, N)) * 0.02).astype(np.float32)
    s = np.exp(0.2 * rng.standard_normal(K)).astype(np.float32)
    absmax = np.abs(O.scale_weights(W, s)).reshape(K // group, group, N).max(axis=1)
    codes, steps, zeros = C.clipped_artifact(W, s, group, absmax)
    q, step, zero, _ = O.asym_qdq(O.scale_weights(W, s), group)
    assert np.array_equal(codes, O.pack_codes(q))
    assert np.array_equal(steps.view(np.uint16), O.fp16_rne(step).view(np.uint16))


def test_silent_group_keeps_the_full_range():
    """A group whose sampled activations are all zero scores 0 for every threshold; the
    first candidate (no clipping) wins, as in the scale search's first minimum."""
    rng = np.random.default_rng(8)
    M, K, N, group = 16, 256, 8, 128
    X = rng.standard_normal((M, K)).astype(np.float32)
    X[:, :group] = 0.0
    W = (rng.standard_normal((K, N)) * 0.02).astype(np.float32)
    r = C.clip_search(X, W, np.ones(K, np.float32), group)
    assert np.all(r.errors[:, 0] == 0.0)
    assert np.all(r.best[0] == 0)
    assert np.array_equal(r.max_val[0], np.abs(W[:group]).max(axis=0))
