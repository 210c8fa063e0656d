"""Pins of the attention-block objective oracle (CPU only).

Page: "AWQ：为什么 4-bit 权重量化要先观察 Activation" (AWQ-P1) §4: a candidate may be scored
on the output of a whole attention module holding several projections. The oracle's
readings (causal multi-head attention of the calibration sequences, heads as contiguous
column blocks, 1/sqrt(head_dim) scaling, bf16 Q/K/V and attention weights) are pinned
here by hand-computed cases, closed forms, symmetries and an explicit-loop restatement.
"""
import math

import numpy as np
import pytest
import torch

import oracle as O
import oracle.awq_attn as ATT


def _bf16(x: float) -> float:
    """bf16 rounding by torch's converter (independent of the oracle's)."""
    return float(torch.tensor([x], dtype=torch.float32).to(torch.bfloat16).float()[0])


def test_first_token_sees_only_itself():
    """Causality: token 0's output is v_0 exactly, whatever the later tokens hold."""
    Q = np.array([[1.0, 2.0], [0.5, -1.0]])
    K = np.array([[3.0, 0.0], [-7.0, 9.0]])
    V = np.array([[0.25, -4.0], [100.0, 200.0]])
    O0 = ATT.causal_attention(Q, K, V, n_seq=1, n_heads=1)
    assert O0[0].tolist() == [0.25, -4.0]
    K2, V2 = K.copy(), V.copy()
    K2[1] = [50.0, 50.0]
    V2[1] = [-1.0, 3.0]
    assert ATT.causal_attention(Q, K2, V2, 1, 1)[0].tolist() == [0.25, -4.0]


def test_equal_scores_average_the_values():
    """q_1 . k_0 == q_1 . k_1: both weights are exp(0) = 1, so o_1 = (v_0 + v_1) / 2."""
    Q = np.array([[1.0, 0.0], [1.0, 1.0]])
    K = np.array([[2.0, 1.0], [1.0, 2.0]])       # q_1 . k = 3 for both keys
    V = np.array([[1.0, -3.0], [5.0, 7.0]])
    O1 = ATT.causal_attention(Q, K, V, 1, 1)[1]
    assert O1.tolist() == [3.0, 2.0]


def test_weights_use_the_scaled_scores_and_the_unrounded_normaliser():
    """head_dim 4 (scale 1/2): scores 0 and 2 give e = [exp(-1), 1]; the weight of key 0 is
    bf16(fp32(exp(-1))) = 0.3671875, the normaliser 1 + exp(-1) (unrounded)."""
    Q = np.array([[1.0, 0, 0, 0], [1.0, 0, 0, 0]])
    K = np.array([[0.0, 0, 0, 0], [2.0, 0, 0, 0]])
    V = np.array([[1.0, 0, 0, 0], [0.0, 1.0, 0, 0]])
    O1 = ATT.causal_attention(Q, K, V, 1, 1)[1]
    e0 = math.exp(-1.0)
    p0 = _bf16(e0)
    assert p0 == 0.3671875
    l = 1.0 + e0
    assert O1[0] == pytest.approx(p0 / l, rel=1e-15)
    assert O1[1] == pytest.approx(1.0 / l, rel=1e-15)
    assert O1[2] == 0.0 and O1[3] == 0.0


def test_sequences_are_independent():
    """Tokens attend within their own sequence: changing sequence 1 leaves sequence 0's
    outputs unchanged, and swapping the two sequences swaps the outputs."""
    rng = np.random.default_rng(3)
    T, D = 5, 8
    Q, K, V = (np.asarray(O.bf16_rne(rng.standard_normal((2 * T, D)).astype(np.float32)), np.float64)
               for _ in range(3))
    base = ATT.causal_attention(Q, K, V, n_seq=2, n_heads=2)
    K2 = K.copy()
    K2[T:] *= -3.0
    assert np.array_equal(ATT.causal_attention(Q, K2, V, 2, 2)[:T], base[:T])
    swap = np.r_[T:2 * T, 0:T]
    assert np.array_equal(ATT.causal_attention(Q[swap], K[swap], V[swap], 2, 2), base[swap])


def test_heads_are_contiguous_column_blocks():
    """Permuting the heads (blocks of head_dim columns, in Q, K and V together) permutes
    the output blocks the same way; moving single columns between heads does not."""
    rng = np.random.default_rng(4)
    T, H, d = 6, 3, 4
    Q, K, V = (np.asarray(O.bf16_rne(rng.standard_normal((T, H * d)).astype(np.float32)), np.float64)
               for _ in range(3))
    base = ATT.causal_attention(Q, K, V, 1, H)
    perm = np.concatenate([np.arange(h * d, (h + 1) * d) for h in (2, 0, 1)])
    assert np.array_equal(ATT.causal_attention(Q[:, perm], K[:, perm], V[:, perm], 1, H), base[:, perm])
    inter = np.arange(H * d).reshape(d, H).T.reshape(-1)   # column h + H j into head h
    assert not np.allclose(ATT.causal_attention(Q[:, inter], K[:, inter], V[:, inter], 1, H), base[:, inter])


def test_qkv_are_rounded_to_bf16():
    """X W = 1 + 2^-10 is not a bf16 value: V rounds to 1, and a single token's output is
    its own value."""
    X = np.array([[1.0]])
    W = np.array([[1.0, 1.0, 1.0 + 2.0 ** -10]])
    Ot = ATT.attn_forward(X, W, n_seq=1, n_heads=1)
    assert Ot.tolist() == [[1.0]]


def test_matches_an_explicit_loop():
    """The module output written out with loops (math.exp, torch's bf16 converter) on
    2 sequences x 3 tokens, 2 heads of dimension 2."""
    rng = np.random.default_rng(5)
    n_seq, T, H, d, Kin = 2, 3, 2, 2, 8
    D = H * d
    X = rng.standard_normal((n_seq * T, Kin)).astype(np.float32)
    W = (rng.standard_normal((Kin, 3 * D)) * 0.5).astype(np.float32)
    Xb = O.bf16_rne(X).astype(np.float64)
    Wb = O.bf16_rne(W).astype(np.float64)
    got = ATT.attn_forward(Xb, Wb, n_seq, H)

    def proj(m, col):
        return _bf16(sum(float(Xb[m, k]) * float(Wb[k, col]) for k in range(Kin)))

    want = np.zeros((n_seq * T, D))
    for b in range(n_seq):
        for h in range(H):
            for i in range(T):
                qi = [proj(b * T + i, h * d + t) for t in range(d)]
                scores = []
                for j in range(i + 1):
                    kj = [proj(b * T + j, D + h * d + t) for t in range(d)]
                    scores.append(sum(qi[t] * kj[t] for t in range(d)))
                mx = max(scores)
                es = [math.exp((s - mx) / math.sqrt(d)) for s in scores]
                norm = sum(es)
                for t in range(d):
                    acc = 0.0
                    for j in range(i + 1):
                        acc += _bf16(es[j]) * proj(b * T + j, 2 * D + h * d + t)
                    want[b * T + i, h * d + t] = acc / norm
    assert np.allclose(got, want, rtol=1e-12, atol=1e-300)


def test_weights_on_the_grid_give_zero_loss_at_alpha_zero():
    """alpha = 0: every scale is 1, and weights already on their group's 16-level grid
    (exact in bf16) quantize to themselves, so candidate 0 reproduces the module."""
    rng = np.random.default_rng(6)
    M, K, D, g = 8, 64, 8, 32
    levels = rng.integers(0, 16, size=(K, 3 * D)).astype(np.float64)
    levels[0::g] = 0.0
    levels[1::g] = 15.0
    W = (levels * 0.125 - 1.0).astype(np.float32)
    X = rng.standard_normal((M, K)).astype(np.float32)
    r = ATT.attn_search(X, W, n_seq=2, n_heads=2, group=g, n_grid=5)
    assert r.losses[0] == 0.0 and r.best == 0
    assert np.all(r.losses[1:] >= 0.0) and np.any(r.losses[1:] > 0.0)


def test_search_losses_match_the_loop_module():
    """Every candidate's loss equals the mean squared difference of two module outputs
    computed by attn_forward from the candidates' bf16 weights (AWQ-P1 §4)."""
    rng = np.random.default_rng(7)
    M, K, D, g = 6, 16, 4, 8
    X = rng.standard_normal((M, K)).astype(np.float32)
    W = (rng.standard_normal((K, 3 * D)) * 0.4).astype(np.float32)
    r = ATT.attn_search(X, W, n_seq=2, n_heads=2, group=g, n_grid=4)
    Xb = O.bf16_rne(X).astype(np.float64)
    ref = ATT.attn_forward(Xb, O.bf16_rne(W).astype(np.float64), 2, 2)
    for i in range(4):
        out = ATT.attn_forward(Xb, O.bf16_rne(O.candidate_what(W, r.S[i], g)).astype(np.float64), 2, 2)
        assert r.losses[i] == pytest.approx(float(np.mean((out - ref) ** 2)), rel=1e-12, abs=1e-300)
    assert r.best == O.first_argmin(list(r.losses))


def test_silent_module_keeps_the_first_candidate():
    """Zero activations: every candidate's Q, K, V and output are 0, every loss 0, and the
    first minimum (alpha = 0) is kept (AWQ-P1 §3)."""
    rng = np.random.default_rng(8)
    X = np.zeros((4, 64), np.float32)
    W = (rng.standard_normal((64, 24)) * 0.1).astype(np.float32)
    r = ATT.attn_search(X, W, n_seq=2, n_heads=2, group=32, n_grid=6)
    assert np.all(r.losses == 0.0) and r.best == 0
