"""Pins of the MLP-block objective oracle (CPU only).

Page: "AWQ：为什么 4-bit 权重量化要先观察 Activation" (AWQ-P1) §4: a candidate may be scored
on the output of the whole module (here an MLP block down(silu(gate) * up)).
"""
import math

import numpy as np
import pytest

import oracle as O
import oracle.awq_module as MOD


def test_silu_special_values():
    assert MOD.silu(0.0) == 0.0
    assert MOD.silu(40.0) == pytest.approx(40.0, rel=1e-15)
    assert abs(MOD.silu(-40.0)) < 1e-15
    # silu(1) = 1 / (1 + 1/e) = e / (e + 1)
    assert MOD.silu(1.0) == pytest.approx(math.e / (math.e + 1.0), rel=1e-15)


def test_block_forward_hand_example():
    """Gate outputs chosen at 0 and at 40 make silu exact (0 and 40 in fp32), so the
    block output follows by hand: h = [0 * u0, 40 * u1], Y = h W_down."""
    X = np.array([[1.0, 2.0]], np.float64)
    W_gu = np.array([[0.0, 4.0, 0.5, 0.25],     # gate columns 0-1, up columns 2-3
                     [0.0, 18.0, 0.5, 0.125]], np.float64)
    # G = [0, 4 + 36] = [0, 40]; U = [1.5, 0.5]; h = [0, 20]
    W_down = np.array([[3.0, 1.0], [0.5, -2.0]], np.float64)
    Y = MOD.mlp_forward(X, W_gu, W_down)
    assert Y.tolist() == [[10.0, -40.0]]


def test_block_forward_rounds_the_intermediate_to_bf16():
    # h = silu(40) * U with U = 1 + 2^-10 is not a bf16 value: it rounds to 40 exactly
    X = np.array([[1.0]], np.float64)
    W_gu = np.array([[40.0, 1.0 + 2.0 ** -10]], np.float64)
    Y = MOD.mlp_forward(X, W_gu, np.array([[1.0]]))
    assert Y[0, 0] == 40.0


def test_weights_on_the_grid_give_zero_loss_at_alpha_zero():
    """With alpha = 0 every scale is 1; weights already on their group's 16-level grid
    (and exact in bf16) quantize to themselves, so candidate 0 reproduces the block."""
    rng = np.random.default_rng(0)
    M, K, F, Ko, g = 16, 64, 8, 24, 32
    levels = rng.integers(0, 16, size=(K, 2 * F)).astype(np.float64)
    levels[0::g] = 0.0   # every group holds both ends of the grid
    levels[1::g] = 15.0
    W_gu = (levels * 0.125 - 1.0).astype(np.float32)
    X = rng.standard_normal((M, K)).astype(np.float32)
    W_down = (rng.standard_normal((F, Ko)) * 0.1).astype(np.float32)
    r = MOD.mlp_search(X, W_gu, W_down, group=g, n_grid=5)
    assert r.losses[0] == 0.0 and r.best == 0
    assert np.all(r.losses[1:] >= 0.0)


def test_block_loss_matches_an_explicit_loop():
    rng = np.random.default_rng(1)
    M, K, F, Ko, g = 3, 8, 2, 3, 4
    X = rng.standard_normal((M, K)).astype(np.float32)
    W_gu = (rng.standard_normal((K, 2 * F)) * 0.3).astype(np.float32)
    W_down = (rng.standard_normal((F, Ko)) * 0.3).astype(np.float32)
    r = MOD.mlp_search(X, W_gu, W_down, group=g, n_grid=4)
    Xb = O.bf16_rne(X).astype(np.float64)
    Wdb = O.bf16_rne(W_down).astype(np.float64)

    def block(Wb):
        out = [[0.0] * Ko for _ in range(M)]
        for m in range(M):
            h = []
            for f in range(F):
                gv = sum(Xb[m, k] * Wb[k, f] for k in range(K))
                uv = sum(Xb[m, k] * Wb[k, F + f] for k in range(K))
                hv = np.float32(gv / (1.0 + math.exp(-gv)) * uv)
                h.append(float(O.bf16_rne(np.array([hv], np.float32))[0]))
            for o in range(Ko):
                out[m][o] = sum(h[f] * Wdb[f, o] for f in range(F))
        return np.array(out)

    ref = block(O.bf16_rne(W_gu).astype(np.float64))
    for i in range(4):
        Wb = O.bf16_rne(O.candidate_what(W_gu, r.S[i], g)).astype(np.float64)
        loss = float(np.mean((block(Wb) - ref) ** 2))
        assert r.losses[i] == pytest.approx(loss, rel=1e-12, abs=1e-300)


def test_silent_block_keeps_the_first_candidate():
    """Zero activations: every candidate's block output is 0, every loss 0, and the first
    minimum (alpha = 0) is kept, as in the scale search (AWQ-P1 §3)."""
    rng = np.random.default_rng(2)
    X = np.zeros((4, 64), np.float32)
    W_gu = (rng.standard_normal((64, 16)) * 0.1).astype(np.float32)
    W_down = (rng.standard_normal((8, 8)) * 0.1).astype(np.float32)
    r = MOD.mlp_search(X, W_gu, W_down, group=32, n_grid=6)
    assert np.all(r.losses == 0.0) and r.best == 0
