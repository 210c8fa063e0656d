"""Pins of the CPU oracle to what the pages and the mathematics fix (CPU only).

Each test names the passage it follows: the AWQ walk-through page
"AWQ：为什么 4-bit 权重量化要先观察 Activation" (cited as AWQ-P1 with its section).
"""
import itertools
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle as O


@pytest.fixture(scope="module")
def example(golden_dir):
    with open(os.path.join(golden_dir, "awq_p1_worked_example.json")) as f:
        return json.load(f)


def _forward(x, w_hat):
    return float((np.asarray(x, np.float64).ravel() @ np.asarray(w_hat, np.float64).ravel()))


# ---------------------------------------------------------------- AWQ-P1 §2-§3 worked example
def test_worked_example_fixed_scales(example):
    x = np.array(example["x"])
    W = np.array(example["w"])[:, None]
    for case in example["fixed_scale_cases"]:
        s = np.array(case["scales"])
        q, step, rec = O.sym_teaching_qdq(O.scale_weights(W, s), example["group"])
        assert q.ravel().tolist() == case["codes"]
        assert step.item() == pytest.approx(case["step"], abs=1e-15)
        w_hat = O.fold_back(rec, s)
        assert _forward(x, w_hat) == pytest.approx(case["output"], abs=1e-12)
        if "reconstructed_scaled_weights" in case:
            assert rec.ravel() == pytest.approx(case["reconstructed_scaled_weights"], abs=1e-12)


def test_worked_example_search(example):
    x = np.array([example["x"]])
    W = np.array(example["w"])[:, None]
    cfg = example["search"]
    r = O.search(x, W, group=example["group"], n_grid=cfg["n_grid"], quantizer="sym_teaching",
                 arith_dtype=np.float64, bf16_operands=False)
    alphas = O.candidate_alphas(cfg["n_grid"])
    assert len(alphas) == 20 and alphas[-1] == cfg["last_alpha"]
    assert alphas[r.best] == pytest.approx(cfg["chosen_alpha"], abs=1e-12)
    w_hat = O.candidate_what(W, r.S[r.best], example["group"], "sym_teaching")
    assert _forward(x, w_hat) == pytest.approx(cfg["chosen_output_approx"], abs=cfg["output_abs_tol"])
    # the search improves on alpha = 0 (no scaling) but does not reach the hand-picked [10, 1]
    assert r.losses[r.best] < r.losses[0]
    assert r.losses[r.best] > 0
    # loss is the squared output error of the single token (M = N = 1)
    target = example["target_output"]
    assert r.losses[r.best] == pytest.approx((_forward(x, w_hat) - target) ** 2, rel=1e-12)


def test_teaching_quantizer_facts(example):
    facts = example["teaching_quantizer_facts"]
    zg = facts["zero_group"]
    q, step, rec = O.sym_teaching_qdq(np.array(zg["values"])[:, None], 2)
    assert q.ravel().tolist() == zg["codes"] and step.item() == zg["step"]
    assert rec.ravel().tolist() == zg["restored"]
    se = facts["symmetric_ends"]
    assert O.sym_teaching_qdq(np.array(se["values"])[:, None], 2)[0].ravel().tolist() == se["codes"]
    te = facts["ties_to_even"]
    assert O.sym_teaching_qdq(np.array(te["values"])[:, None], 3)[0].ravel().tolist() == te["codes"]
    x = np.array(example["x"])
    W = np.array(example["w"])[:, None]
    for c in facts["common_scales"]:
        s = np.array([c, c])
        rec = O.sym_teaching_qdq(O.scale_weights(W, s), 2)[2]
        assert _forward(x, O.fold_back(rec, s)) == pytest.approx(facts["common_scale_output"], abs=1e-12)
    with pytest.raises(ValueError):
        O.sym_teaching_qdq(np.array([[np.nan]]), 1)


# ---------------------------------------------------------------- AWQ-P1 §7 asymmetric QDQ
def test_asym_hand_derived_cases():
    # worked example at alpha = 0: w = [0.1, 1]: step = 0.9/15 = 0.06, zero = 0,
    # codes [rint(1.67), clamp(rint(16.7))] = [2, 15], reconstruction [0.12, 0.9]
    W = np.array([[0.1], [1.0]], dtype=np.float64)
    q, step, zero, rec = O.asym_qdq(W, 2)
    assert q.ravel().tolist() == [2, 15] and zero.item() == 0
    assert step.item() == pytest.approx(0.06, abs=1e-15)
    assert rec.ravel() == pytest.approx([0.12, 0.9], abs=1e-12)
    # a group straddling zero that lands on the grid: [-1, 2] -> step 0.2, zero 5, exact
    q, step, zero, rec = O.asym_qdq(np.array([[-1.0], [2.0]]), 2)
    assert q.ravel().tolist() == [0, 15] and zero.item() == 5
    assert rec.ravel() == pytest.approx([-1.0, 2.0], abs=1e-12)
    # an all-equal group gets step 1 (zero = clamp(rint(-v)))
    q, step, zero, rec = O.asym_qdq(np.array([[-3.0], [-3.0]], dtype=np.float32), 2)
    assert step.item() == 1.0 and zero.item() == 3 and q.ravel().tolist() == [0, 0]
    q, step, zero, rec = O.asym_qdq(np.array([[2.0], [2.0]], dtype=np.float32), 2)
    assert step.item() == 1.0 and zero.item() == 0 and q.ravel().tolist() == [2, 2]
    # the zero point is an integer: -min/step = -0.25 rounds to -0, stored as +0
    q, step, zero, rec = O.asym_qdq(np.array([[0.25], [0.25]], dtype=np.float32), 2)
    assert zero.item() == 0 and not np.signbit(zero).any()
    assert not np.signbit(zero.astype(np.float16)).any()


@pytest.mark.parametrize("gsize", [2, 3, 4])
def test_asym_brute_force_all_codes(gsize):
    """For the produced (step, zero), the codes are the best of all 16**g code vectors."""
    rng = np.random.default_rng(100 + gsize)
    levels = np.arange(16)
    for trial in range(40):
        w = (rng.standard_normal(gsize) * rng.choice([0.01, 1.0, 30.0]) + rng.choice([0.0, 0.5, -2.0]))
        w = w.astype(np.float32)[:, None]
        q, step, zero, rec = O.asym_qdq(w, gsize)
        st, z = np.float64(step.item()), np.float64(zero.item())
        assert 0 <= z <= 15 and st > 0
        # step/zero from the group's own range: when the zero is not clamped (the group
        # straddles 0), the 16 levels span [min, max] up to step/2; a one-signed group
        # clamps the zero and clips one end (AWQ-P1 §7 clamp to [0, 15])
        r = np.rint(-float(w.min()) / st)
        if 0 <= r <= 15:
            assert z == r
            assert -z * st <= float(w.min()) + st * (0.5 + 1e-5)
            assert (15 - z) * st >= float(w.max()) - st * (0.5 + 1e-5)
        else:
            assert z == (0 if r < 0 else 15)
        best_err, best = None, []
        for codes in itertools.product(levels, repeat=gsize):
            err = sum((float(w[i, 0]) - st * (codes[i] - z)) ** 2 for i in range(gsize))
            if best_err is None or err < best_err - 1e-18:
                best_err, best = err, [codes]
            elif abs(err - best_err) <= 1e-18:
                best.append(codes)
        assert tuple(q.ravel().tolist()) in best
        # per-element error bound inside the representable range (AWQ-P1 §3: Delta/2)
        inside = (w[:, 0] >= -z * st) & (w[:, 0] <= (15 - z) * st)
        assert np.all(np.abs(rec[:, 0] - w[:, 0])[inside] <= st / 2 * (1 + 1e-6))


def test_asym_ties_to_even():
    # w'/step exactly x.5 with step 1 after an all-equal group is impossible; use a
    # group whose step is 1: [0, 15] -> step 1, zero 0; 2.5 -> 2, 3.5 -> 4
    W = np.array([[0.0], [15.0], [2.5], [3.5]], dtype=np.float32)
    q, step, zero, _ = O.asym_qdq(W, 4)
    assert step.item() == 1.0 and zero.item() == 0
    assert q.ravel().tolist() == [0, 15, 2, 4]


# ---------------------------------------------------------------- AWQ-P1 §3 fold-back invariants
def test_foldback_without_quantization_reproduces_w():
    rng = np.random.default_rng(7)
    W = (rng.standard_normal((64, 16)) * 0.02).astype(np.float32)
    s = np.exp(rng.standard_normal(64)).astype(np.float32)
    # in fp64 the product of two fp32 numbers is exact, so the round trip is exact
    back64 = O.candidate_what(W.astype(np.float64), s.astype(np.float64), 64, "none")
    assert np.array_equal(back64, W.astype(np.float64))
    # in fp32 each of the two roundings costs at most half an ulp: at most 1 ulp apart
    back32 = O.candidate_what(W, s, 64, "none")
    ulp = np.spacing(np.abs(W))
    assert np.all(np.abs(back32 - W) <= ulp)
    # powers of two are exact in fp32 as well
    s2 = np.exp2(rng.integers(-6, 7, size=64)).astype(np.float32)
    assert np.array_equal(O.candidate_what(W, s2, 64, "none"), W)


def test_common_power_of_two_scale_invariance():
    """Scaling a whole group by 2^k changes steps by 2^k and nothing else (AWQ-P1 §3)."""
    rng = np.random.default_rng(11)
    W = (rng.standard_normal((256, 24)) * 0.02).astype(np.float32)
    s = np.exp(0.5 * rng.standard_normal(256)).astype(np.float32)
    q1, st1, z1, _ = O.asym_qdq(O.scale_weights(W, s), 128)
    for k in (-3, 1, 5):
        s2 = (s * np.float32(2.0 ** k)).astype(np.float32)
        q2, st2, z2, _ = O.asym_qdq(O.scale_weights(W, s2), 128)
        assert np.array_equal(q1, q2) and np.array_equal(z1, z2)
        assert np.array_equal(st2, (st1 * np.float32(2.0 ** k)).astype(np.float32))
        assert np.array_equal(O.candidate_what(W, s, 128), O.candidate_what(W, s2, 128))


# ---------------------------------------------------------------- AWQ-P1 §1 statistic
def test_statistic_rational_brute_force():
    rng = np.random.default_rng(3)
    X = (rng.standard_normal((7, 5)) * np.exp(rng.standard_normal(5))).astype(np.float32)
    X[:, 2] = 0.0
    a = O.activation_statistic(X)
    for j in range(X.shape[1]):
        exact = sum(Fraction(abs(float(v))) for v in X[:, j]) / X.shape[0]
        # the fp32 value nearest the exact rational mean (X is tiny, so fp64 is exact here)
        assert a[j] == np.float32(float(exact))
    assert a[2] == 0.0
    with pytest.raises(ValueError):
        O.activation_statistic(np.array([[1.0, np.inf]]))


# ---------------------------------------------------------------- AWQ-P1 §3-§4 scales
def test_scale_family_brute_force():
    a = np.array([3.0, 0.5, 0.0, 12.0, 1e-6], dtype=np.float32)
    S = O.candidate_scales(a, 20)
    assert S.shape == (20, 5)
    assert np.all(S[0] == 1.0)  # alpha = 0 gives all ones, even for a zero channel
    for i in range(20):
        alpha = i / 20
        raw = [max(math.pow(float(v), alpha), 1e-4) for v in a]  # clamp BEFORE normalising
        nrm = math.sqrt(max(raw) * min(raw))
        assert S[i].tolist() == [float(np.float32(r / nrm)) for r in raw]
        # geometric normalisation: max * min == 1 up to the final fp32 rounding
        assert float(S[i].max()) * float(S[i].min()) == pytest.approx(1.0, rel=1e-6)
    assert np.all(O.candidate_alphas(20) < 1.0)


# ---------------------------------------------------------------- AWQ-P1 §1, §4 loss
def _gram_loss(X, W, W_hat):
    """Sum_n e_n^T (X^T X) e_n / (M N), written with explicit loops (the X^T X form)."""
    M, K = len(X), len(X[0])
    N = len(W[0])
    G = [[sum(X[m][i] * X[m][j] for m in range(M)) for j in range(K)] for i in range(K)]
    total = 0.0
    for n in range(N):
        e = [W_hat[k][n] - W[k][n] for k in range(K)]
        total += sum(e[i] * G[i][j] * e[j] for i in range(K) for j in range(K))
    return total / (M * N)


def test_loss_matches_gram_form():
    rng = np.random.default_rng(5)
    X = rng.standard_normal((6, 8))
    W = rng.standard_normal((8, 3)) * 0.1
    W_hat = W + rng.standard_normal((8, 3)) * 0.01
    got = O.output_loss(X, W, W_hat)
    ref = _gram_loss(X.tolist(), W.tolist(), W_hat.tolist())
    assert got == pytest.approx(ref, rel=1e-10)
    # a single token and a single output reduce to the squared output error
    x = X[:1]
    assert O.output_loss(x, W[:, :1], W_hat[:, :1]) == pytest.approx(
        float((x @ (W_hat[:, :1] - W[:, :1])).item()) ** 2, rel=1e-12)


def test_search_loss_matches_gram_form_end_to_end():
    rng = np.random.default_rng(9)
    X = (rng.standard_normal((5, 64)) * np.exp(rng.standard_normal(64))).astype(np.float32)
    W = (rng.standard_normal((64, 8)) * 0.02).astype(np.float32)
    r = O.search(X, W, group=32, n_grid=4)
    Xb = O.bf16_rne(X).astype(np.float64)
    Wb = O.bf16_rne(W).astype(np.float64)
    for i in range(4):
        W_hat = O.bf16_rne(O.candidate_what(W, r.S[i], 32)).astype(np.float64)
        assert r.losses[i] == pytest.approx(_gram_loss(Xb.tolist(), Wb.tolist(), W_hat.tolist()), rel=1e-9)


def test_zero_loss_when_weights_sit_on_the_grid():
    rng = np.random.default_rng(13)
    K, N, group = 64, 8, 32
    step = np.float32(0.0625)
    q = rng.integers(0, 16, size=(K, N))
    q[0::group, :] = 0
    q[1::group, :] = 15          # every group spans the full code range
    zero = 7
    W = ((q - zero) * step).astype(np.float32)
    X = rng.standard_normal((4, K)).astype(np.float32)
    r = O.search(X, W, group=group, n_grid=3)
    assert r.losses[0] == 0.0     # alpha = 0: s = 1, Q(W) = W exactly
    assert r.best == 0
    assert np.array_equal(r.q, q) and np.all(r.zero == zero) and np.all(r.step == step)


# ---------------------------------------------------------------- number formats
def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(17)
    v = np.concatenate([
        rng.standard_normal(20000).astype(np.float32) * np.float32(10.0) ** rng.integers(-30, 30, 20000),
        np.array([1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, -(1.0 + 2.0 ** -8), 0.0, -0.0, 1e-40, 3.3e38],
                 dtype=np.float32),
    ]).astype(np.float32)
    ref = torch.from_numpy(v).to(torch.bfloat16).float().numpy()
    got = O.bf16_rne(v)
    assert np.array_equal(got.view(np.uint32), ref.view(np.uint32))


def test_first_argmin_keeps_first():
    assert O.first_argmin([3.0, 1.0, 1.0, 2.0]) == 1
    assert O.first_argmin([0.5]) == 0


# ---------------------------------------------------------------- AWQ-P1 §7-§8 artifact
def test_pack_roundtrip_and_layout():
    rng = np.random.default_rng(19)
    q = rng.integers(0, 16, size=(6, 16))
    words = O.pack_codes(q)
    assert words.dtype == np.int32 and words.shape == (6, 2)
    assert np.array_equal(O.unpack_codes(words, 16), q)
    w0 = int(words.view(np.uint32)[0, 0])
    assert [(w0 >> (4 * i)) & 0xF for i in range(8)] == q[0, :8].tolist()


def test_artifact_decodes_to_search_reconstruction():
    """Decode codes/steps/zeros and compare with the search's own Q/DQ (AWQ-P1 §7 check)."""
    rng = np.random.default_rng(23)
    X = (rng.standard_normal((16, 256)) * np.exp(0.5 * rng.standard_normal(256))).astype(np.float32)
    W = (rng.standard_normal((256, 16)) * 0.02).astype(np.float32)
    r = O.search(X, W, group=128, n_grid=20)
    dec = O.decode_artifact(r.codes, r.steps_f16, r.zeros_f16, 128, 16)
    rec = O.asym_qdq(O.scale_weights(W, r.scales), 128)[3]
    # only the fp16 rounding of the step separates the two
    st = np.repeat(r.step, 128, axis=0)
    assert np.all(np.abs(dec - rec) <= 15 * st * 2.0 ** -11 + 1e-30)


def test_bits_per_weight_budget():
    # AWQ-P1 §8: group 128 with fp16 step + fp16 zero -> 4.25 bits/weight, ~3.76x vs 16-bit
    assert O.bits_per_weight(4096, 4096, 128) == 4.25
    assert 16 / O.bits_per_weight(4096, 4096, 128) == pytest.approx(3.76, abs=0.005)


def test_symmetric_artifact_decodes_to_the_teaching_quantizer():
    """The teaching quantizer (AWQ-P1 §2) in the unsigned artifact: code = q + 7, zero 7;
    the page's worked example at S = diag(10, 1) has q = [7, 7], so the codes are 14."""
    Wp = np.array([[1.0], [1.0]], np.float32)  # 10 * 0.1 and 1 * 1 in one group
    q, step, zero = O.sym_artifact(Wp, 2)
    assert q[:, 0].tolist() == [14, 14] and zero.tolist() == [[7.0]]
    assert step[0, 0] == np.float32(1.0) / np.float32(7.0)
    rng = np.random.default_rng(31)
    W = (rng.standard_normal((256, 16)) * 0.02).astype(np.float32)
    W[:128, 3] = 0.0                                   # an all-zero group: step 1, codes 7
    q, step, zero = O.sym_artifact(W, 128)
    assert q.min() >= 0 and q.max() <= 14 and np.all(q[:128, 3] == 7) and step[0, 3] == 1.0
    rec = O.sym_teaching_qdq(W, 128)[2]
    dec = O.decode_artifact(O.pack_codes(q), O.fp16_rne(step), zero.astype(np.float16), 128, 16)
    st = np.repeat(step, 128, axis=0)
    assert np.all(np.abs(dec - rec) <= 7 * st * 2.0 ** -11 + 1e-30)
