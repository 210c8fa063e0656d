"""Planted mistakes in the oracle must each fail at least one pin (CPU only).

Each mutation below is a plausible slip in restating the search (a wrong rounding, a
flipped sign, a dropped term, an off-by-one grid, a transposed operand). The test
swaps it into the oracle module, runs the pins of test_oracle_pins.py, and requires
that at least one of them fails; the real oracle is restored afterwards.
"""
import json
import os

import numpy as np
import pytest

import oracle
import oracle.awq_oracle as AO
from tests import test_oracle_pins as P

PINS_FAST_FIRST = [
    "test_worked_example_fixed_scales", "test_worked_example_search", "test_teaching_quantizer_facts",
    "test_asym_hand_derived_cases", "test_asym_ties_to_even", "test_foldback_without_quantization_reproduces_w",
    "test_common_power_of_two_scale_invariance", "test_statistic_rational_brute_force",
    "test_scale_family_brute_force", "test_loss_matches_gram_form", "test_search_loss_matches_gram_form_end_to_end",
    "test_zero_loss_when_weights_sit_on_the_grid", "test_bf16_rounding_matches_torch",
    "test_first_argmin_keeps_first", "test_pack_roundtrip_and_layout",
    "test_artifact_decodes_to_search_reconstruction",
]


def _example():
    with open(os.path.join(os.path.dirname(__file__), "golden", "awq_p1_worked_example.json")) as f:
        return json.load(f)


def _some_pin_fails() -> bool:
    ex = _example()
    for name in PINS_FAST_FIRST:
        fn = getattr(P, name)
        try:
            if "example" in fn.__code__.co_varnames[: fn.__code__.co_argcount]:
                fn(ex)
            else:
                fn()
        except Exception:
            return True
    # the brute-force pin last (slowest)
    try:
        P.test_asym_brute_force_all_codes(3)
    except Exception:
        return True
    return False


def _asym_variant(*, rounding=np.rint, zero_sign=1.0, levels=15):
    def asym_qdq(Wp, group):
        Wp = np.asarray(Wp)
        dt = Wp.dtype.type
        Wg = AO._groups(Wp, group)
        mn, mx = Wg.min(axis=1), Wg.max(axis=1)
        step = ((mx - mn) / dt(levels)).astype(dt)
        step = np.where((mx == mn) | (step == 0), dt(1), step).astype(dt)
        zero = np.clip(rounding((zero_sign * -mn / step).astype(dt)), 0, 15).astype(dt)
        q = np.clip(rounding((Wg / step[:, None, :]).astype(dt)) + zero[:, None, :], 0, 15).astype(dt)
        rec = ((q - zero[:, None, :]) * step[:, None, :]).astype(dt)
        K, N = Wp.shape
        return q.reshape(K, N).astype(np.int32), step, zero, rec.reshape(K, N)
    return asym_qdq


def _sym_variant(*, rounding=np.rint, levels=7):
    def sym_teaching_qdq(Wp, group):
        Wp = np.asarray(Wp)
        dt = Wp.dtype.type
        if not np.all(np.isfinite(Wp)):
            raise ValueError("finite")
        Wg = AO._groups(Wp, group)
        peak = np.abs(Wg).max(axis=1)
        step = np.where(peak == 0, dt(1), peak / dt(levels)).astype(dt)
        q = np.clip(rounding(Wg / step[:, None, :]), -7, 7).astype(dt)
        rec = (q * step[:, None, :]).astype(dt)
        K, N = Wp.shape
        return q.reshape(K, N).astype(np.int32), step, rec.reshape(K, N)
    return sym_teaching_qdq


def _half_away(v):
    return np.sign(v) * np.floor(np.abs(v) + 0.5)


def _scales_variant(*, normalise_first=False, include_one=False):
    def candidate_scales(a, n_grid, out_dtype=np.float32):
        a64 = np.asarray(a, dtype=np.float64)
        S = np.empty((n_grid, a64.size), dtype=out_dtype)
        for i in range(n_grid):
            alpha = i / (n_grid - 1) if include_one else i / n_grid
            raw = np.power(a64, alpha)
            if normalise_first:
                raw = np.maximum(raw / np.sqrt(raw.max() * max(raw.min(), 1e-300)), AO.CLAMP_MIN)
                S[i] = raw.astype(out_dtype)
            else:
                raw = np.maximum(raw, AO.CLAMP_MIN)
                S[i] = (raw / np.sqrt(raw.max() * raw.min())).astype(out_dtype)
        return S
    return candidate_scales


def _fold_back_multiply(rec, s):
    return (np.asarray(rec) * np.asarray(s, dtype=np.asarray(rec).dtype)[:, None]).astype(np.asarray(rec).dtype)


def _statistic_signed(X, out_dtype=np.float32):
    X64 = np.asarray(X, dtype=np.float64)
    return np.abs(X64.sum(axis=0) / X64.shape[0]).astype(out_dtype)


def _bf16_truncate(x):
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    return (u & np.uint32(0xFFFF0000)).view(np.float32)


def _last_argmin(losses):
    best = 0
    for i in range(1, len(losses)):
        if losses[i] <= losses[best]:
            best = i
    return best


def _pack_reversed(q):
    q = np.asarray(q, dtype=np.int64)
    K, N = q.shape
    words = np.zeros((K, N // 8), dtype=np.int64)
    for i in range(8):
        words |= (q[:, i::8] & 0xF) << (4 * (7 - i))
    return words.astype(np.uint32).view(np.int32)


def _loss_abs(Yhat, Y):
    return float(np.mean(np.abs(np.asarray(Yhat) - np.asarray(Y))))


MUTATIONS = {
    "floor_instead_of_rint": {"asym_qdq": _asym_variant(rounding=np.floor)},
    "round_half_away": {"asym_qdq": _asym_variant(rounding=_half_away),
                        "sym_teaching_qdq": _sym_variant(rounding=_half_away)},
    "zero_sign_flipped": {"asym_qdq": _asym_variant(zero_sign=-1.0)},
    "sixteen_levels": {"asym_qdq": _asym_variant(levels=16)},
    "teaching_eight_levels": {"sym_teaching_qdq": _sym_variant(levels=8)},
    "clamp_after_normalising": {"candidate_scales": _scales_variant(normalise_first=True)},
    "grid_includes_one": {"candidate_scales": _scales_variant(include_one=True)},
    "fold_back_multiplies": {"fold_back": _fold_back_multiply},
    "statistic_of_signed_mean": {"activation_statistic": _statistic_signed},
    "bf16_truncates": {"bf16_rne": _bf16_truncate},
    "argmin_keeps_last": {"first_argmin": _last_argmin},
    "pack_nibbles_reversed": {"pack_codes": _pack_reversed},
    "loss_abs_not_square": {"squared_error_mean": _loss_abs},
}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_planted_mistake_is_caught(name, monkeypatch):
    for attr, fn in MUTATIONS[name].items():
        monkeypatch.setattr(AO, attr, fn)
        monkeypatch.setattr(oracle, attr, fn)
    assert _some_pin_fails(), f"mutation {name!r} passed every pin"
