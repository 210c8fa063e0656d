"""Planted mistakes in the clipping-search oracle must each fail a pin (CPU only).

Each mutation rewrites one expression of the oracle's clip_search (a plausible slip
in restating AWQ-P1 §5's search), runs the pins of test_oracle_clip_pins.py against
the planted version, and requires that at least one pin fails. The real function is
restored afterwards.
"""
import inspect
import json
import os

import pytest

import oracle.awq_clip as C
from tests import test_oracle_clip_pins as P

MUTATIONS = {
    "weight_mse_instead_of_output_mse": ("partial = xg @ delta", "partial = delta"),
    "unscaled_activations": ("X[rows] / s[None, :]", "X[rows] * s[None, :]"),
    "one_sided_clamp": ("np.minimum(np.maximum(wg, -c[None, :]), c[None, :])", "np.minimum(wg, c[None, :])"),
    "error_against_clamped_weights": ("rec.astype(np.float64) - wg.astype(np.float64)",
                                      "rec.astype(np.float64) - wc.astype(np.float64)"),
    "square_of_mean": ("np.mean(partial ** 2, axis=0)", "np.mean(partial, axis=0) ** 2"),
    "threshold_from_max_not_absmax": ("absmax = np.abs(wg).max(axis=0)", "absmax = wg.max(axis=0)"),
    "last_minimum_wins": ("first_argmin(list(errors[:, g, n]))",
                          "len(errors) - 1 - first_argmin(list(errors[::-1, g, n]))"),
}


def _example():
    with open(os.path.join(os.path.dirname(__file__), "golden", "awq_p1_clipping_counterexample.json")) as f:
        return json.load(f)


def _some_pin_fails() -> bool:
    pins = [lambda: P.test_counterexample_local_gain_whole_loss(_example()),
            P.test_errors_match_an_independent_gram_form,
            P.test_factor_one_is_the_unclipped_quantizer_and_best_is_first_min,
            P.test_silent_group_keeps_the_full_range]
    for pin in pins:
        try:
            pin()
        except Exception:
            return True
    return False


def test_real_oracle_passes_the_pins():
    assert not _some_pin_fails()


@pytest.mark.parametrize("name", list(MUTATIONS))
def test_planted_mistake_is_caught(name, monkeypatch):
    old, new = MUTATIONS[name]
    src = inspect.getsource(C.clip_search)
    assert src.count(old) == 1, f"mutation site not found: {old}"
    ns = dict(vars(C))
    exec(compile(src.replace(old, new), C.__file__, "exec"), ns)
    monkeypatch.setattr(C, "clip_search", ns["clip_search"])
    assert _some_pin_fails(), f"planted mistake {name} passed every pin"
