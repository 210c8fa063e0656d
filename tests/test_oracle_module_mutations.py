"""Planted mistakes in the MLP-block oracle must each fail a pin (CPU only).

Each mutation rewrites one expression of the oracle (a plausible slip in restating the
block objective of AWQ-P1 §4), runs the pins of test_oracle_module_pins.py, and requires
that at least one fails; the real function is restored afterwards.
"""
import inspect

import pytest

import oracle.awq_module as MOD
from tests import test_oracle_module_pins as P

MUTATIONS = {
    "gelu_tanh_instead_of_silu": ("silu", "return x / (1.0 + np.exp(-x))",
                                  "return 0.5 * x * (1.0 + np.tanh(0.7978845608 * (x + 0.044715 * x ** 3)))"),
    "sigmoid_instead_of_silu": ("silu", "return x / (1.0 + np.exp(-x))", "return 1.0 / (1.0 + np.exp(-x))"),
    "gate_and_up_swapped": ("mlp_forward", "(silu(H[:, :F]) * H[:, F:])", "(silu(H[:, F:]) * H[:, :F])"),
    "no_bf16_rounding_of_h": ("mlp_forward", "h_b = bf16_rne(h).astype(np.float64)", "h_b = h.astype(np.float64)"),
    "down_quantized_too": ("mlp_search", "Wd_b = bf16_rne(W_down).astype(np.float64)",
                           "Wd_b = bf16_rne(candidate_what(W_down, np.ones(W_down.shape[0], np.float32), "
                           "min(group, W_down.shape[0]))).astype(np.float64)"),
    "reference_from_candidate_zero": ("mlp_search", "Y_ref = mlp_forward(X_b, bf16_rne(W_gu).astype(np.float64), Wd_b)",
                                      "Y_ref = mlp_forward(X_b, bf16_rne(candidate_what(W_gu, S[-1], group)).astype("
                                      "np.float64), Wd_b)"),
    "last_minimum": ("mlp_search", "best = first_argmin(losses)",
                     "best = len(losses) - 1 - first_argmin(list(losses[::-1]))"),
}


def _some_pin_fails() -> bool:
    pins = [P.test_silu_special_values, P.test_block_forward_hand_example,
            P.test_block_forward_rounds_the_intermediate_to_bf16, P.test_weights_on_the_grid_give_zero_loss_at_alpha_zero,
            P.test_block_loss_matches_an_explicit_loop, P.test_silent_block_keeps_the_first_candidate]
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
    fn, old, new = MUTATIONS[name]
    src = inspect.getsource(getattr(MOD, fn))
    assert src.count(old) == 1, f"mutation site not found: {old}"
    ns = dict(vars(MOD))
    exec(compile(src.replace(old, new), MOD.__file__, "exec"), ns)
    monkeypatch.setattr(MOD, fn, ns[fn])
    assert _some_pin_fails(), f"planted mistake {name} passed every pin"
