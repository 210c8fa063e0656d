"""Planted mistakes in the attention-block oracle must each fail a pin (CPU only).

Each mutation rewrites one expression of the oracle (a plausible slip in restating the
attention-module objective of AWQ-P1 §4), runs the pins of test_oracle_attn_pins.py, and
requires that at least one fails; the real function is restored afterwards.
"""
import inspect

import pytest

import oracle.awq_attn as ATT
from tests import test_oracle_attn_pins as P

MUTATIONS = {
    "no_causal_mask": ("causal_attention", "s = np.where(causal, s, -np.inf)", "s = s"),
    "no_scaling": ("causal_attention", "e = np.exp((s - m) * inv_sqrt_d)", "e = np.exp(s - m)"),
    "scaled_by_one_over_d": ("causal_attention", "inv_sqrt_d = 1.0 / np.sqrt(float(d))", "inv_sqrt_d = 1.0 / float(d)"),
    "normaliser_from_rounded_weights": ("causal_attention", "l = e.sum(axis=1, keepdims=True)",
                                        "l = bf16_rne(e.astype(np.float32)).astype(np.float64).sum(axis=1, keepdims=True)"),
    "weights_not_rounded": ("causal_attention", "p = bf16_rne(e.astype(np.float32)).astype(np.float64)",
                            "p = e"),
    "softmax_over_queries": ("causal_attention", "m = s.max(axis=1, keepdims=True)",
                             "m = s.max(axis=0, keepdims=True)"),
    "sequences_not_separated": ("causal_attention", "T, d = M // n_seq, D // n_heads", "T, d = M, D // n_heads"),
    "heads_interleaved": ("causal_attention", "cols = slice(h * d, (h + 1) * d)", "cols = slice(h, D, n_heads)"),
    "keys_and_values_swapped": ("attn_forward",
                                "causal_attention(QKV_b[:, :D], QKV_b[:, D:2 * D], QKV_b[:, 2 * D:], n_seq, n_heads)",
                                "causal_attention(QKV_b[:, :D], QKV_b[:, 2 * D:], QKV_b[:, D:2 * D], n_seq, n_heads)"),
    "qkv_not_rounded": ("attn_forward", "QKV_b = bf16_rne(QKV.astype(np.float32)).astype(np.float64)",
                        "QKV_b = QKV"),
    "reference_from_last_candidate": ("attn_search",
                                      "O_ref = attn_forward(X_b, bf16_rne(W_qkv).astype(np.float64), n_seq, n_heads)",
                                      "O_ref = attn_forward(X_b, bf16_rne(candidate_what(W_qkv, S[-1], group)).astype("
                                      "np.float64), n_seq, n_heads)"),
    "last_minimum": ("attn_search", "best = first_argmin(losses)",
                     "best = len(losses) - 1 - first_argmin(list(losses[::-1]))"),
}


def _some_pin_fails() -> bool:
    pins = [P.test_first_token_sees_only_itself, P.test_equal_scores_average_the_values,
            P.test_weights_use_the_scaled_scores_and_the_unrounded_normaliser, P.test_sequences_are_independent,
            P.test_heads_are_contiguous_column_blocks, P.test_qkv_are_rounded_to_bf16, P.test_matches_an_explicit_loop,
            P.test_weights_on_the_grid_give_zero_loss_at_alpha_zero, P.test_search_losses_match_the_loop_module,
            P.test_silent_module_keeps_the_first_candidate]
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
    src = inspect.getsource(getattr(ATT, fn))
    assert src.count(old) == 1, f"mutation site not found: {old}"
    ns = dict(vars(ATT))
    exec(compile(src.replace(old, new), ATT.__file__, "exec"), ns)
    monkeypatch.setattr(ATT, fn, ns[fn])
    assert _some_pin_fails(), f"planted mistake {name} passed every pin"
