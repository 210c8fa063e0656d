"""Planted mistakes in the W4A16 consumer oracle must each fail a pin (CPU only).

Each mutation rewrites one expression of the oracle (a plausible slip in restating the
consumer of AWQ-P1 §6-§8), runs the pins of test_oracle_w4a16_pins.py, and requires that
at least one of them fails; the real function is restored afterwards.
"""
import inspect

import pytest

import oracle.awq_w4a16 as Q
from tests import test_oracle_w4a16_pins as P

MUTATIONS = {
    "zero_added": ("dequant_operand", "exact = (q - zr) * st", "exact = (q + zr) * st"),
    "bf16_rounding": ("dequant_operand", "return exact.astype(np.float16)",
                      "return ((exact.astype(np.float32).view(np.uint32) + 0x8000) & 0xFFFF0000)"
                      ".view(np.float32).astype(np.float16)"),
    "step_not_applied": ("dequant_operand", "exact = (q - zr) * st", "exact = (q - zr)"),
    "groups_tiled_not_repeated": ("dequant_operand",
                                  "st = np.repeat(np.asarray(steps_f16, dtype=np.float16).astype(np.float64), group, axis=0)",
                                  "st = np.tile(np.asarray(steps_f16, dtype=np.float16).astype(np.float64), (group, 1))"),
    "activations_times_scales": ("fp16_activations", "(X / s[None, :])", "(X * s[None, :])"),
    "weights_transposed": ("w4a16_matmul", "return A @ W", "return A @ W[::-1]"),
}


def _some_pin_fails() -> bool:
    pins = [P.test_hand_built_artifact_decodes_to_the_definition, P.test_matmul_is_the_exact_sum_of_exact_products,
            P.test_alignment_check_against_the_search, P.test_activations_are_divided_by_the_scales,
            P.test_group_boundaries_use_their_own_step]
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
    src = inspect.getsource(getattr(Q, fn))
    assert src.count(old) == 1, f"mutation site not found: {old}"
    ns = dict(vars(Q))
    exec(compile(src.replace(old, new), Q.__file__, "exec"), ns)
    monkeypatch.setattr(Q, fn, ns[fn])  # also what w4a16_matmul finds in the module's globals
    assert _some_pin_fails(), f"planted mistake {name} passed every pin"
