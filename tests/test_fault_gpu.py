"""Failure detection: a bounded wait in the loss GEMM runs out (B200 only).

The fault hook makes the loss GEMM's producer skip one stage's loads and its arrive,
so the MMA thread waits on a barrier nothing will complete. Every wait in the kernel
is bounded (here 50 ms): the waiting thread raises the CTA's abort flag, the other
roles stop at their next wait, copies and MMAs already issued are allowed to land,
tensor memory is freed, and the call returns AWQ_ERR_TIMEOUT. No trap, no fault,
no hang; the context stays usable and the next search is exact again.
"""
import pytest
import torch

import post_quantization_column_b200 as awq
from workloads import custom_spec, generate

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("variant,form,qdq", [("1", "fused", "standalone"), ("1", "own", "standalone"),
                                              ("1", "own", "warps"), ("2", "own", "standalone")])
def test_wait_that_runs_out_returns_timeout_and_the_context_survives(variant, form, qdq, monkeypatch):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    monkeypatch.setenv("AWQ_GEMM_VARIANT", variant)
    monkeypatch.setenv("AWQ_REFERENCE_LAUNCH", form)
    if qdq == "standalone":
        monkeypatch.setenv("AWQ_QDQ", "standalone")
    else:
        monkeypatch.delenv("AWQ_QDQ", raising=False)
    spec = custom_spec(520, 512, 776, seed=31)
    X, W = (t.cuda() for t in generate(spec))
    ref = awq.search(X, W)
    awq.debug_set_fault(1, 50_000_000)
    try:
        with pytest.raises(awq.AwqError) as err:
            awq.search(X, W)
        assert err.value.status == 6  # AWQ_ERR_TIMEOUT
        assert "wait" in str(err.value)
    finally:
        awq.debug_set_fault(0)
    again = awq.search(X, W)
    for name in ("scales", "codes", "steps", "zeros", "losses"):
        assert torch.equal(getattr(again, name), getattr(ref, name)), name


def test_qdq_warps_count_that_never_arrives_returns_timeout(monkeypatch):
    """The loss GEMM's QDQ warps (bf16 W, group 128) withhold one finished tile's count:
    the producer's bounded wait for that column tile runs out, the call returns
    AWQ_ERR_TIMEOUT, and the next call is exact again."""
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    monkeypatch.delenv("AWQ_QDQ", raising=False)
    monkeypatch.delenv("AWQ_GEMM_VARIANT", raising=False)
    spec = custom_spec(520, 512, 776, seed=32)
    X, W = (t.cuda() for t in generate(spec))
    ref = awq.search(X, W)
    awq.debug_set_fault(3, 50_000_000)
    try:
        with pytest.raises(awq.AwqError) as err:
            awq.search(X, W)
        assert err.value.status == 6  # AWQ_ERR_TIMEOUT
    finally:
        awq.debug_set_fault(0)
    again = awq.search(X, W)
    for name in ("scales", "codes", "steps", "zeros", "losses", "best_index"):
        assert torch.equal(getattr(again, name), getattr(ref, name)), name
