"""Each step's kernel against the oracle, bit for bit (B200 only).

The per-step entry points run the same kernels the search runs. Every input a step
takes from an earlier step comes from the oracle here, so each kernel is checked on
its own: the statistic on X, the scale family on the oracle's statistic, and the
candidate QDQ + fold-back on the oracle's scales.
"""
import numpy as np
import pytest
import torch

import oracle as O
import post_quantization_column_b200 as awq
from workloads import WORKLOADS, custom_spec, generate, as_f32_numpy

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def _bits(a):
    a = np.ascontiguousarray(a)
    return a.view(np.uint32 if a.dtype == np.float32 else np.uint16)


def _oracle_operands(W32, S, group):
    """(n_grid + 1, N, K) bf16 bit patterns: bf16(W)^T, then bf16(W_hat_i)^T."""
    slots = [O.bf16_rne(W32).T]
    for i in range(S.shape[0]):
        slots.append(O.bf16_rne(O.candidate_what(W32, S[i], group)).T)
    return np.stack([(np.ascontiguousarray(s).view(np.uint32) >> 16).astype(np.uint16) for s in slots])


def _gpu_operands(W, S, group):
    out = awq.qdq_candidates(W.cuda(), torch.from_numpy(S).cuda(), group)
    return out.view(torch.int16).cpu().numpy().view(np.uint16)


@pytest.mark.parametrize("name", list(WORKLOADS))
def test_statistic_bit_exact(name):
    spec = WORKLOADS[name]
    X, _ = generate(spec)
    a = awq.activation_statistic(X.cuda()).cpu().numpy()
    ref = O.activation_statistic(as_f32_numpy(X))
    assert np.array_equal(_bits(a), _bits(ref))


@pytest.mark.parametrize("M,K,dtype", [(1000, 4832, "bf16"), (777, 2400, "f32"), (37, 4096, "bf16"),
                                       (3001, 256, "f32"), (130, 11008, "bf16")])
def test_statistic_ragged_shapes(M, K, dtype):
    # row counts that leave a partial batch of row loads, and K that leaves the last
    # cluster's column block partly outside X, in both cluster widths (64/128 bf16 columns
    # per cluster for K up to / above about 4.7k; 32/64 fp32 ones up to / above 2.4k)
    X, _ = generate(custom_spec(M, K, 8, dtype=dtype, seed=5))
    a = awq.activation_statistic(X.cuda()).cpu().numpy()
    ref = O.activation_statistic(as_f32_numpy(X))
    assert np.array_equal(_bits(a), _bits(ref))


@pytest.mark.parametrize("name", list(WORKLOADS))
def test_scales_bit_exact_for_every_candidate(name):
    spec = WORKLOADS[name]
    X, _ = generate(spec)
    a = O.activation_statistic(as_f32_numpy(X))
    S = awq.candidate_scales(torch.from_numpy(a).cuda(), spec.n_grid).cpu().numpy()
    ref = O.candidate_scales(a, spec.n_grid)
    bad = np.argwhere(_bits(S) != _bits(ref))
    assert bad.size == 0, f"{len(bad)} scales differ, first {bad[:4].tolist()}"


def test_scales_edge_cases():
    # zero channels, a single channel, tiny and huge statistics (clamp before normalising)
    for a in (np.array([0.0, 0.0, 3.0, 1e-30], np.float32), np.array([2.5], np.float32),
              np.array([1e-12, 1e12, 1.0, 0.0], np.float32)):
        S = awq.candidate_scales(torch.from_numpy(a).cuda(), 20).cpu().numpy()
        assert np.array_equal(_bits(S), _bits(O.candidate_scales(a, 20)))


@pytest.mark.parametrize("M,K,N,group,dtype", [
    (64, 384, 520, 128, "bf16"), (64, 160, 264, 32, "bf16"), (64, 320, 776, 64, "f32"), (64, 256, 8, 128, "bf16"),
])
def test_qdq_candidates_bit_exact(M, K, N, group, dtype):
    spec = custom_spec(M, K, N, dtype=dtype, group=group, seed=K + N)
    X, W = generate(spec)
    S = O.candidate_scales(O.activation_statistic(as_f32_numpy(X)), 20)
    got = _gpu_operands(W, S, group)
    ref = _oracle_operands(as_f32_numpy(W), S, group)
    bad = np.argwhere(got != ref)
    assert bad.size == 0, f"{len(bad)} operand values differ, first (slot, n, k) {bad[:4].tolist()}"


@pytest.mark.parametrize("name", ["llama7b_mlp_down_4096x11008x4096", "llama70b_mlp_gate_up_16384x8192x57344"])
def test_qdq_candidates_bit_exact_on_workload_columns(name):
    spec = WORKLOADS[name]
    X, W = generate(spec)
    S = O.candidate_scales(O.activation_statistic(as_f32_numpy(X)), spec.n_grid)
    cols = torch.cat([W[:, :256], W[:, -256:]], dim=1).contiguous()
    got = _gpu_operands(cols, S, spec.group)
    ref = _oracle_operands(as_f32_numpy(cols), S, spec.group)
    bad = np.argwhere(got != ref)
    assert bad.size == 0, f"{len(bad)} operand values differ, first {bad[:4].tolist()}"


def test_qdq_exact_ties_take_the_exact_path():
    # every scaled weight sits exactly half-way between two levels (rint ties to even),
    # and the steps make many folded-back values land on bf16 rounding midpoints
    K, N, group = 256, 64, 128
    k = np.arange(K)[:, None] % 16
    W = np.zeros((K, N), np.float32)
    W[:, :32] = (k * 0.0625 + 0.03125).astype(np.float32)       # x.5 quotients, step 1/16
    W[:, 32:] = (k * (1.0 + 2.0 ** -8)).astype(np.float32)       # multiples of a bf16-midpoint step
    S = np.ones((3, K), np.float32)
    S[1] = 2.0                                                   # power-of-two scales: exact
    S[2] = np.linspace(0.5, 3.0, K, dtype=np.float32)            # generic scales
    got = _gpu_operands(torch.from_numpy(W), S, group)
    ref = _oracle_operands(W, S, group)
    assert np.array_equal(got, ref)


def test_pack_matches_oracle_on_ties():
    # the artifact kernel shares the fast path: exact ties must still round to even
    K, N, group = 128, 64, 128
    k = np.arange(K)[:, None] % 16
    W = np.tile((k * 0.0625 + 0.03125).astype(np.float32), (1, N))
    X = np.ones((4, K), np.float32)
    out = awq.search(torch.from_numpy(X).cuda(), torch.from_numpy(W).cuda(), group, 1)
    q, step, zero, _ = O.asym_qdq(W, group)
    assert np.array_equal(out.codes.cpu().numpy(), O.pack_codes(q))
    assert np.array_equal(out.zeros.cpu().numpy().view(np.uint16), zero.astype(np.float16).view(np.uint16))
