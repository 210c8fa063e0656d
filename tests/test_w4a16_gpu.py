"""The W4A16 consumer of the artifact against the oracle (B200 only).

Pages: "AWQ：为什么 4-bit 权重量化要先观察 Activation" §6-§8 (the artifact's consumer and
its alignment check). The dequantized operand is bit-exact; the output's products are
exact on both sides and only the order of the fp32 sums differs, so every output lies
within ACC_RTOL x sum_k |a| |w| of the oracle's exact value (the fp32 accumulation bound
for these depths, with margin).
"""
import numpy as np
import pytest
import torch

import oracle as O
import oracle.awq_w4a16 as Q
import post_quantization_column_b200 as awq
from workloads import WORKLOADS, custom_spec, generate, as_f32_numpy

pytestmark = pytest.mark.gpu

ACC_RTOL = 2e-5


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def _random_artifact(K, N, group, seed):
    rng = np.random.default_rng(seed)
    q = rng.integers(0, 16, size=(K, N))
    steps = (rng.random((K // group, N)) * 0.01 + 1e-4).astype(np.float16)
    zeros = rng.integers(0, 16, size=(K // group, N)).astype(np.float16)
    return O.pack_codes(q), steps, zeros


def _dev(codes, steps, zeros):
    return (torch.from_numpy(np.ascontiguousarray(codes)).cuda(), torch.from_numpy(steps).cuda(),
            torch.from_numpy(zeros).cuda())


def _check_output(Y, A16, codes, steps, zeros, group):
    ref = Q.w4a16_matmul(A16, codes, steps, zeros, group)
    W = Q.dequant_operand(codes, steps, zeros, group, steps.shape[1]).astype(np.float64)
    bound = ACC_RTOL * (np.abs(A16.astype(np.float64)) @ np.abs(W)) + 1e-30
    bad = np.argwhere(np.abs(Y.astype(np.float64) - ref) > bound)
    assert bad.size == 0, f"{len(bad)} outputs off, first {bad[:4].tolist()}: {Y[tuple(bad[0])]} vs {ref[tuple(bad[0])]}"


@pytest.mark.parametrize("K,N,group", [(256, 264, 128), (160, 72, 32), (384, 520, 64), (128, 8, 128)])
def test_dequant_operand_bit_exact(K, N, group):
    codes, steps, zeros = _random_artifact(K, N, group, K + N)
    got = awq.w4a16_dequant(*_dev(codes, steps, zeros), group).cpu().numpy()
    ref = Q.dequant_operand(codes, steps, zeros, group, N).T
    assert np.array_equal(got.view(np.uint16), np.ascontiguousarray(ref).view(np.uint16))


@pytest.mark.parametrize("M", [1, 2, 3, 5, 8, 9, 16, 17, 64, 300])
@pytest.mark.parametrize("K,N,group", [(256, 264, 128), (160, 72, 32), (384, 520, 64)])
def test_matmul_matches_oracle(M, K, N, group):
    codes, steps, zeros = _random_artifact(K, N, group, M * 7 + K)
    A = (np.random.default_rng(M).standard_normal((M, K)) * 2).astype(np.float16)
    Y = awq.w4a16_matmul(torch.from_numpy(A).cuda(), *_dev(codes, steps, zeros), group).cpu().numpy()
    _check_output(Y, A, codes, steps, zeros, group)


def test_search_artifact_end_to_end_alignment():
    """AWQ-P1 §7: search on the GPU, consume its artifact on the GPU with the activations
    divided by the chosen scales; the output is the oracle consumer's and stays within the
    16-bit roundings of the folded-back layer's output."""
    spec = custom_spec(512, 512, 264, dtype="bf16", seed=17)
    X, W = generate(spec)
    out = awq.search(X.cuda(), W.cuda(), 128, 20)
    X32, W32 = as_f32_numpy(X), as_f32_numpy(W)
    s = out.scales.cpu().numpy()
    codes, steps, zeros = (t.cpu().numpy() for t in (out.codes, out.steps, out.zeros))
    A16 = Q.fp16_activations(X32, s)
    Y = awq.w4a16_matmul(torch.from_numpy(A16).cuda(), out.codes, out.steps, out.zeros, 128).cpu().numpy()
    _check_output(Y, A16, codes, steps, zeros, 128)
    rec = O.asym_qdq(O.scale_weights(W32, s), 128)[3].astype(np.float64)
    ref = X32.astype(np.float64) @ O.fold_back(rec, s.astype(np.float64))
    assert np.linalg.norm(Y - ref) <= 2e-3 * np.linalg.norm(ref)
    # and the few-token path on the same artifact
    Y4 = awq.w4a16_matmul(torch.from_numpy(A16[:4]).cuda(), out.codes, out.steps, out.zeros, 128).cpu().numpy()
    _check_output(Y4, A16[:4], codes, steps, zeros, 128)


def test_clipped_artifact_is_consumed_too():
    spec = custom_spec(256, 256, 136, dtype="bf16", seed=19)
    X, W = generate(spec)
    out = awq.search(X.cuda(), W.cuda(), 128, 20)
    clip = awq.clip_search(X.cuda(), W.cuda(), out.scales, 128)
    A16 = Q.fp16_activations(as_f32_numpy(X), out.scales.cpu().numpy())
    for M in (1, 200):
        Y = awq.w4a16_matmul(torch.from_numpy(A16[:M]).cuda(), clip.codes, clip.steps, clip.zeros, 128).cpu().numpy()
        _check_output(Y, A16[:M], clip.codes.cpu().numpy(), clip.steps.cpu().numpy(), clip.zeros.cpu().numpy(), 128)


def test_matmul_is_deterministic():
    codes, steps, zeros = _random_artifact(512, 1032, 128, 3)
    d = _dev(codes, steps, zeros)
    for M in (1, 7, 130):
        A = torch.from_numpy((np.random.default_rng(M).standard_normal((M, 512))).astype(np.float16)).cuda()
        a, b = awq.w4a16_matmul(A, *d, 128), awq.w4a16_matmul(A, *d, 128)
        assert torch.equal(a, b)


@pytest.mark.parametrize("name", ["llama7b_mlp_down_4096x11008x4096", "llama70b_mlp_gate_up_16384x8192x57344"])
@pytest.mark.parametrize("M", [1, 16, 256])
def test_full_size_sampled_columns(name, M):
    """A random artifact of the layer's shape; the oracle recomputes column blocks."""
    spec = WORKLOADS[name]
    K, N, g = spec.K, spec.N, spec.group
    rng = np.random.default_rng(5)
    q_dev = torch.randint(-2 ** 31, 2 ** 31 - 1, (K, N // 8), dtype=torch.int32, device="cuda")
    steps = torch.from_numpy((rng.random((K // g, N)) * 0.01 + 1e-4).astype(np.float16)).cuda()
    zeros = torch.from_numpy(rng.integers(0, 16, size=(K // g, N)).astype(np.float16)).cuda()
    A16 = (rng.standard_normal((M, K))).astype(np.float16)
    Y = awq.w4a16_matmul(torch.from_numpy(A16).cuda(), q_dev, steps, zeros, g).cpu().numpy()
    codes = q_dev.cpu().numpy()
    st, zr = steps.cpu().numpy(), zeros.cpu().numpy()
    for c0, c1 in [(0, 64), (N // 2 - 32, N // 2 + 32), (N - 72, N)]:
        _check_output(Y[:, c0:c1], A16, codes[:, c0 // 8:c1 // 8], st[:, c0:c1], zr[:, c0:c1], g)


@pytest.mark.parametrize("M", [1, 5, 9, 16])
@pytest.mark.parametrize("K,N,group", [(256, 256, 128), (160, 128, 32), (384, 576, 64), (128, 1024, 128)])
def test_repacked_decode_matches_oracle(M, K, N, group):
    codes, steps, zeros = _random_artifact(K, N, group, 7 * M + N)
    c, st, zr = _dev(codes, steps, zeros)
    packed = awq.w4a16_repack(c)
    A = (np.random.default_rng(M + 1).standard_normal((M, K)) * 2).astype(np.float16)
    Y = awq.w4a16_matmul_packed(torch.from_numpy(A).cuda(), packed, st, zr, group).cpu().numpy()
    _check_output(Y, A, codes, steps, zeros, group)


def test_repacked_decode_full_size_70b_columns():
    spec = WORKLOADS["llama70b_mlp_gate_up_16384x8192x57344"]
    K, N, g = spec.K, spec.N, spec.group
    rng = np.random.default_rng(9)
    q_dev = torch.randint(-2 ** 31, 2 ** 31 - 1, (K, N // 8), dtype=torch.int32, device="cuda")
    steps = torch.from_numpy((rng.random((K // g, N)) * 0.01 + 1e-4).astype(np.float16)).cuda()
    zeros = torch.from_numpy(rng.integers(0, 16, size=(K // g, N)).astype(np.float16)).cuda()
    A16 = rng.standard_normal((3, K)).astype(np.float16)
    Y = awq.w4a16_matmul_packed(torch.from_numpy(A16).cuda(), awq.w4a16_repack(q_dev), steps, zeros, g).cpu().numpy()
    codes, st, zr = q_dev.cpu().numpy(), steps.cpu().numpy(), zeros.cpu().numpy()
    for c0, c1 in [(0, 64), (N // 2 - 64, N // 2 + 64), (N - 128, N)]:
        _check_output(Y[:, c0:c1], A16, codes[:, c0 // 8:c1 // 8], st[:, c0:c1], zr[:, c0:c1], g)
