"""The MLP-block objective on the GPU against the oracle (B200 only).

Page: "AWQ：为什么 4-bit 权重量化要先观察 Activation" §4 (a candidate scored on the output of
the whole module). Both sides round the block's intermediate h to bf16; the GPU rounds it
from fp32 GEMM sums, the oracle from exact ones, so an h value lying next to a bf16
rounding boundary can round differently. That perturbs every loss a little, and the
losses are held to LOSS_RTOL; the chosen alpha is the oracle's unless the oracle's two best
losses lie within ALPHA_TIE_RTOL; given alpha the scales, codes, steps and zeros are
bit-exact.
"""
import numpy as np
import pytest
import torch

import oracle as O
import oracle.awq_module as MOD
import post_quantization_column_b200 as awq
from workloads import custom_spec, generate, generate_down, as_f32_numpy

pytestmark = pytest.mark.gpu

LOSS_RTOL = 1e-3
ALPHA_TIE_RTOL = 1e-3


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def _run(M, K, F, Ko, group, dtype, seed, n_grid=20):
    spec = custom_spec(M, K, 2 * F, dtype=dtype, group=group, seed=seed)
    X, W_gu = generate(spec)
    W_down = generate_down(spec, Ko)
    out = awq.search_mlp(X.cuda(), W_gu.cuda(), W_down.cuda(), group, n_grid)
    X32, Wgu32, Wd32 = as_f32_numpy(X), as_f32_numpy(W_gu), as_f32_numpy(W_down)
    r = MOD.mlp_search(X32, Wgu32, Wd32, group, n_grid)
    return out, r, Wgu32


def _check(out, r, Wgu32, group):
    gl = out.losses.cpu().numpy().astype(np.float64)
    rel = np.abs(gl - r.losses) / np.abs(r.losses)
    print(f"max relative loss difference {rel.max():.2e}")
    assert np.all(rel <= LOSS_RTOL), f"losses differ: {rel.max():.2e}"
    b, ob = out.best, r.best
    if b != ob:
        assert r.losses[b] - r.losses[ob] <= ALPHA_TIE_RTOL * r.losses[ob], (b, ob, r.losses[[b, ob]])
    s = r.S[b]
    assert np.array_equal(out.scales.cpu().numpy().view(np.uint32), s.view(np.uint32))
    q, step, zero, _ = O.asym_qdq(O.scale_weights(Wgu32, s), group)
    assert np.array_equal(out.codes.cpu().numpy(), O.pack_codes(q))
    assert np.array_equal(out.steps.cpu().numpy().view(np.uint16), O.fp16_rne(step).view(np.uint16))
    assert np.array_equal(out.zeros.cpu().numpy().view(np.uint16), zero.astype(np.float16).view(np.uint16))
    return rel.max()


@pytest.mark.parametrize("M,K,F,Ko,group,dtype", [
    (128, 256, 128, 256, 128, "f32"),
    (300, 384, 136, 264, 128, "bf16"),   # ragged rows, ragged block-output columns
    (64, 160, 64, 72, 32, "bf16"),
    (200, 320, 96, 128, 64, "f32"),
])
def test_mlp_block_search_matches_oracle(M, K, F, Ko, group, dtype):
    out, r, Wgu32 = _run(M, K, F, Ko, group, dtype, seed=M + K + F)
    _check(out, r, Wgu32, group)


def test_mlp_block_full_width_7b_shape():
    """The 7B MLP block's widths (K 4096, F 11008, K_out 4096) with 64 calibration tokens,
    so that the complete oracle stays within a minute on the host."""
    out, r, Wgu32 = _run(64, 4096, 11008, 4096, 128, "bf16", seed=3)
    _check(out, r, Wgu32, 128)


def test_mlp_block_is_deterministic():
    spec = custom_spec(130, 256, 2 * 64, dtype="bf16", seed=11)
    X, W_gu = (t.cuda() for t in generate(spec))
    W_down = generate_down(spec, 136).cuda()
    a, b = awq.search_mlp(X, W_gu, W_down, 128, 20), awq.search_mlp(X, W_gu, W_down, 128, 20)
    for name in ("scales", "codes", "steps", "zeros", "losses"):
        assert torch.equal(getattr(a, name), getattr(b, name)), name


def test_fused_epilogue_matches_separate_elementwise_kernel(monkeypatch):
    """F % 128 == 0 runs the silu-mul in the first GEMM's epilogue (gate and up columns
    interleaved by 128 in the candidate operand); the separate elementwise kernel must give
    the same bits, losses included."""
    spec = custom_spec(200, 256, 2 * 256, dtype="bf16", seed=5)
    X, W_gu = (t.cuda() for t in generate(spec))
    W_down = generate_down(spec, 264).cuda()
    fused = awq.search_mlp(X, W_gu, W_down, 128, 20)
    monkeypatch.setenv("AWQ_MLP_UNFUSED", "1")
    plain = awq.search_mlp(X, W_gu, W_down, 128, 20)
    for name in ("scales", "codes", "steps", "zeros", "losses"):
        assert torch.equal(getattr(fused, name), getattr(plain, name)), name


@pytest.mark.parametrize("M,K,F,Ko,n_grid", [(300, 384, 256, 264, 20), (129, 256, 384, 136, 7), (64, 512, 128, 64, 64)])
def test_qdq_warps_match_the_qdq_kernel_in_the_mlp_block(M, K, F, Ko, n_grid, monkeypatch):
    """bf16 W with group 128 and F % 128 == 0: the first GEMM's QDQ warps make the candidate
    operands of [W_gate | W_up] candidate by candidate (claimed while the reference block
    runs, the rest during the candidates' first GEMM, each candidate's loads waiting for its
    slot); AWQ_QDQ=standalone makes them with qdq_kernel first. Both match the oracle and
    give the same bits."""
    out, r, Wgu32 = _run(M, K, F, Ko, 128, "bf16", seed=M + 2 * K + F, n_grid=n_grid)
    _check(out, r, Wgu32, 128)
    spec = custom_spec(M, K, 2 * F, dtype="bf16", group=128, seed=M + 2 * K + F)
    X, W_gu = (t.cuda() for t in generate(spec))
    W_down = generate_down(spec, Ko).cuda()
    warps = awq.search_mlp(X, W_gu, W_down, 128, n_grid)
    monkeypatch.setenv("AWQ_QDQ", "standalone")
    plain = awq.search_mlp(X, W_gu, W_down, 128, n_grid)
    for name in ("scales", "codes", "steps", "zeros", "losses"):
        assert torch.equal(getattr(warps, name), getattr(plain, name)), name
