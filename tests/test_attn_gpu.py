"""The attention-block objective on the GPU against the oracle (B200 only).

Page: "AWQ：为什么 4-bit 权重量化要先观察 Activation" §4 (a candidate scored on the output of
the module it belongs to; the module may be an attention block holding several
projections). Both sides round Q, K, V and the attention weights to bf16; the GPU rounds
them from fp32 tensor-core sums and a fp32 exp2, the oracle from exact values, so a value
lying next to a bf16 rounding boundary can round differently on the two sides. That
perturbs every loss a little: the losses are held to LOSS_RTOL, the chosen alpha is the
oracle's unless the oracle's two best losses lie within ALPHA_TIE_RTOL, and given alpha the
scales, codes, steps and zeros are bit-exact.
"""
import numpy as np
import pytest
import torch

import oracle as O
import oracle.awq_attn as ATT
import post_quantization_column_b200 as awq
from workloads import WORKLOADS, custom_spec, generate, generate_qkv, as_f32_numpy

pytestmark = pytest.mark.gpu

LOSS_RTOL = 1e-3
ALPHA_TIE_RTOL = 1e-3


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def _layer(M, K, D, dtype, group, seed):
    """X (M x K) of a seeded layer and its [W_q | W_k | W_v] restricted to D columns each
    (D <= K): columns 0 .. D-1 of each of the three K x K projections."""
    spec = custom_spec(M, K, K, dtype=dtype, group=group, seed=seed)
    X, _ = generate(spec)
    W = generate_qkv(spec)
    cols = torch.from_numpy(np.r_[0:D, K:K + D, 2 * K:2 * K + D])
    return X, W[:, cols].contiguous()


def _run(X, W, n_heads, seq_len, group, n_grid=20):
    out = awq.search_attn(X.cuda(), W.cuda(), n_heads, seq_len, group, n_grid)
    X32, W32 = as_f32_numpy(X), as_f32_numpy(W)
    r = ATT.attn_search(X32, W32, X.shape[0] // seq_len, n_heads, group, n_grid)
    return out, r, W32


def _check(out, r, W32, group):
    gl = out.losses.cpu().numpy().astype(np.float64)
    rel = np.abs(gl - r.losses) / np.abs(r.losses)
    print(f"max relative loss difference {rel.max():.2e}")
    assert np.all(rel <= LOSS_RTOL), f"losses differ: {rel.max():.2e} ({gl} vs {r.losses})"
    b, ob = out.best, r.best
    assert b == O.first_argmin(list(gl))
    if b != ob:
        assert r.losses[b] - r.losses[ob] <= ALPHA_TIE_RTOL * r.losses[ob], (b, ob, r.losses[[b, ob]])
    s = r.S[b]
    assert np.array_equal(out.scales.cpu().numpy().view(np.uint32), s.view(np.uint32))
    q, step, zero, _ = O.asym_qdq(O.scale_weights(W32, s), group)
    assert np.array_equal(out.codes.cpu().numpy(), O.pack_codes(q))
    assert np.array_equal(out.steps.cpu().numpy().view(np.uint16), O.fp16_rne(step).view(np.uint16))
    assert np.array_equal(out.zeros.cpu().numpy().view(np.uint16), zero.astype(np.float16).view(np.uint16))
    return rel.max()


@pytest.mark.parametrize("M,K,n_heads,seq_len,group,dtype", [
    (256, 256, 1, 128, 128, "bf16"),    # two sequences of one query block each
    (512, 384, 2, 256, 64, "f32"),      # fp32 inputs, two query blocks per sequence
    (384, 160, 1, 384, 32, "bf16"),     # three query blocks (odd), ragged K blocks
    (1024, 256, 2, 512, 128, "bf16"),   # the longest sequences: all 512 tensor-memory columns
])
def test_attention_block_search_matches_oracle(M, K, n_heads, seq_len, group, dtype):
    X, W = _layer(M, K, n_heads * awq.ATTN_HEAD_DIM, dtype, group, seed=M + K + n_heads)
    out, r, W32 = _run(X, W, n_heads, seq_len, group)
    _check(out, r, W32, group)


def test_attention_block_7b_shape():
    """The Llama-7B attention block: 8 sequences x 512 tokens, K 4096, 32 heads of 128
    (W_q is the 4096^3 layer's W), against the complete oracle."""
    spec = WORKLOADS["llama7b_attn_proj_4096x4096x4096"]
    X, _ = generate(spec)
    out, r, W32 = _run(X, generate_qkv(spec), 32, 512, spec.group)
    _check(out, r, W32, spec.group)


def test_attention_block_is_deterministic():
    X, W = _layer(512, 256, 128, "bf16", 128, seed=12)
    Xd, Wd = X.cuda(), W.cuda()
    a, b = awq.search_attn(Xd, Wd, 1, 256), awq.search_attn(Xd, Wd, 1, 256)
    for name in ("scales", "codes", "steps", "zeros", "losses", "best_index"):
        assert torch.equal(getattr(a, name), getattr(b, name)), name


def test_attention_block_rejects_bad_shapes():
    X = torch.zeros(256, 128, dtype=torch.bfloat16, device="cuda")
    W = torch.zeros(128, 3 * 128, dtype=torch.bfloat16, device="cuda")
    for heads, seq in ((2, 128), (1, 64), (1, 1024), (1, 96)):
        with pytest.raises(awq.AwqError) as e:
            awq.search_attn(X, W, heads, seq)
        assert e.value.status == 2   # AWQ_ERR_SHAPE
    Xn = X.clone()
    Xn[3, 4] = float("nan")
    with pytest.raises(awq.AwqError) as e:
        awq.search_attn(Xn, W, 1, 128)
    assert e.value.status == 3       # AWQ_ERR_NONFINITE


def test_attention_wait_that_runs_out_returns_timeout():
    """The attention kernel's producer skips a key tile: the MMA thread's bounded wait runs
    out, the call returns AWQ_ERR_TIMEOUT, and the next call is exact again."""
    X, W = _layer(256, 256, 128, "bf16", 128, seed=13)
    Xd, Wd = X.cuda(), W.cuda()
    ref = awq.search_attn(Xd, Wd, 1, 128)
    awq.debug_set_fault(1, 50_000_000)
    try:
        with pytest.raises(awq.AwqError) as err:
            awq.search_attn(Xd, Wd, 1, 128)
        assert err.value.status == 6
    finally:
        awq.debug_set_fault(0)
    again = awq.search_attn(Xd, Wd, 1, 128)
    for name in ("scales", "codes", "steps", "zeros", "losses"):
        assert torch.equal(getattr(again, name), getattr(ref, name)), name


@pytest.mark.parametrize("M,K,n_heads,seq_len,n_grid", [(256, 256, 1, 128, 20), (1024, 384, 2, 512, 7),
                                                         (512, 512, 2, 256, 64)])
def test_qdq_warps_match_the_qdq_kernel_in_the_attention_block(M, K, n_heads, seq_len, n_grid, monkeypatch):
    """bf16 W with group 128: the Q|K GEMM's QDQ warps make the candidate operands of
    [W_q | W_k] (its loads of a slot's tile waiting for that tile) and then of W_v (read by
    the next launch); AWQ_QDQ=standalone makes them with qdq_kernel first. Both give the
    same bits, and the warps' form matches the oracle."""
    X, W = _layer(M, K, n_heads * awq.ATTN_HEAD_DIM, "bf16", 128, seed=M + 3 * K)
    monkeypatch.delenv("AWQ_QDQ", raising=False)
    out, r, W32 = _run(X, W, n_heads, seq_len, 128, n_grid)
    _check(out, r, W32, 128)
    monkeypatch.setenv("AWQ_QDQ", "standalone")
    plain = awq.search_attn(X.cuda(), W.cuda(), n_heads, seq_len, 128, n_grid)
    for name in ("scales", "codes", "steps", "zeros", "losses", "best_index"):
        assert torch.equal(getattr(out, name), getattr(plain, name)), name
