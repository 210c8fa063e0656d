"""Clipping search on the GPU against the oracle (B200 only).

Page: "AWQ：为什么 4-bit 权重量化要先观察 Activation", §5 (clipping after the scaling).

Both sides compute every candidate's error in fp64 from the same fp32 operands; they
differ only in summation order (the oracle forms the partial outputs X'_g delta and
squares them, the kernels form delta^T (X'_g^T X'_g) delta), so the errors agree to
ERR_RTOL relative to the column's largest error. The chosen shrink factor is the
oracle's unless the oracle's two best errors lie within TIE_RTOL of each other; given
the chosen factor, the threshold, codes, steps and zeros are bit-exact.
"""
import numpy as np
import pytest
import torch

import oracle as O
import oracle.awq_clip as C
import post_quantization_column_b200 as awq
from workloads import WORKLOADS, custom_spec, generate, as_f32_numpy

pytestmark = pytest.mark.gpu

ERR_RTOL = 1e-9
TIE_RTOL = 1e-9


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def run_clip(X, W, s, group, n_shrink=10, max_tokens=512):
    out = awq.clip_search(X.cuda(), W.cuda(), torch.as_tensor(s).cuda(), group, n_shrink, max_tokens, errors=True)
    torch.cuda.synchronize()
    return {k: getattr(out, k).cpu().numpy() for k in ("max_val", "best", "codes", "steps", "zeros", "errors")}


def check_clip(gpu, X32, W32, s, group, n_shrink=10, max_tokens=512):
    """Compare the GPU result with the oracle, column for column."""
    N = W32.shape[1]
    for c0, c1 in [(0, N)]:
        r = C.clip_search(X32, W32[:, c0:c1], s, group, n_shrink, max_tokens=max_tokens)
        ge = gpu["errors"][:, :, c0:c1]
        scale = np.max(np.abs(r.errors), axis=0, keepdims=True)
        bad = np.argwhere(np.abs(ge - r.errors) > ERR_RTOL * scale)
        assert bad.size == 0, (f"{len(bad)} errors differ, first (i, g, n) {bad[:4].tolist()}: "
                               f"gpu {ge[tuple(bad[0])]!r} oracle {r.errors[tuple(bad[0])]!r}")
        gb = gpu["best"][:, c0:c1]
        for g, n in np.argwhere(gb != r.best):
            e = r.errors[:, g, n]
            lo = e[r.best[g, n]]
            assert e[gb[g, n]] - lo <= TIE_RTOL * abs(lo), (
                f"(g={g}, n={c0 + n}): GPU chose {gb[g, n]}, oracle {r.best[g, n]}, errors {e.tolist()}")
        chosen = np.take_along_axis(r.thresholds, gb[None].astype(np.int64), axis=0)[0]
        mv = gpu["max_val"][:, c0:c1]
        assert np.array_equal(mv.view(np.uint32), chosen.view(np.uint32)), "thresholds differ"
        codes, steps, zeros = C.clipped_artifact(W32[:, c0:c1], s, group, mv)
        g_codes = gpu["codes"][:, c0 // 8:c1 // 8]
        if not np.array_equal(g_codes, codes):
            badw = np.argwhere(g_codes != codes)
            raise AssertionError(f"codes differ at {len(badw)} words, first {badw[:4].tolist()}")
        assert np.array_equal(gpu["steps"][:, c0:c1].view(np.uint16), steps.view(np.uint16)), "steps differ"
        assert np.array_equal(gpu["zeros"][:, c0:c1].view(np.uint16), zeros.view(np.uint16)), "zeros differ"


def _scales(X32, alpha_index=10, n_grid=20):
    return O.candidate_scales(O.activation_statistic(X32), n_grid)[alpha_index]


@pytest.mark.parametrize("M,K,N,group,dtype", [
    (128, 256, 256, 128, "f32"),     # the single-layer case
    (300, 384, 520, 128, "bf16"),    # ragged: 520 columns = 8 CTAs of 64 + 8
    (1500, 192, 136, 64, "bf16"),    # M > 512: every 2nd row, first 512 of them
    (40, 96, 72, 32, "f32"),
    (1, 128, 64, 128, "bf16"),       # one token
])
def test_clip_matches_oracle_small(M, K, N, group, dtype):
    spec = custom_spec(M, K, N, dtype=dtype, group=group, seed=M + K + N)
    X, W = generate(spec)
    X32, W32 = as_f32_numpy(X), as_f32_numpy(W)
    s = _scales(X32)
    check_clip(run_clip(X, W, s, group), X32, W32, s, group)


@pytest.mark.parametrize("n_shrink,max_tokens", [(1, 512), (4, 512), (20, 512), (10, 37)])
def test_clip_grid_and_token_options(n_shrink, max_tokens):
    spec = custom_spec(700, 256, 200, dtype="bf16", seed=5)
    X, W = generate(spec)
    X32, W32 = as_f32_numpy(X), as_f32_numpy(W)
    s = _scales(X32, 7)
    check_clip(run_clip(X, W, s, 128, n_shrink, max_tokens), X32, W32, s, 128, n_shrink, max_tokens)


def test_clip_after_the_gpu_search_end_to_end():
    spec = custom_spec(512, 512, 264, dtype="bf16", seed=9)
    X, W = generate(spec)
    X32, W32 = as_f32_numpy(X), as_f32_numpy(W)
    out = awq.search(X.cuda(), W.cuda(), 128, 20)
    s = out.scales.cpu().numpy()
    assert np.array_equal(s.view(np.uint32), _scales(X32, out.best).view(np.uint32))
    check_clip(run_clip(X, W, s, 128), X32, W32, s, 128)


def test_single_factor_reproduces_the_search_artifact():
    # with the one factor 1 there is no clipping: the artifact is the search's own
    spec = custom_spec(256, 384, 136, dtype="bf16", seed=11)
    X, W = generate(spec)
    out = awq.search(X.cuda(), W.cuda(), 128, 20)
    gpu = run_clip(X, W, out.scales.cpu().numpy(), 128, n_shrink=1)
    assert np.all(gpu["best"] == 0)
    assert np.array_equal(gpu["codes"], out.codes.cpu().numpy())
    assert np.array_equal(gpu["steps"].view(np.uint16), out.steps.cpu().numpy().view(np.uint16))
    assert np.array_equal(gpu["zeros"].view(np.uint16), out.zeros.cpu().numpy().view(np.uint16))


def test_clip_edge_cases():
    rng = np.random.default_rng(3)
    M, K, N, group = 64, 256, 72, 128
    X32 = rng.standard_normal((M, K)).astype(np.float32)
    X32[:, :group] = 0.0                                   # a silent group: every error 0, factor 1 kept
    W32 = (rng.standard_normal((K, N)) * 0.02).astype(np.float32)
    W32[:, 0] = 0.0                                        # an all-zero column
    W32[:, 1] = 0.03125                                    # constant columns
    W32[:, 2] = -0.5
    W32[5, 3] = 1.0                                        # one outlier weight
    W32[200, 4] = -2.0
    s = np.exp(0.3 * rng.standard_normal(K)).astype(np.float32)
    gpu = run_clip(torch.from_numpy(X32), torch.from_numpy(W32), s, group)
    check_clip(gpu, X32, W32, s, group)
    assert np.all(gpu["errors"][:, 0] == 0.0) and np.all(gpu["best"][0] == 0)


def test_clip_is_deterministic():
    spec = custom_spec(600, 512, 328, dtype="bf16", seed=13)
    X, W = generate(spec)
    s = _scales(as_f32_numpy(X))
    a, b = run_clip(X, W, s, 128), run_clip(X, W, s, 128)
    for k in a:
        assert np.array_equal(a[k], b[k]), k


def test_clip_rejects_bad_scales_and_non_finite_weights():
    spec = custom_spec(64, 256, 64, dtype="bf16", seed=1)
    X, W = (t.cuda() for t in generate(spec))
    for bad in (0.0, -1.0, float("nan"), float("inf")):
        s = torch.ones(256, dtype=torch.float32, device="cuda")
        s[17] = bad
        with pytest.raises(awq.AwqError) as err:
            awq.clip_search(X, W, s)
        assert err.value.status == 1
    W2 = W.clone()
    W2[3, 5] = float("nan")
    with pytest.raises(awq.AwqError) as err:
        awq.clip_search(X, W2, torch.ones(256, dtype=torch.float32, device="cuda"))
    assert err.value.status == 3
    # the context stays usable
    awq.clip_search(X, W, torch.ones(256, dtype=torch.float32, device="cuda"))


@pytest.mark.parametrize("name", [n for n in WORKLOADS if n != "single_linear_128x256x256_f32"])
def test_clip_full_size_sampled_columns(name):
    """Whole layer on the GPU; the oracle recomputes sampled column blocks (each
    (group, column) is independent given the sampled tokens and the scales)."""
    spec = WORKLOADS[name]
    X, W = generate(spec)
    X32 = as_f32_numpy(X)
    s = _scales(X32)
    gpu = run_clip(X, W, s, spec.group)
    N = spec.N
    for c0, c1 in [(0, 64), (N // 2 - 32, N // 2 + 32), (N - 72, N)]:
        sub = {"errors": gpu["errors"][:, :, c0:c1], "best": gpu["best"][:, c0:c1],
               "max_val": gpu["max_val"][:, c0:c1], "codes": gpu["codes"][:, c0 // 8:c1 // 8],
               "steps": gpu["steps"][:, c0:c1], "zeros": gpu["zeros"][:, c0:c1]}
        W32 = np.ascontiguousarray(W[:, c0:c1].float().numpy())
        check_clip(sub, X32, W32, s, spec.group)
