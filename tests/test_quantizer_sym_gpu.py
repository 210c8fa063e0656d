"""The symmetric [-7, 7] teaching quantizer as the candidates' quantizer (B200 only).

Page: "AWQ：为什么 4-bit 权重量化要先观察 Activation" §2 (the teaching quantizer), §4 (the
search), §5 (clipping), §7 (the artifact). Same bar as the asymmetric search: the chosen
alpha is the oracle's unless its two best losses lie within 1e-4; given alpha the scales,
codes (q + 7), steps and zeros (7) are bit-exact; every loss within 1e-3.
"""
import numpy as np
import pytest
import torch

import oracle as O
import oracle.awq_clip as C
import post_quantization_column_b200 as awq
from tests.parity import check_alpha, check_losses
from workloads import custom_spec, generate, as_f32_numpy

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


@pytest.mark.parametrize("M,K,N,group,dtype", [
    (128, 256, 256, 128, "f32"), (300, 384, 520, 128, "bf16"), (64, 160, 264, 32, "bf16"), (96, 320, 136, 64, "f32"),
])
def test_symmetric_search_matches_oracle(M, K, N, group, dtype):
    spec = custom_spec(M, K, N, dtype=dtype, group=group, seed=M + N)
    X, W = generate(spec)
    out = awq.search(X.cuda(), W.cuda(), group, 20, quantizer="sym")
    X32, W32 = as_f32_numpy(X), as_f32_numpy(W)
    r = O.search(X32, W32, group=group, n_grid=20, quantizer="sym_teaching")
    losses = out.losses.cpu().numpy().astype(np.float64)
    check_losses(losses, r.losses)
    check_alpha(out.best, r.losses)
    s = r.S[out.best]
    assert np.array_equal(out.scales.cpu().numpy().view(np.uint32), s.view(np.uint32))
    q, step, zero = O.sym_artifact(O.scale_weights(W32, s), group)
    assert np.array_equal(out.codes.cpu().numpy(), O.pack_codes(q))
    assert np.array_equal(out.steps.cpu().numpy().view(np.uint16), O.fp16_rne(step).view(np.uint16))
    assert np.array_equal(out.zeros.cpu().numpy().view(np.uint16), zero.astype(np.float16).view(np.uint16))


def test_symmetric_clipping_matches_oracle():
    spec = custom_spec(300, 256, 136, dtype="bf16", seed=23)
    X, W = generate(spec)
    X32, W32 = as_f32_numpy(X), as_f32_numpy(W)
    s = O.candidate_scales(O.activation_statistic(X32), 20)[9]
    out = awq.clip_search(X.cuda(), W.cuda(), torch.from_numpy(s).cuda(), 128, 10, errors=True, quantizer="sym")
    gpu = {k: getattr(out, k).cpu().numpy() for k in ("max_val", "best", "codes", "steps", "zeros", "errors")}
    r = C.clip_search(X32, W32, s, 128, 10, quantizer="sym_teaching")
    scale = np.max(np.abs(r.errors), axis=0, keepdims=True)
    assert np.all(np.abs(gpu["errors"] - r.errors) <= 1e-9 * scale)
    for g, n in np.argwhere(gpu["best"] != r.best):
        e = r.errors[:, g, n]
        assert e[gpu["best"][g, n]] - e[r.best[g, n]] <= 1e-9 * abs(e[r.best[g, n]])
    codes, steps, zeros = C.clipped_artifact(W32, s, 128, gpu["max_val"], quantizer="sym")
    assert np.array_equal(gpu["codes"], codes)
    assert np.array_equal(gpu["steps"].view(np.uint16), steps.view(np.uint16))
    assert np.array_equal(gpu["zeros"].view(np.uint16), zeros.view(np.uint16))


def test_symmetric_artifact_is_consumed_by_the_w4a16_kernel():
    import oracle.awq_w4a16 as Q
    spec = custom_spec(256, 256, 72, dtype="bf16", seed=29)
    X, W = generate(spec)
    out = awq.search(X.cuda(), W.cuda(), 128, 20, quantizer="sym")
    A16 = Q.fp16_activations(as_f32_numpy(X), out.scales.cpu().numpy())
    for M in (1, 100):
        Y = awq.w4a16_matmul(torch.from_numpy(A16[:M]).cuda(), out.codes, out.steps, out.zeros, 128).cpu().numpy()
        ref = Q.w4a16_matmul(A16[:M], out.codes.cpu().numpy(), out.steps.cpu().numpy(), out.zeros.cpu().numpy(), 128)
        Wd = Q.dequant_operand(out.codes.cpu().numpy(), out.steps.cpu().numpy(), out.zeros.cpu().numpy(), 128, 72)
        bound = 2e-5 * (np.abs(A16[:M].astype(np.float64)) @ np.abs(Wd.astype(np.float64)))
        assert np.all(np.abs(Y - ref) <= bound + 1e-30)
