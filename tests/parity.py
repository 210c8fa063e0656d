"""Comparison of the CUDA search with the CPU oracle (test-side helpers).

Tolerances (from the search's contract): the chosen alpha is identical unless the
oracle's two best losses lie within 1e-4 relative of each other; given the chosen
alpha, scales, codes, steps and zeros are bit-exact; every candidate loss agrees
within 1e-3 relative (the GPU accumulates in fp32, the oracle in fp64).
"""
from __future__ import annotations

import numpy as np
import torch

import oracle as O
import post_quantization_column_b200 as awq
from workloads import as_f32_numpy

LOSS_RTOL = 1e-3
ALPHA_TIE_RTOL = 1e-4


def run_gpu(X: torch.Tensor, W: torch.Tensor, group: int, n_grid: int, tiles: bool = True):
    out = awq.search(X.cuda(), W.cuda(), group=group, n_grid=n_grid, tile_sq_err=tiles)
    torch.cuda.synchronize()
    return {
        "scales": out.scales.cpu().numpy(),
        "codes": out.codes.cpu().numpy(),
        "steps": out.steps.cpu().numpy(),
        "zeros": out.zeros.cpu().numpy(),
        "losses": out.losses.cpu().numpy().astype(np.float64),
        "best": out.best,
        "tiles": out.tile_sq_err.cpu().numpy() if tiles else None,
    }


def check_alpha(gpu_best: int, orc_losses: np.ndarray):
    orc_best = O.first_argmin(list(orc_losses))
    if gpu_best == orc_best:
        return
    lo = orc_losses[orc_best]
    assert (orc_losses[gpu_best] - lo) <= ALPHA_TIE_RTOL * lo, (
        f"GPU chose alpha index {gpu_best}, oracle {orc_best}; oracle losses "
        f"{orc_losses[gpu_best]!r} vs {lo!r} are not within {ALPHA_TIE_RTOL} relative")


def check_losses(gpu_losses: np.ndarray, orc_losses: np.ndarray):
    err = np.abs(gpu_losses - orc_losses)
    bound = LOSS_RTOL * np.abs(orc_losses) + 1e-30
    bad = np.nonzero(err > bound)[0]
    assert bad.size == 0, f"losses differ at {bad.tolist()}: gpu {gpu_losses[bad]} oracle {orc_losses[bad]}"


def oracle_artifact(W32: np.ndarray, s: np.ndarray, group: int, cols: slice | None = None):
    """Codes (packed), fp16 steps and fp16 zeros of the oracle's QDQ for scales s."""
    Wc = W32 if cols is None else W32[:, cols]
    q, step, zero, _ = O.asym_qdq(O.scale_weights(Wc, s), group)
    return O.pack_codes(q), O.fp16_rne(step), zero.astype(np.float16)


def check_artifact(gpu: dict, W32: np.ndarray, S_orc: np.ndarray, group: int, col_chunk: int = 8192):
    b = gpu["best"]
    s = S_orc[b]
    assert np.array_equal(gpu["scales"].view(np.uint32), s.view(np.uint32)), "scales differ"
    N = W32.shape[1]
    for c0 in range(0, N, col_chunk):
        c1 = min(N, c0 + col_chunk)
        codes, steps, zeros = oracle_artifact(W32, s, group, slice(c0, c1))
        g_codes = gpu["codes"][:, c0 // 8: c1 // 8]
        if not np.array_equal(g_codes, codes):
            bad = np.argwhere(g_codes != codes)
            raise AssertionError(f"codes differ at {len(bad)} words, first {bad[:5].tolist()}")
        assert np.array_equal(gpu["steps"][:, c0:c1].view(np.uint16), steps.view(np.uint16)), "steps differ"
        assert np.array_equal(gpu["zeros"][:, c0:c1].view(np.uint16), zeros.view(np.uint16)), "zeros differ"


def oracle_tile_sq_err(X32, W32, S_orc, group, c, mt, nt, tm=128, tn=256):
    """Oracle sum of (X_b W_hat_c,b - X_b W_b)^2 over one output tile."""
    M, N = X32.shape[0], W32.shape[1]
    rows = slice(mt * tm, min(M, (mt + 1) * tm))
    cols = slice(nt * tn, min(N, (nt + 1) * tn))
    Xb = O.bf16_rne(X32[rows]).astype(np.float64)
    Wc = W32[:, cols]
    Wb = O.bf16_rne(Wc).astype(np.float64)
    What = O.bf16_rne(O.candidate_what(Wc, S_orc[c], group)).astype(np.float64)
    return O.block_squared_error(Xb, Wb, What)


def check_tiles(gpu: dict, X32, W32, S_orc, group, samples):
    tiles = gpu["tiles"]
    M, N = X32.shape[0], W32.shape[1]
    # property at any size: the loss is the fixed-order sum of the tile partials / (M N)
    sums = tiles.reshape(tiles.shape[0], -1).sum(axis=1) / (M * N)
    assert np.allclose(sums, gpu["losses"], rtol=1e-6, atol=0), "losses are not the sum of the tile partials"
    for (c, mt, nt) in samples:
        ref = oracle_tile_sq_err(X32, W32, S_orc, group, c, mt, nt)
        got = tiles[c, mt, nt]
        assert abs(got - ref) <= LOSS_RTOL * abs(ref) + 1e-30, f"tile ({c},{mt},{nt}): gpu {got} oracle {ref}"


def full_parity(X: torch.Tensor, W: torch.Tensor, group: int, n_grid: int):
    """Element-by-element comparison with the complete oracle (small layers)."""
    X32, W32 = as_f32_numpy(X), as_f32_numpy(W)
    gpu = run_gpu(X, W, group, n_grid, tiles=True)
    orc = O.search(X32, W32, group=group, n_grid=n_grid)
    # the index the library returned is the first minimum of the losses it returned
    # (AWQ-P1 §3), and follows the oracle's choice up to near-ties
    assert gpu["best"] == O.first_argmin(list(gpu["losses"])), "library index is not its losses' first minimum"
    check_alpha(gpu["best"], orc.losses)
    check_losses(gpu["losses"], orc.losses)
    check_artifact(gpu, W32, orc.S, group)
    tm, tn = 128, 256
    T = gpu["tiles"]
    samples = [(c, mt, nt) for c in range(n_grid) for mt in range(T.shape[1]) for nt in range(T.shape[2])]
    if len(samples) > 64:
        rng = np.random.default_rng(0)
        corners = [(c, T.shape[1] - 1, T.shape[2] - 1) for c in (0, n_grid - 1)]
        samples = corners + [samples[i] for i in rng.choice(len(samples), 62, replace=False)]
    check_tiles(gpu, X32, W32, orc.S, group, samples)
    return gpu, orc
