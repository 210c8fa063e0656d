"""Seeded synthetic calibration layers for the AWQ scale search.

This module only draws random inputs: it holds none of the search's arithmetic, so
both the CUDA path (through its tests and ``bench.py``) and the CPU oracle may take
their inputs from here.

Recipe (the five layer shapes of the workloads, all seeded):

* activations ``X`` (M x K): per-channel magnitude ``c_j = exp(sigma * N(0,1))``
  (log-normal(0, sigma)); ``round(0.01 * K)`` outlier channels, picked by a seeded
  permutation, are multiplied by ``outlier_mult``; ``X[m, j] = z[m, j] * c_j`` with
  ``z ~ N(0,1)`` ("normal" law) or ``|N(0,1)|`` ("abs_normal" law, the non-negative
  heavy-tailed input of an MLP down projection);
* weights ``W`` (K x N, the paper orientation: K input channels, N output channels):
  ``N(0, w_std)``;
* bf16 layers round both tensors to bf16 (round-to-nearest-even, done by torch);
  fp32 layers keep them in fp32.

Random numbers come from numpy's counter-based Philox generator, one independent
substream per tensor (``SeedSequence.spawn``), so a layer is a pure function of its
parameters and seed.
"""
from __future__ import annotations

from dataclasses import dataclass, asdict

import numpy as np
import torch


@dataclass(frozen=True)
class LayerSpec:
    name: str
    M: int
    K: int
    N: int
    dtype: str          # "bf16" or "f32": storage type of X and W
    law: str            # "normal" or "abs_normal"
    sigma: float        # log-normal sigma of the per-channel magnitude
    outlier_mult: float
    w_std: float
    group: int = 128
    n_grid: int = 20
    seed: int = 0

    def as_dict(self) -> dict:
        return asdict(self)

    @property
    def candidate_flops(self) -> float:
        """2*M*K*N per candidate GEMM, times the grid size."""
        return 2.0 * self.M * self.K * self.N * self.n_grid


# The five workloads: a small single linear layer and four Llama-shaped layers.
WORKLOADS = {
    "single_linear_128x256x256_f32": LayerSpec(
        "single_linear_128x256x256_f32", 128, 256, 256, "f32", "normal", 0.5, 20.0, 0.02),
    "llama7b_attn_proj_4096x4096x4096": LayerSpec(
        "llama7b_attn_proj_4096x4096x4096", 4096, 4096, 4096, "bf16", "normal", 0.5, 20.0, 0.02),
    "llama7b_mlp_gate_up_4096x4096x22016": LayerSpec(
        "llama7b_mlp_gate_up_4096x4096x22016", 4096, 4096, 22016, "bf16", "normal", 0.5, 20.0, 0.02),
    "llama7b_mlp_down_4096x11008x4096": LayerSpec(
        "llama7b_mlp_down_4096x11008x4096", 4096, 11008, 4096, "bf16", "abs_normal", 1.0, 50.0, 0.015),
    "llama70b_mlp_gate_up_16384x8192x57344": LayerSpec(
        "llama70b_mlp_gate_up_16384x8192x57344", 16384, 8192, 57344, "bf16", "normal", 0.5, 20.0, 0.01),
}
WORKLOAD_ORDER = list(WORKLOADS)


def custom_spec(M: int, K: int, N: int, *, dtype: str = "bf16", law: str = "normal",
                sigma: float = 0.5, outlier_mult: float = 20.0, w_std: float = 0.02,
                group: int = 128, n_grid: int = 20, seed: int = 0) -> LayerSpec:
    name = f"custom_{M}x{K}x{N}_{dtype}_{law}_g{group}_s{seed}"
    return LayerSpec(name, M, K, N, dtype, law, sigma, outlier_mult, w_std, group, n_grid, seed)


def _streams(seed: int, n: int):
    return [np.random.Generator(np.random.Philox(s)) for s in np.random.SeedSequence(seed).spawn(n)]


def generate(spec: LayerSpec) -> tuple[torch.Tensor, torch.Tensor]:
    """Return host tensors ``(X, W)`` of shapes (M, K) and (K, N), dtype bf16 or fp32."""
    g_mag, g_out, g_x, g_w = _streams(spec.seed, 4)
    K = spec.K
    mag = np.exp(spec.sigma * g_mag.standard_normal(K)).astype(np.float32)
    n_out = int(round(0.01 * K))
    outliers = g_out.permutation(K)[:n_out]
    mag[outliers] *= np.float32(spec.outlier_mult)

    z = g_x.standard_normal((spec.M, K), dtype=np.float32)
    if spec.law == "abs_normal":
        np.abs(z, out=z)
    elif spec.law != "normal":
        raise ValueError(f"unknown activation law {spec.law!r}")
    z *= mag[None, :]
    w = g_w.standard_normal((K, spec.N), dtype=np.float32)
    w *= np.float32(spec.w_std)

    X = torch.from_numpy(z)
    W = torch.from_numpy(w)
    if spec.dtype == "bf16":
        X = X.to(torch.bfloat16)
        W = W.to(torch.bfloat16)
    elif spec.dtype != "f32":
        raise ValueError(f"unknown storage dtype {spec.dtype!r}")
    return X, W


def outlier_channels(spec: LayerSpec) -> np.ndarray:
    """The outlier channel indices `generate` used (for tests of the recipe)."""
    _, g_out, _, _ = _streams(spec.seed, 4)
    return np.sort(g_out.permutation(spec.K)[: int(round(0.01 * spec.K))])


def as_f32_numpy(t: torch.Tensor) -> np.ndarray:
    """Exact float32 view of a bf16/fp32 host tensor, for the CPU side."""
    return t.detach().to("cpu").float().contiguous().numpy()


def generate_down(spec: LayerSpec, K_out: int, w_std: float = 0.015) -> torch.Tensor:
    """The down projection (F x K_out, F = N / 2) of an MLP block whose [gate | up] weights
    are `generate(spec)`'s W; its own Philox substream (the fifth of the layer's seed), so X
    and W are unchanged. Same storage dtype as the layer."""
    if spec.N % 2:
        raise ValueError("the [gate | up] layer has an even number of columns")
    g = _streams(spec.seed, 5)[4]
    w = g.standard_normal((spec.N // 2, K_out), dtype=np.float32)
    w *= np.float32(w_std)
    t = torch.from_numpy(w)
    return t.to(torch.bfloat16) if spec.dtype == "bf16" else t


def generate_qkv(spec: LayerSpec) -> torch.Tensor:
    """[W_q | W_k | W_v] (K x 3K) of an attention block whose query projection is
    `generate(spec)`'s W (K x K): the key and value projections are drawn from their own
    Philox substreams (the sixth and seventh of the layer's seed), N(0, w_std), so X and
    W_q are unchanged. Same storage dtype as the layer."""
    if spec.N != spec.K:
        raise ValueError("the query projection of an attention block is square (K x K)")
    _, W_q = generate(spec)
    streams = _streams(spec.seed, 7)
    parts = [W_q.float()]
    for g in streams[5:7]:
        w = g.standard_normal((spec.K, spec.K), dtype=np.float32)
        w *= np.float32(spec.w_std)
        parts.append(torch.from_numpy(w))
    W = torch.cat(parts, dim=1).contiguous()
    return W.to(torch.bfloat16) if spec.dtype == "bf16" else W
