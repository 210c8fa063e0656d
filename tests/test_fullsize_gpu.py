"""The four Llama-shaped workloads at full size, in the launch configuration bench.py
times (B200 only).

The complete oracle would need 21 fp64 GEMMs of up to 16384 x 8192 x 57344, so at
these sizes the comparison is:
* the chosen scales, codes, steps and zeros bit-exact against the oracle's statistic,
  scale family and QDQ at the GPU's alpha, over every column (O(MK + KN) on the CPU);
* every loss equals the fixed-order sum of the per-tile partial sums / (M N) — a
  property of the reduction at any size;
* sampled output tiles (first, last, random; three candidates including the chosen
  one), each recomputed by the oracle from its own bf16 operands in fp64, within the
  1e-3 relative loss tolerance;
* where AWQ_FULL_ORACLE_TFLOP allows (an fp64 budget on the host, default 20 TFLOP:
  every layer but the 70B one), the complete oracle loss vector and the alpha rule.
"""
import os

import numpy as np
import pytest
import torch

import oracle as O
from tests import parity as P
from workloads import WORKLOADS, generate, as_f32_numpy

pytestmark = pytest.mark.gpu

FULL = ["llama7b_attn_proj_4096x4096x4096", "llama7b_mlp_gate_up_4096x4096x22016",
        "llama7b_mlp_down_4096x11008x4096", "llama70b_mlp_gate_up_16384x8192x57344"]


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


@pytest.mark.parametrize("name", FULL)
def test_full_size_workload(name):
    spec = WORKLOADS[name]
    X, W = generate(spec)
    gpu = P.run_gpu(X, W, spec.group, spec.n_grid, tiles=True)
    torch.cuda.empty_cache()
    X32, W32 = as_f32_numpy(X), as_f32_numpy(W)
    del X, W
    a = O.activation_statistic(X32)
    S = O.candidate_scales(a, spec.n_grid)
    P.check_artifact(gpu, W32, S, spec.group)

    T = gpu["tiles"]
    tm_n, tn_n = T.shape[1], T.shape[2]
    rng = np.random.default_rng(7)
    cands = sorted({0, gpu["best"], spec.n_grid - 1})
    samples = []
    for c in cands:
        samples += [(c, 0, 0), (c, tm_n - 1, tn_n - 1), (c, int(rng.integers(tm_n)), int(rng.integers(tn_n)))]
    P.check_tiles(gpu, X32, W32, S, spec.group, samples)

    budget = float(os.environ.get("AWQ_FULL_ORACLE_TFLOP", "20"))
    fp64_tflop = 2.0 * spec.M * spec.K * spec.N * (spec.n_grid + 1) / 1e12
    if fp64_tflop <= budget:
        orc = O.search(X32, W32, group=spec.group, n_grid=spec.n_grid)
        P.check_alpha(gpu["best"], orc.losses)
        P.check_losses(gpu["losses"], orc.losses)


def test_llama70b_column_slice_against_the_complete_oracle():
    """The 70B gate+up layer's full X (16384 x 8192, 64 groups) with 1024 columns from
    each half of W (the first of the gate half and of the up half): the layer the
    complete oracle can finish in about a minute on the host. Alpha rule, every loss,
    the artifact over every column and sampled tiles, as for the small layers."""
    spec = WORKLOADS["llama70b_mlp_gate_up_16384x8192x57344"]
    X, W = generate(spec)
    half = spec.N // 2
    Ws = torch.cat([W[:, :1024], W[:, half:half + 1024]], dim=1).contiguous()
    del W
    gpu = P.run_gpu(X, Ws, spec.group, spec.n_grid, tiles=True)
    torch.cuda.empty_cache()
    X32, W32 = as_f32_numpy(X), as_f32_numpy(Ws)
    del X, Ws
    orc = O.search(X32, W32, group=spec.group, n_grid=spec.n_grid)
    assert gpu["best"] == O.first_argmin(list(gpu["losses"]))
    P.check_alpha(gpu["best"], orc.losses)
    P.check_losses(gpu["losses"], orc.losses)
    P.check_artifact(gpu, W32, orc.S, spec.group)
    T = gpu["tiles"]
    samples = [(c, mt, nt) for c in sorted({0, gpu["best"], spec.n_grid - 1})
               for mt, nt in ((0, 0), (T.shape[1] - 1, T.shape[2] - 1), (T.shape[1] // 2, T.shape[2] // 2))]
    P.check_tiles(gpu, X32, W32, orc.S, spec.group, samples)
