#!/usr/bin/env python
"""Benchmark of the AWQ per-layer activation-aware scale search on B200.

One step = one complete search of one synthetic layer (statistic, 20 candidate scale
vectors, QDQ + fold-back of every candidate, the reference GEMM, 20 candidate GEMMs
with the fused squared-error epilogue, argmin, packing) through the library's C ABI.
The headline layer is the largest one, the Llama-70B-shaped gate+up projection
(16384 x 8192 x 57344); the other four layers of the workload set are timed in the
same run and reported as objects of the same line (``workloads``).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

Under torchrun each rank searches its own layer (a different seed) on its own GPU:
independent problems, no data-path collective, weak scaling. Rank 0 prints one JSON
line. ``--impl reference`` times the CPU oracle on the host cores instead.
"""
from __future__ import annotations

import argparse
import csv
import gc
import io
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

from workloads import WORKLOADS, LayerSpec, generate, as_f32_numpy  # noqa: E402

METRIC = "AWQ search candidate-GEMM TFLOP/s & layers/s; % of BF16 tensor peak"
DEFAULT_WORKLOAD = "llama70b_mlp_gate_up_16384x8192x57344"
# the layer the clipping search, the W4A16 consumer and the kernel-level objects run on
SIDE_WORKLOAD = "llama7b_attn_proj_4096x4096x4096"
FLUSH_BYTES = 256 << 20   # > 126 MB L2


def parse_args(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(WORKLOADS))
    ap.add_argument("--e2e-steps", type=int, default=None, help="steps of the host-buffer run (default: --steps)")
    ap.add_argument("--cpu-seconds", type=float, default=15.0, help="target CPU time of the oracle sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-clip", action="store_true", help="skip the clipping-search measurement")
    ap.add_argument("--no-w4a16", action="store_true", help="skip the W4A16 consumer measurement")
    ap.add_argument("--no-mlp-block", action="store_true", help="skip the MLP-block objective measurement")
    ap.add_argument("--no-attn-block", action="store_true", help="skip the attention-block objective measurement")
    ap.add_argument("--no-other-workloads", action="store_true",
                    help="time only the headline layer (skip the other layers' objects)")
    ap.add_argument("--slice-columns", type=int, default=0,
                    help="search a column slice of the layer instead: the first C columns of each half of a "
                         "[gate | up] layer (2C columns), else the first C; full X. For sized profiling captures")
    return ap.parse_args(argv)


# ----------------------------------------------------------------------------- helpers
def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


def recorded_traffic(kernel: str, workload: str):
    """DRAM bytes per launch from the committed ncu record, if it still matches the source."""
    import hashlib
    path = os.path.join(ROOT, "profiles", "roofline_traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        recs = json.load(f).get("records", [])
    for rec in recs:
        if rec.get("kernel") != kernel or rec.get("workload") != workload:
            continue
        for rel, digest in rec.get("sources_sha256", {}).items():
            full = os.path.join(ROOT, rel)
            if not os.path.exists(full):
                return None
            with open(full, "rb") as f:
                if hashlib.sha256(f.read()).hexdigest() != digest:
                    return None
        return float(rec["dram_bytes_per_launch"])
    return None


def cpu_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count() or 1


class ClockSampler:
    """nvidia-smi clocks and throttle reasons, sampled during the timed region."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int, period_ms: int = 50):
        self.proc = None
        self.file = None
        try:
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            ident = uuid if uuid.startswith("GPU-") else f"GPU-{uuid}"
            self.file = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", str(period_ms), "-i", ident], stdout=self.file, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.file.seek(0)
        rows = [r for r in csv.reader(io.StringIO(self.file.read())) if len(r) >= 9]
        self.file.close()
        os.unlink(self.file.name)
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].strip().replace(".", "").isdigit()]
        smax = [float(r[2]) for r in rows if r[2].strip().replace(".", "").isdigit()]
        watts = [float(r[3]) for r in rows if r[3].strip().replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].strip() == "Active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": reasons, "samples": len(rows),
                "power_w_median": statistics.median(watts) if watts else None}


def cpu_oracle_sample(spec: LayerSpec, target_s: float, X=None, W=None):
    """Time the oracle as it stands on a column slice of the layer (full X)."""
    import oracle as O
    if X is None:
        X, W = generate(spec)
    X32, W32 = as_f32_numpy(X), as_f32_numpy(W)

    def run(ncols):
        t0 = time.perf_counter()
        O.search(X32, W32[:, :ncols], group=spec.group, n_grid=spec.n_grid)
        return time.perf_counter() - t0

    n = min(spec.N, 64)
    t = run(n)
    while t < target_s / 3 and n < spec.N:
        n = min(spec.N, n * 4)
        t = run(n)
    flops = 2.0 * spec.M * spec.K * n * spec.n_grid
    return {"value": flops / t / 1e12, "unit": "TFLOP/s", "cores": cpu_threads(), "kind": "oracle",
            "sample": f"{n} of {spec.N} output columns with the full {spec.M}x{spec.K} X "
                      f"({t:.1f} s, numpy fp64 oracle)",
            "seconds": t, "columns": n}


def clip_fmas(spec: LayerSpec, n_shrink: int) -> float:
    """Multiply-adds the clipping search needs: for every (threshold, group, column) the
    distinct products of the symmetric quadratic form delta^T H delta, g (g + 1) / 2."""
    g = spec.group
    return float(n_shrink) * (spec.K // g) * spec.N * g * (g + 1) / 2


def measure_clip(awq, spec: LayerSpec, Xd, Wd, scales, stream, flush, steps: int, n_shrink: int = 10):
    """Device time of the clipping search (Gram matrices + search + clipped artifact) on
    the same resident layer, with the fp64 tensor-core roofline of its search kernel."""
    for _ in range(2):
        awq.clip_search(Xd, Wd, scales, spec.group, n_shrink, stream=stream)
    s_ev = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    e_ev = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    gram, search = [], []
    for i in range(steps):
        flush.zero_()
        s_ev[i].record(stream)
        awq.clip_search(Xd, Wd, scales, spec.group, n_shrink, stream=stream)
        e_ev[i].record(stream)
        p = awq.clip_profile_last()
        gram.append(p["gram"])
        search.append(p["clip_search"])
    torch.cuda.synchronize()
    call_ms = statistics.mean(s.elapsed_time(e) for s, e in zip(s_ev, e_ev))
    peak = awq.fp64_mma_peak(stream=stream)
    flops = 2.0 * clip_fmas(spec, n_shrink)
    ms = statistics.mean(search)
    achieved = flops / (ms / 1e3) / 1e12
    return {
        "n_shrink": n_shrink, "tokens": awq.clip_token_count(spec.M), "steps": steps,
        "ms_per_call": call_ms, "gram_ms": statistics.mean(gram), "search_ms": ms,
        "layers_per_s": 1e3 / call_ms, "gpu_launches_per_call": awq.last_launch_count(),
        "roofline": {"bound": "tensor", "kernel": "clip_kernel (fp64 MMA quadratic forms + clipped artifact)",
                     "achieved": achieved, "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
                     "peak_source": "fp64 tensor-core MMA throughput measured in this run (awq_fp64_mma_peak)",
                     "work": "2 * n_shrink * groups * N * g (g + 1) / 2 flops (distinct products of the "
                             "symmetric quadratic forms)",
                     "traffic": recorded_traffic("clip_kernel", spec.name),
                     "traffic_unit": "DRAM bytes per launch (ncu dram__bytes_read.sum + dram__bytes_write.sum)"},
    }


def _time_w4a16(awq, fn, flush, steps):
    """Device time of one call (the library's own events around its launches). A short
    device-side spin after the L2 flush keeps the GPU busy while the host enqueues the
    call, so the events see the kernels, not the host's launch latency."""
    for _ in range(2):
        fn()
    awq.profile_enable(True)
    ms = []
    for _ in range(steps):
        flush.zero_()
        torch.cuda._sleep(200_000)  # about 0.1 ms at the B200's clocks
        fn()
        ms.append(awq.w4a16_profile_last())
    return statistics.median(ms), awq.last_launch_count()


def measure_w4a16(awq, spec: LayerSpec, X, out, stream, flush, steps: int, peaks):
    """The artifact's W4A16 consumer on the same layer: decode (1 token on the repacked
    codes, fused GEMV; HBM roofline over the 4.25-bit weight stream), the same on a
    Llama-70B gate+up-shaped artifact (where the stream, 250 MB, dwarfs launch latency),
    and prefill (all M tokens, dequantize + tensor-core GEMM; fp16 tensor roofline)."""
    Xd = X.to(out.scales.device).float()
    A = (Xd / out.scales[None, :]).half()  # activations divided by the chosen scales
    hbm = float(peaks["hbm_gbs"])

    def decode_entry(K, N, group, t, launches, kernel):
        stream_bytes = K * N / 2 + 4 * (K // group) * N + 2 * K + 4 * N
        gbs = stream_bytes / (t / 1e3) / 1e9
        return {"M": 1, "K": K, "N": N, "ms": t, "gpu_launches_per_call": launches, "GB/s": gbs,
                "roofline": {"bound": "hbm", "kernel": kernel, "achieved": gbs, "peak": hbm, "unit": "GB/s",
                             "frac": gbs / hbm, "work": "K N / 2 code bytes + 4 bytes per (group, column) + 2 K + 4 N"}}

    res = {}
    packed = awq.w4a16_repack(out.codes, stream=stream)  # once, as at load time
    A1 = A[:1].contiguous()
    t, n = _time_w4a16(awq, lambda: awq.w4a16_matmul_packed(A1, packed, out.steps, out.zeros, spec.group,
                                                             stream=stream), flush, steps)
    res["decode"] = decode_entry(spec.K, spec.N, spec.group, t, n, "gemv_stream_kernel (repacked codes)")
    t, n = _time_w4a16(awq, lambda: awq.w4a16_matmul(A1, out.codes, out.steps, out.zeros, spec.group,
                                                      stream=stream), flush, steps)
    res["decode_plain_layout"] = decode_entry(spec.K, spec.N, spec.group, t, n, "gemv_kernel (artifact layout)")
    big = WORKLOADS["llama70b_mlp_gate_up_16384x8192x57344"]
    gen = torch.Generator(device=out.codes.device).manual_seed(0)
    codes70 = torch.randint(-2 ** 31, 2 ** 31 - 1, (big.K, big.N // 8), dtype=torch.int32, device=out.codes.device,
                            generator=gen)
    steps70 = (torch.rand(big.K // big.group, big.N, device=out.codes.device, generator=gen) * 0.01 + 1e-4).half()
    zeros70 = torch.randint(0, 16, (big.K // big.group, big.N), device=out.codes.device, generator=gen).half()
    packed70 = awq.w4a16_repack(codes70, stream=stream)
    A70 = torch.randn(1, big.K, device=out.codes.device, generator=gen).half()
    t, n = _time_w4a16(awq, lambda: awq.w4a16_matmul_packed(A70, packed70, steps70, zeros70, big.group,
                                                             stream=stream), flush, steps)
    res["decode_70b_gate_up_shape"] = decode_entry(big.K, big.N, big.group, t, n,
                                                   "gemv_stream_kernel (random artifact of the 70B gate+up shape)")
    del codes70, steps70, zeros70, packed70
    M = spec.M
    Am = A[:M].contiguous()
    t, launches = _time_w4a16(awq, lambda: awq.w4a16_matmul(Am, out.codes, out.steps, out.zeros, spec.group,
                                                             stream=stream), flush, steps)
    tflops = 2.0 * M * spec.K * spec.N / (t / 1e3) / 1e12
    peak = float(peaks["bf16_tflops"])
    res["prefill"] = {"M": M, "ms": t, "gpu_launches_per_call": launches, "TFLOP/s": tflops,
                      "roofline": {"bound": "tensor", "kernel": "dequant_kernel + loss_gemm_kernel mode 2 (fp16)",
                                   "achieved": tflops, "peak": peak, "unit": "TFLOP/s", "frac": tflops / peak,
                                   "peak_source": "bf16 dense burst peak (fp16 runs at the same rate)",
                                   "work": "2 M K N flops (both kernels' time)"}}
    awq.profile_enable(True)
    return res


MLP_BLOCK = "llama7b_mlp_gate_up_4096x4096x22016"  # [gate | up] of the block; the down projection 11008 x 4096


def measure_mlp_block(awq, stream, flush, steps: int, peaks, k_out: int = 4096):
    """The module-level objective on a Llama-7B MLP block: the gate and up projections
    searched on down(silu(gate) * up). Device time of the whole call (CUDA events);
    the work is every candidate's two GEMMs plus the reference block's."""
    from workloads import generate_down
    spec = WORKLOADS[MLP_BLOCK]
    X, W_gu = generate(spec)
    W_down = generate_down(spec, k_out)
    dev = torch.device("cuda", torch.cuda.current_device())
    Xd, Wg, Wd = X.to(dev), W_gu.to(dev), W_down.to(dev)
    for _ in range(2):
        out = awq.search_mlp(Xd, Wg, Wd, spec.group, spec.n_grid, stream=stream)
    s_ev = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    e_ev = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    for i in range(steps):
        flush.zero_()
        s_ev[i].record(stream)
        out = awq.search_mlp(Xd, Wg, Wd, spec.group, spec.n_grid, stream=stream)
        e_ev[i].record(stream)
    torch.cuda.synchronize()
    ms = statistics.mean(s.elapsed_time(e) for s, e in zip(s_ev, e_ev))
    F = spec.N // 2
    flops = (spec.n_grid + 1) * (2.0 * spec.M * spec.K * spec.N + 2.0 * spec.M * F * k_out)
    achieved = flops / (ms / 1e3) / 1e12
    peak = float(peaks["bf16_tflops"])
    del Xd, Wg, Wd
    return {"workload": f"{MLP_BLOCK} + down {F}x{k_out}", "ms_per_search": ms, "steps": steps,
            "gpu_launches_per_search": awq.last_launch_count(), "chosen_alpha_index": out.best,
            "TFLOP/s": achieved,
            "roofline": {"bound": "tensor", "kernel": "loss_gemm_kernel modes 3 and 1 (silu-mul fused in the first GEMM epilogue; + QDQ, pack)",
                         "achieved": achieved, "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
                         "peak_source": "measured bf16_tflops (burst)",
                         "work": "(n_grid + 1) x (2 M K 2F + 2 M F K_out) flops over the whole call"}}


ATTN_BLOCK = "llama7b_attn_proj_4096x4096x4096"  # the query projection; 8 sequences x 512 tokens, 32 heads


def attn_flops_per_slot(M: int, D: int, T: int) -> float:
    """Tensor-core flops of the causal attention of one slot: for every query block i of
    128 rows, (i + 1) key tiles of 128 x 128 x 128 for the scores and as many for P V."""
    nqt = T // 128
    return 4.0 * 128 ** 3 * (nqt * (nqt + 1) / 2) * (M // T) * (D // 128)


def measure_attn_block(awq, stream, flush, steps: int, peaks, seq_len: int = 512, n_heads: int = 32):
    """The module-level objective on a Llama-7B attention block: the query, key and value
    projections searched on their causal multi-head attention output. Device time of the
    whole call (CUDA events) and of its phases (the library's events)."""
    from workloads import generate_qkv
    spec = WORKLOADS[ATTN_BLOCK]
    X, _ = generate(spec)
    W = generate_qkv(spec)
    dev = torch.device("cuda", torch.cuda.current_device())
    Xd, Wd = X.to(dev), W.to(dev)
    for _ in range(2):
        out = awq.search_attn(Xd, Wd, n_heads, seq_len, spec.group, spec.n_grid, stream=stream)
    s_ev = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    e_ev = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    phases = []
    for i in range(steps):
        flush.zero_()
        s_ev[i].record(stream)
        out = awq.search_attn(Xd, Wd, n_heads, seq_len, spec.group, spec.n_grid, stream=stream)
        e_ev[i].record(stream)
        phases.append(awq.attn_profile_last())
    torch.cuda.synchronize()
    ms = statistics.mean(s.elapsed_time(e) for s, e in zip(s_ev, e_ev))
    M, K, D = spec.M, spec.K, spec.K
    slots = spec.n_grid + 1
    gemm_flops = slots * 2.0 * M * K * 3 * D
    attn_flops = slots * attn_flops_per_slot(M, D, seq_len)
    ph = {k: statistics.mean(p[k] for p in phases) for k in phases[0]}
    gemm_ms = ph["gemm_qk"] + ph["gemm_vt"]
    att_ms = ph["attention_reference"] + ph["attention_loss"]
    peak = float(peaks["bf16_tflops"])
    gemm_tf = gemm_flops / (gemm_ms / 1e3) / 1e12
    att_tf = attn_flops / (att_ms / 1e3) / 1e12
    total_tf = (gemm_flops + attn_flops) / (ms / 1e3) / 1e12
    del Xd, Wd
    return {"workload": f"{ATTN_BLOCK} as W_q of [W_q | W_k | W_v] 4096x12288, {M // seq_len} sequences x "
                        f"{seq_len} tokens, {n_heads} heads of 128",
            "ms_per_search": ms, "steps": steps, "gpu_launches_per_search": awq.last_launch_count(),
            "chosen_alpha_index": out.best, "TFLOP/s": total_tf, "phases_ms": ph,
            "roofline": {"bound": "tensor", "kernel": "loss_gemm_kernel mode 5 (Q|K and V^T products of all slots)",
                         "achieved": gemm_tf, "peak": peak, "unit": "TFLOP/s", "frac": gemm_tf / peak,
                         "peak_source": "measured bf16_tflops (burst)",
                         "work": "(n_grid + 1) x 2 M K 3D flops"},
            "attention_roofline": {"bound": "tensor",
                                   "kernel": "attn_loss_kernel (tcgen05 scores and P V, exact-max softmax, fused loss)",
                                   "achieved": att_tf, "peak": peak, "unit": "TFLOP/s", "frac": att_tf / peak,
                                   "peak_source": "measured bf16_tflops (burst)",
                                   "work": "(n_grid + 1) x 4 x 128^3 x (causal key tiles) flops",
                                   "ms": att_ms}}


def cpu_clip_sample(spec: LayerSpec, target_s: float, n_shrink: int = 10):
    """The clipping oracle as it stands on a column slice (full X, same scales reading)."""
    import oracle as O
    import oracle.awq_clip as C
    X, W = generate(spec)
    X32, W32 = as_f32_numpy(X), as_f32_numpy(W)
    s = O.candidate_scales(O.activation_statistic(X32), spec.n_grid)[spec.n_grid // 2]

    def run(ncols):
        t0 = time.perf_counter()
        C.clip_search(X32, W32[:, :ncols], s, spec.group, n_shrink)
        return time.perf_counter() - t0

    n = min(spec.N, 64)
    t = run(n)
    while t < target_s / 3 and n < spec.N:
        n = min(spec.N, n * 4)
        t = run(n)
    sub = LayerSpec(**{**spec.as_dict(), "N": n})
    return {"value": 2.0 * clip_fmas(sub, n_shrink) / t / 1e12, "unit": "TFLOP/s", "cores": cpu_threads(),
            "kind": "oracle", "sample": f"{n} of {spec.N} output columns ({t:.1f} s, numpy fp64 oracle)"}


def rank_spec(base: LayerSpec, rank: int) -> LayerSpec:
    """The layer rank `rank` searches: the workload's shape with its own seed."""
    return LayerSpec(**{**base.as_dict(), "seed": base.seed + rank})


def max_over_ranks(values, device) -> list:
    """Element-wise maximum over all ranks (the slowest rank's device times)."""
    t = torch.tensor(values, dtype=torch.float64, device=device)
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def weak_scaling_tflops(world: int, steps: int, flops_per_step: float, total_ms: float) -> float:
    """All ranks' candidate-GEMM work divided by the slowest rank's time."""
    return world * steps * flops_per_step / (total_ms / 1e3) / 1e12


# ----------------------------------------------------------------------------- arms
def run_reference(args, rank, world):
    spec = WORKLOADS[args.workload]
    if rank != 0:
        return 0
    import oracle as O
    X, W = generate(spec)
    X32, W32 = as_f32_numpy(X), as_f32_numpy(W)
    # size the per-step sample so warm-up + steps end within a few minutes
    per_step_s = max(1.0, 150.0 / max(1, args.steps + args.warmup))
    n = min(spec.N, 64)
    t0 = time.perf_counter()
    O.search(X32, W32[:, :n], group=spec.group, n_grid=spec.n_grid)
    t = time.perf_counter() - t0
    while t < per_step_s / 3 and n < spec.N:
        n = min(spec.N, n * 4)
        t0 = time.perf_counter()
        O.search(X32, W32[:, :n], group=spec.group, n_grid=spec.n_grid)
        t = time.perf_counter() - t0
    for _ in range(args.warmup):
        O.search(X32, W32[:, :n], group=spec.group, n_grid=spec.n_grid)
    times = []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        O.search(X32, W32[:, :n], group=spec.group, n_grid=spec.n_grid)
        times.append(time.perf_counter() - t0)
    total = sum(times)
    flops = 2.0 * spec.M * spec.K * n * spec.n_grid
    value = flops * args.steps / total / 1e12
    sample = f"{n} of {spec.N} output columns with the full {spec.M}x{spec.K} X per step"
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": spec.name, "M": spec.M, "K": spec.K, "N": spec.N, "group": spec.group,
                   "n_grid": spec.n_grid, "sample_columns": n},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cpu_threads(), "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def time_searches(awq, spec: LayerSpec, Xd, Wd, stream, flush, steps: int, warmup: int, barrier=None,
                  sample_clocks: int | None = None):
    """Device time of `steps` searches of one resident layer, enqueued back to back through
    the asynchronous entry point (a model's layers are searched this way). Each step's
    events bracket its own kernels; the L2 flush before it stays outside them. Returns the
    per-step times, the phase times of every step and the last search's output."""
    for _ in range(warmup):
        awq.search(Xd, Wd, spec.group, spec.n_grid, stream=stream)
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    # every step's outputs and status word exist before the timed region, so the host
    # enqueues the steps without allocating (and without the garbage collector running)
    outs = [awq.alloc_outputs(spec.K, spec.N, spec.group, spec.n_grid, Xd.device) for _ in range(steps)]
    words = [torch.full((1,), -1, dtype=torch.int32, pin_memory=True) for _ in range(steps)]
    if barrier:
        barrier()
    torch.cuda.synchronize()
    clocks = ClockSampler(sample_clocks) if sample_clocks is not None else None
    pending = []
    gc.collect()
    gc.disable()
    try:
        for i in range(steps):
            flush.zero_()
            starts[i].record(stream)
            pending.append(awq.search_async(Xd, Wd, spec.group, spec.n_grid, stream=stream, out=outs[i],
                                            status=words[i]))
            ends[i].record(stream)
        torch.cuda.synchronize()
    finally:
        gc.enable()
    clock_info = clocks.stop() if clocks is not None else None
    phases = []
    out = None
    for p in pending:
        out = p.wait()
        phases.append(p.profile())
    if barrier:
        barrier()
    return {"step_ms": [s.elapsed_time(e) for s, e in zip(starts, ends)], "phases": phases, "out": out,
            "launches": awq.last_launch_count() * steps, "clocks": clock_info}


def search_object(awq, spec: LayerSpec, t: dict, peaks: dict, peak_kind: str, sustained: bool) -> dict:
    """ms per search, layers/s, candidate-GEMM TFLOP/s and the rooflines of one layer."""
    steps = len(t["step_ms"])
    total_ms = float(sum(t["step_ms"]))
    phases = t["phases"]
    mean = lambda key: statistics.mean(p[key] for p in phases)  # noqa: E731
    gemm_ms = statistics.mean(p["gemm_reference"] + p["gemm_loss"] for p in phases)
    gemm_flops = spec.candidate_flops * (spec.n_grid + 1) / spec.n_grid
    achieved = gemm_flops / (gemm_ms / 1e3) / 1e12
    peak_key = "bf16_tflops_sustained" if sustained else "bf16_tflops"
    peak = float(peaks[peak_key])
    gemm_kernel = ("loss_gemm_pair_kernel" if awq.loss_gemm_variant(spec.M, spec.K, spec.N, spec.n_grid) == 2
                   else "loss_gemm_kernel")
    tdt = torch.bfloat16 if spec.dtype == "bf16" else torch.float32
    gemm_launches = awq.loss_gemm_launches(spec.M, spec.K, spec.N, spec.n_grid, spec.group, tdt)
    qdq_warps = awq.qdq_in_loss_gemm(spec.M, spec.K, spec.N, spec.n_grid, spec.group, tdt)
    eb = 2 if spec.dtype == "bf16" else 4
    hbm = float(peaks["hbm_gbs"])
    qdq_bytes = (eb + 2 * (spec.n_grid + 1)) * spec.K * spec.N
    stat_bytes = spec.M * spec.K * eb + 4 * spec.K
    pack_bytes = spec.K * spec.N * (eb + 0.5) + 4 * (spec.K // spec.group) * spec.N + 4 * spec.K
    phase_tot = {}
    for p in phases:
        for k, v in p.items():
            phase_tot[k] = phase_tot.get(k, 0.0) + v

    def hbm_obj(name, nbytes, ms, work):
        gbs = nbytes / (ms / 1e3) / 1e9
        return {"kernel": name, "ms": ms, "bytes": nbytes, "GB/s": gbs, "hbm_frac": gbs / hbm, "work": work}

    if gemm_launches == 1:
        what = " (reference output + candidate GEMMs + fused squared error, one launch)"
    elif gemm_kernel == "loss_gemm_kernel":
        what = (" (reference output in its own launch, then the candidate GEMMs + fused squared error, every"
                " candidate of a column tile before the next; per launch = averaged over the two launches)")
    else:
        what = " (candidate GEMMs + fused squared error; reference output in its own launch)"
    if qdq_warps:
        what += "; its QDQ warps make the candidate operands (QDQ) inside the same launches"
    roof = {"bound": "tensor",
            "kernel": gemm_kernel + what,
            "launches_per_search": gemm_launches,
            "work": "(n_grid + 1) x 2 M K N flops per search (the reference output and every candidate)",
            "achieved": achieved, "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
            "peak_source": f"{peak_kind} {peak_key} ({'sustained: the kernel runs for a long step' if sustained else 'burst'})",
            "traffic": recorded_traffic(gemm_kernel, spec.name),
            "traffic_unit": "DRAM bytes per launch (ncu dram__bytes_read.sum + dram__bytes_write.sum)",
            "ms_per_launch": gemm_ms / gemm_launches}
    return {
        "workload": spec.name, "M": spec.M, "K": spec.K, "N": spec.N, "group": spec.group, "n_grid": spec.n_grid,
        "input_dtype": spec.dtype, "steps": steps, "ms_per_step": total_ms / steps,
        "ms_per_step_min_max": [min(t["step_ms"]), max(t["step_ms"])],
        "layers_per_s": steps / (total_ms / 1e3),
        "TFLOP/s": spec.candidate_flops * steps / (total_ms / 1e3) / 1e12,
        "roofline": roof,
        "other_kernels": {
            "qdq": (hbm_obj("qdq_kernel (the reference operand alone)", (eb + 2) * spec.K * spec.N, mean("qdq"),
                            "reads W once, writes the bf16 reference operand; the n_grid candidate operands "
                            "are made by the loss GEMM's QDQ warps inside its two launches") if qdq_warps else
                    hbm_obj("qdq_kernel", qdq_bytes, mean("qdq"), "reads W once, writes n_grid + 1 bf16 operand slots")),
            "statistic": hbm_obj("statistic_kernel", stat_bytes, mean("statistic"), "reads X once, writes a"),
            "pack": hbm_obj("pack_kernel", pack_bytes, mean("pack"),
                            "reads W once, writes the codes, steps, zeros and scales"),
            "scales_ms": mean("scales"), "loss_reduce_ms": mean("loss_reduce"),
        },
        "phases_ms": {k: v / steps for k, v in phase_tot.items()},
        "host_gap_ms": total_ms / steps - statistics.mean(sum(p.values()) for p in phases),
        "gpu_launches_per_search": t["launches"] // steps,
        "chosen_alpha_index": t["out"].best,
    }


def measure_e2e(awq, spec: LayerSpec, X, W, stream, flush, dev, steps: int, barrier):
    """The same metric end to end through the host-buffer entry points: every step copies
    its X and W from pinned host memory, searches, and copies its artifact back. The
    batched call (the way a model's layers are quantized) overlaps step i + 1's upload and
    step i - 1's download with step i's search; the one-layer call is reported beside it."""
    Xh, Wh = X.pin_memory(), W.pin_memory()

    def host_outputs():
        return (torch.empty(spec.K, dtype=torch.float32, pin_memory=True),
                torch.empty(spec.K, spec.N // 8, dtype=torch.int32, pin_memory=True),
                torch.empty(spec.K // spec.group, spec.N, dtype=torch.float16, pin_memory=True),
                torch.empty(spec.K // spec.group, spec.N, dtype=torch.float16, pin_memory=True),
                torch.empty(spec.n_grid, dtype=torch.float32, pin_memory=True),
                torch.empty(1, dtype=torch.int32, pin_memory=True))

    # two output sets used in turn: layer i and i + 2 copy back on one stream, in order
    sets = [host_outputs(), host_outputs()]
    outs = [sets[i % 2] for i in range(steps)]
    awq.search_host_batch([Xh, Xh], [Wh, Wh], spec.group, spec.n_grid, stream=stream, outs=sets, device=dev)
    barrier()
    torch.cuda.synchronize(dev)
    flush.zero_()
    b_s, b_e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    b_s.record(stream)
    awq.search_host_batch([Xh] * steps, [Wh] * steps, spec.group, spec.n_grid, stream=stream, outs=outs, device=dev)
    b_e.record(stream)
    torch.cuda.synchronize(dev)
    barrier()
    e2e_ms = float(b_s.elapsed_time(b_e))
    single_steps = 3
    e_s = [torch.cuda.Event(enable_timing=True) for _ in range(single_steps)]
    e_e = [torch.cuda.Event(enable_timing=True) for _ in range(single_steps)]
    for i in range(single_steps):
        flush.zero_()
        e_s[i].record(stream)
        awq.search_host(Xh, Wh, spec.group, spec.n_grid, stream=stream, out=sets[0], device=dev)
        e_e[i].record(stream)
    torch.cuda.synchronize(dev)
    single_ms = float(sum(s.elapsed_time(e) for s, e in zip(e_s, e_e))) / single_steps
    h2d = X.numel() * X.element_size() + W.numel() * W.element_size()
    d2h = sum(t.numel() * t.element_size() for t in sets[0])
    return e2e_ms, single_ms, h2d, d2h


def other_workload(awq, name: str, stream, flush, steps: int, warmup: int, peaks, peak_kind):
    """One of the other layers of the workload set, timed like the headline (its own
    inputs resident in HBM, L2 flushed between steps). Its oracle sample is taken later,
    once every GPU timing is done, so that no host thread competes with the enqueueing."""
    spec = WORKLOADS[name]
    X, W = generate(spec)
    Xd, Wd = X.cuda(), W.cuda()
    t = time_searches(awq, spec, Xd, Wd, stream, flush, steps, warmup, sample_clocks=Xd.device.index)
    obj = search_object(awq, spec, t, peaks, peak_kind, sustained=False)
    obj["clocks"] = t["clocks"]  # sampled during this layer's timed region
    if spec.M * spec.K * spec.N <= 128 * 256 * 256:
        obj["bound"] = ("latency: 7 launches of a few microseconds each; the tensor and HBM "
                        "fractions are not meaningful at this size")
    del Xd, Wd
    return obj, (spec, X, t["out"])


def column_slice(spec: LayerSpec, W: torch.Tensor, cols: int):
    """The layer restricted to a column slice of W (the same values as in the full layer):
    for a joint [gate | up] layer the first `cols` columns of each half, else the first
    `cols` columns."""
    if cols <= 0 or cols % 8:
        raise ValueError("--slice-columns takes a positive multiple of 8")
    if "gate_up" in spec.name:
        half = spec.N // 2
        Ws = torch.cat([W[:, :min(cols, half)], W[:, half:half + min(cols, half)]], dim=1).contiguous()
        tag = f"cols0-{min(cols, half)}+{half}-{half + min(cols, half)}"
    else:
        Ws = W[:, :min(cols, spec.N)].contiguous()
        tag = f"cols0-{min(cols, spec.N)}"
    return LayerSpec(**{**spec.as_dict(), "name": f"{spec.name}[{tag}]", "N": Ws.shape[1]}), Ws


def run_ours(args, rank, world, local):
    import post_quantization_column_b200 as awq
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    spec = rank_spec(WORKLOADS[args.workload], rank)
    X, W = generate(spec)
    if args.slice_columns:
        spec, W = column_slice(spec, W, args.slice_columns)
    Xd, Wd = X.to(dev), W.to(dev)
    stream = torch.cuda.Stream(dev)
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    awq.profile_enable(True)
    peaks, peak_kind = measured_peaks()
    # a step of the large layers runs its loss GEMM for tens to hundreds of milliseconds:
    # the power-capped sustained peak is its ceiling; the small layers' steps are bursts
    sustained = spec.candidate_flops >= 50e12

    def barrier():
        if world > 1:
            import torch.distributed as dist
            dist.barrier(device_ids=[local])

    with torch.cuda.stream(stream):
        t = time_searches(awq, spec, Xd, Wd, stream, flush, args.steps, args.warmup, barrier, sample_clocks=local)
        total_ms = float(sum(t["step_ms"]))
        head = search_object(awq, spec, t, peaks, peak_kind, sustained)
        out = t["out"]
        del Xd, Wd
        e2e_steps = args.e2e_steps or max(3, min(args.steps, 20))
        e2e_ms, single_ms, h2d, d2h = measure_e2e(awq, spec, X, W, stream, flush, dev, e2e_steps, barrier)

        # the other layers of the workload set (rank 0 of a single-GPU run only: under
        # torchrun every rank runs the headline layer alone)
        others = {}
        side = None
        if world == 1 and not args.no_other_workloads:
            for name in WORKLOADS:
                if name == spec.name:
                    continue
                obj, keep = other_workload(awq, name, stream, flush, max(3, min(args.steps, 20)), max(3, args.warmup),
                                           peaks, peak_kind)
                others[name] = obj
                if name == SIDE_WORKLOAD:
                    side = keep
        if side is None and spec.name == SIDE_WORKLOAD:
            side = (spec, X, out)

        # the next rows of the pipeline on the 4096^3 layer: clipping search with the
        # chosen scales, the artifact's W4A16 consumer, and the MLP-block objective
        clip = w4a16 = mlp = None
        if side is not None:
            s_spec, s_X, s_out = side
            s_Xd, s_Wd = (t_.to(dev) for t_ in generate(s_spec))
            clip = None if args.no_clip else measure_clip(awq, s_spec, s_Xd, s_Wd, s_out.scales, stream, flush,
                                                          max(3, min(args.steps, 10)))
            w4a16 = None if args.no_w4a16 else measure_w4a16(awq, s_spec, s_X, s_out, stream, flush,
                                                             max(5, min(args.steps, 20)), peaks)
            del s_Xd, s_Wd
        mlp = None if args.no_mlp_block else measure_mlp_block(awq, stream, flush, 3, peaks)
        attn = None if args.no_attn_block else measure_attn_block(awq, stream, flush, 3, peaks)

    total_ms, e2e_ms = max_over_ranks([total_ms, e2e_ms], dev)
    flops = spec.candidate_flops
    value = weak_scaling_tflops(world, args.steps, flops, total_ms)
    e2e_value = weak_scaling_tflops(world, e2e_steps, flops, e2e_ms)
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": total_ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": spec.name, "M": spec.M, "K": spec.K, "N": spec.N, "group": spec.group,
                   "n_grid": spec.n_grid, "input_dtype": spec.dtype, "parallelism": f"independent layers x{world}",
                   "l2": "flushed between steps (256 MiB device write outside the timed events)"},
        "layers_per_s": world * args.steps / (total_ms / 1e3),
        "roofline": head["roofline"],
        "other_kernels": head["other_kernels"],
        "phases_ms": head["phases_ms"],
        "host_gap_ms": head["host_gap_ms"],
        "e2e": {"value": e2e_value, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "ms_per_step": e2e_ms / e2e_steps, "steps": e2e_steps,
                "api": "awq_search_host_batch over the steps (step i + 1 uploaded while step i runs)",
                "single_call_ms": single_ms,
                "single_call_value": flops / (single_ms / 1e3) / 1e12},
        "gpu_launches": t["launches"],
        "clocks": t["clocks"],
        "chosen_alpha_index": out.best,
    }
    if others:
        line["workloads"] = others
    if clip is not None:
        line["clip_search"] = clip
    if w4a16 is not None:
        line["w4a16"] = w4a16
    if mlp is not None:
        line["mlp_block"] = mlp
    if attn is not None:
        line["attn_block"] = attn
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        # the oracle samples, after every GPU timing
        line["cpu_baseline"] = cpu_oracle_sample(spec, args.cpu_seconds, X, W)
        for name, obj in others.items():
            obj["cpu_baseline"] = cpu_oracle_sample(WORKLOADS[name], min(args.cpu_seconds, 5.0))
        if clip is not None:
            clip["cpu_baseline"] = cpu_clip_sample(side[0], min(args.cpu_seconds, 10.0))
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


def main(argv=None):
    args = parse_args(argv)
    rank, world, local = dist_env()
    if args.impl == "reference":
        return run_reference(args, rank, world)
    return run_ours(args, rank, world, local)


if __name__ == "__main__":
    sys.exit(main())
