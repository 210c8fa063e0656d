#!/usr/bin/env python
"""Benchmark of the AWQ per-layer activation-aware scale search on B200.

One step = one complete search of one synthetic layer (statistic, 20 candidate scale
vectors, QDQ + fold-back of every candidate, the reference GEMM, 20 candidate GEMMs
with the fused squared-error epilogue, argmin, packing) through the library's C ABI.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

Under torchrun each rank searches its own layer (a different seed) on its own GPU:
independent problems, no data-path collective, weak scaling. Rank 0 prints one JSON
line. ``--impl reference`` times the CPU oracle on the host cores instead.
"""
from __future__ import annotations

import argparse
import csv
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
DEFAULT_WORKLOAD = "llama7b_attn_proj_4096x4096x4096"
FLUSH_BYTES = 256 << 20   # > 126 MB L2


def parse_args(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(WORKLOADS))
    ap.add_argument("--e2e-steps", type=int, default=None, help="steps of the host-buffer run (default: --steps)")
    ap.add_argument("--cpu-seconds", type=float, default=15.0, help="target CPU time of the oracle sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-clip", action="store_true", help="skip the clipping-search measurement")
    ap.add_argument("--no-w4a16", action="store_true", help="skip the W4A16 consumer measurement")
    ap.add_argument("--no-mlp-block", action="store_true", help="skip the MLP-block objective measurement")
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


def cpu_oracle_sample(spec: LayerSpec, target_s: float):
    """Time the oracle as it stands on a column slice of the layer (full X)."""
    import oracle as O
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
    Xd, Wd = X.to(dev), W.to(dev)
    stream = torch.cuda.Stream(dev)
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    awq.profile_enable(True)

    def barrier():
        if world > 1:
            import torch.distributed as dist
            dist.barrier(device_ids=[local])

    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            awq.search(Xd, Wd, spec.group, spec.n_grid, stream=stream)
        starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
        ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
        gemm_ms, qdq_ms, stat_ms, pack_ms, phase_sums = [], [], [], [], []
        phase_tot = {}
        barrier()
        torch.cuda.synchronize(dev)
        clocks = ClockSampler(local)
        # the steps are enqueued back to back through the asynchronous entry point (a
        # model's layers are searched this way); each step's events bracket its own
        # kernels, the L2 flush before it stays outside them
        pending = []
        for i in range(args.steps):
            flush.zero_()
            starts[i].record(stream)
            pending.append(awq.search_async(Xd, Wd, spec.group, spec.n_grid, stream=stream))
            ends[i].record(stream)
        torch.cuda.synchronize(dev)
        for p in pending:
            out = p.wait()
            prof = p.profile()
            for k, v in prof.items():
                phase_tot[k] = phase_tot.get(k, 0.0) + v
            phase_sums.append(sum(prof.values()))
            gemm_ms.append(prof["gemm_reference"] + prof["gemm_loss"])  # one launch (or two) for both
            qdq_ms.append(prof["qdq"])
            stat_ms.append(prof["statistic"])
            pack_ms.append(prof["pack"])
        torch.cuda.synchronize(dev)
        barrier()
        clock_info = clocks.stop()
        launches = awq.last_launch_count() * args.steps
        step_ms = [s.elapsed_time(e) for s, e in zip(starts, ends)]
        total_ms = float(sum(step_ms))

        # end to end through the host-buffer entry points: every step copies its X and W
        # from pinned host memory, searches, and copies its artifact back. The batched call
        # (the way a model's layers are quantized) overlaps step i + 1's upload and step
        # i - 1's download with step i's search; the one-layer call is reported beside it.
        e2e_steps = args.e2e_steps or max(3, min(args.steps, 20))
        Xh, Wh = X.pin_memory(), W.pin_memory()

        def host_outputs():
            return (torch.empty(spec.K, dtype=torch.float32, pin_memory=True),
                    torch.empty(spec.K, spec.N // 8, dtype=torch.int32, pin_memory=True),
                    torch.empty(spec.K // spec.group, spec.N, dtype=torch.float16, pin_memory=True),
                    torch.empty(spec.K // spec.group, spec.N, dtype=torch.float16, pin_memory=True),
                    torch.empty(spec.n_grid, dtype=torch.float32, pin_memory=True))

        outs = [host_outputs() for _ in range(max(2, e2e_steps))]
        awq.search_host_batch([Xh, Xh], [Wh, Wh], spec.group, spec.n_grid, stream=stream, outs=outs[:2], device=dev)
        barrier()
        torch.cuda.synchronize(dev)
        flush.zero_()
        b_s, b_e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        b_s.record(stream)
        awq.search_host_batch([Xh] * e2e_steps, [Wh] * e2e_steps, spec.group, spec.n_grid, stream=stream,
                              outs=outs[:e2e_steps], device=dev)
        b_e.record(stream)
        torch.cuda.synchronize(dev)
        barrier()
        e2e_ms = float(b_s.elapsed_time(b_e))
        single_steps = max(3, min(e2e_steps, 10))
        e_s = [torch.cuda.Event(enable_timing=True) for _ in range(single_steps)]
        e_e = [torch.cuda.Event(enable_timing=True) for _ in range(single_steps)]
        for i in range(single_steps):
            flush.zero_()
            e_s[i].record(stream)
            awq.search_host(Xh, Wh, spec.group, spec.n_grid, stream=stream, out=outs[0], device=dev)
            e_e[i].record(stream)
        torch.cuda.synchronize(dev)
        single_ms = float(sum(s.elapsed_time(e) for s, e in zip(e_s, e_e))) / single_steps

        # the next rows of the pipeline: clipping search with the chosen scales, and the
        # artifact's W4A16 consumer
        clip = None if args.no_clip else measure_clip(awq, spec, Xd, Wd, out.scales, stream, flush,
                                                      max(3, min(args.steps, 10)))
        w4a16 = None if args.no_w4a16 else measure_w4a16(awq, spec, X, out, stream, flush,
                                                         max(5, min(args.steps, 20)), measured_peaks()[0])
        mlp = None if args.no_mlp_block else measure_mlp_block(awq, stream, flush, 3, measured_peaks()[0])

    total_ms, e2e_ms = max_over_ranks([total_ms, e2e_ms], dev)

    flops = spec.candidate_flops
    gemm_kernel = ("loss_gemm_pair_kernel" if awq.loss_gemm_variant(spec.M, spec.K, spec.N, spec.n_grid) == 2
                   else "loss_gemm_kernel")
    value = weak_scaling_tflops(world, args.steps, flops, total_ms)
    layers_per_s = world * args.steps / (total_ms / 1e3)
    e2e_value = weak_scaling_tflops(world, e2e_steps, flops, e2e_ms)
    peaks, peak_kind = measured_peaks()
    gemm_avg = statistics.mean(gemm_ms)
    gemm_flops = flops * (spec.n_grid + 1) / spec.n_grid  # the candidates' GEMMs and the reference output's
    achieved = gemm_flops / (gemm_avg / 1e3) / 1e12
    peak = float(peaks["bf16_tflops"])
    h2d = X.numel() * X.element_size() + W.numel() * W.element_size()
    d2h = sum(t.numel() * t.element_size() for t in outs[0])
    qdq_bytes = (W.element_size() + 2 * (spec.n_grid + 1)) * spec.K * spec.N
    stat_bytes = X.numel() * X.element_size() + 4 * spec.K
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": total_ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": spec.name, "M": spec.M, "K": spec.K, "N": spec.N, "group": spec.group,
                   "n_grid": spec.n_grid, "input_dtype": spec.dtype, "parallelism": f"independent layers x{world}",
                   "l2": "flushed between steps (256 MiB device write outside the timed events)"},
        "layers_per_s": layers_per_s,
        "roofline": {"bound": "tensor",
                     "kernel": gemm_kernel + (" (reference output + candidate GEMMs + fused squared error, one launch)"
                                              if gemm_kernel == "loss_gemm_kernel" else
                                              " (candidate GEMMs + fused squared error; reference output in its own launch)"),
                     "work": "(n_grid + 1) x 2 M K N flops per search (the reference output and every candidate)",
                     "achieved": achieved, "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
                     "peak_source": f"{peak_kind} bf16_tflops (burst)",
                     "traffic": recorded_traffic(gemm_kernel, spec.name),
                     "traffic_unit": "DRAM bytes per launch (ncu dram__bytes_read.sum + dram__bytes_write.sum)",
                     "ms_per_launch": gemm_avg},
        "other_kernels": {
            "qdq": {"ms": statistics.mean(qdq_ms),
                    "GB/s": qdq_bytes / (statistics.mean(qdq_ms) / 1e3) / 1e9,
                    "hbm_frac": qdq_bytes / (statistics.mean(qdq_ms) / 1e3) / 1e9 / float(peaks["hbm_gbs"])},
            "statistic": {"ms": statistics.mean(stat_ms),
                          "GB/s": stat_bytes / (statistics.mean(stat_ms) / 1e3) / 1e9,
                          "hbm_frac": stat_bytes / (statistics.mean(stat_ms) / 1e3) / 1e9 / float(peaks["hbm_gbs"])},
            "pack": {"ms": statistics.mean(pack_ms)},
        },
        "phases_ms": {k: v / args.steps for k, v in phase_tot.items()},
        "host_gap_ms": total_ms / args.steps - statistics.mean(phase_sums),
        "e2e": {"value": e2e_value, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "ms_per_step": e2e_ms / e2e_steps, "steps": e2e_steps,
                "api": "awq_search_host_batch over the steps (step i + 1 uploaded while step i runs)",
                "single_call_ms": single_ms,
                "single_call_value": flops / (single_ms / 1e3) / 1e12},
        "gpu_launches": launches,
        "clocks": clock_info,
        "chosen_alpha_index": out.best,
    }
    if clip is not None:
        line["clip_search"] = clip
    if w4a16 is not None:
        line["w4a16"] = w4a16
    if mlp is not None:
        line["mlp_block"] = mlp
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_oracle_sample(spec, args.cpu_seconds)
        if clip is not None:
            clip["cpu_baseline"] = cpu_clip_sample(spec, min(args.cpu_seconds, 10.0))
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
