"""Benchmark: exact causal GQA attention forward (Hq=16, Hkv=4, d=256) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]
                    [--fp32-path ffma|tc] [--pass fwd|bwd]

One step = one forward call over one synthetic input of the workload (default:
causal self-attention at L = 60,926 in fp32, the length the headline metric is
quoted at; --workload picks another configuration).  Inputs are resident in HBM
before the timed region and are larger than L2 (no flush needed).  Time: CUDA
events on the launching stream, W warm-up steps, then exactly K steps between a
barrier + synchronize on both sides; max over ranks.  Under torchrun every rank
runs its own replica (its own batch entry): weak scaling, no collective on the
data path.  Rank 0 prints one JSON line.

The default line (the fp32 workload at L = 60,926, one GPU) also carries, measured in
the same process after its own timing: `bf16` (the bf16 forward at L = 60,926, timed
the same way, with its roofline against both measured bf16 peaks and its clocks),
`bwd` (the backward at L = 16,384 in bf16 and fp32) and `memory_sweep` (peak device
memory over inputs against L, the 1M-token packed call and the fp32 tensor-core path,
beside the L x L score matrix of the math path).  --no-extras leaves them out.

--impl reference times the fp64 CPU oracle (the only reference this method has)
on a bounded sample of the same workload, on the host cores.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import long_context_causal_flash_b200 as gqa  # noqa: E402
from long_context_causal_flash_b200 import inputs, workloads  # noqa: E402

METRIC = "attention TFLOP/s and % of FP32/BF16 roofline at L=60,926; peak GiB vs L"
UNIT = "TFLOP/s"
SM_COUNT_B200 = 148
FP32_LANES_PER_SM = 128  # FFMA lanes per SM (4 sub-partitions x 32)


# ----------------------------------------------------------------------------- helpers
# DRAM bytes per launch (dram__bytes_read.sum + dram__bytes_write.sum) of the dominant
# kernel, from one single-pass ncu capture of the same bench command, keyed to the
# SHA-256 of the kernel's sources at capture time: a kernel changed since its capture
# reports null until it is captured again.
_TRAFFIC = {
    # (kernel, workload): (bytes per launch, sha256 of the sources)
    ("fwd_f32_kernel", "causal_60926_f32"): (6_452_098_048 + 983_006_464, "27f847b574f9dda9a3791d0943acae8649c80802be798649c00c4695e6b62834"),
    ("fwd_bf16_kernel", "causal_60926_bf16"): (1_182_908_928 + 468_306_688, "a82bb08b149624bc9f7bde68babab8fe2a30507381223273f606b96c6eaeab6a"),
    ("fwd_f32_tc_kernel", "causal_60926_f32"): (4_194_565_376 + 989_071_104, "ca2e569f7cc018d812899f9567e262ef5c0e4bd6513dd2a35754a41ad7a84746"),
}
_KERNEL_SOURCES = {
    "fwd_f32_kernel": ("fwd_f32.cu", "common.cuh", "internal.h"),
    "fwd_f32_tc_kernel": ("fwd_f32_tc.cu", "common.cuh", "tcgen05.cuh", "internal.h"),
    "fwd_bf16_kernel": ("fwd_bf16.cu", "common.cuh", "tcgen05.cuh", "internal.h"),
}


def kernel_digest(kernel):
    h = hashlib.sha256()
    for f in _KERNEL_SOURCES[kernel]:
        with open(os.path.join(ROOT, "long_context_causal_flash_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()


def _traffic(kernel, workload):
    ent = _TRAFFIC.get((kernel, workload))
    if ent is None or ent[1] != kernel_digest(kernel):
        return None
    return ent[0]


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "sm_max_mhz": 1965.0}, \
        "fallback"


def _fp32_peak_tflops(sm_count, sm_mhz):
    """FFMA roofline: SMs x 128 lanes x 2 flop x clock."""
    return sm_count * FP32_LANES_PER_SM * 2 * sm_mhz * 1e6 / 1e12


_FFMA2_CEILING = {}


def _ffma2_ceiling(dev, form=1):
    """Attainable rate of fp32 FMAs in one operand form (1: the FFMA kernels' packed form
    in the order they issue most of it),
    measured once per process with the library's register-only probe
    (`gqa_attn_probe_ffma2`, one CTA of 256 threads per SM, about 15-20 ms per
    repetition, the best of three)."""
    key = (str(dev), form)
    if key not in _FFMA2_CEILING:
        lib = gqa._lib.load()
        out = torch.empty(SM_COUNT_B200 * 256, dtype=torch.float32, device=dev)
        stream = torch.cuda.current_stream(dev)
        iters = 200_000
        gqa._lib.check("gqa_attn_probe_ffma2", lib.gqa_attn_probe_ffma2(out.data_ptr(), SM_COUNT_B200, 1000, form,
                                                                         stream.cuda_stream))
        best = 0.0
        for _ in range(3):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            gqa._lib.check("gqa_attn_probe_ffma2", lib.gqa_attn_probe_ffma2(out.data_ptr(), SM_COUNT_B200, iters,
                                                                             form, stream.cuda_stream))
            e1.record(stream)
            torch.cuda.synchronize(dev)
            ms = e0.elapsed_time(e1)
            best = max(best, 2.0 * SM_COUNT_B200 * 256 * iters * 64 / (ms * 1e-3) / 1e12)
        _FFMA2_CEILING[key] = best
    return _FFMA2_CEILING[key]


def _tile_summary(w, dtype_code, sq, skv, dev):
    """Tile configuration of the call and its block-skip plan's class counts, from the
    library's own plan export (`gqa_attn_tile_plan`); the counts are left out when the
    class matrix would exceed 64 M entries (the 1M-token calls)."""
    br, bc = gqa.tile_sizes(dtype_code, w.Hq, w.Hkv)
    nq, nk = -(-w.Lq // br), -(-w.Lk // bc)
    t = {"query_positions_per_tile": br, "query_rows_per_tile": br * (w.Hq // w.Hkv), "keys_per_tile": bc,
         "query_tiles": nq, "key_tiles": nk}
    if nq * nk <= (64 << 20):
        classes, _ = gqa.tile_plan(w.Hq, w.Hkv, w.Lq, w.Lk, dtype=dtype_code, mask_kind=w.mask_kind,
                                   q_pos_offset=w.q_pos_offset, seg_q=sq, seg_kv=skv, device=dev)
        counts = np.bincount(classes.reshape(-1), minlength=3)
        t.update({"skip": int(counts[0]), "partial": int(counts[1]), "full": int(counts[2]),
                  "per": "(query tile, key tile) pair of one kv head"})
    else:
        t["classes"] = f"not exported ({nq * nk} pairs)"
    return t


def _with_ffma2_ceiling(roof, dev):
    """Adds the measured packed-FMA ceiling next to the nominal FP32 peak of an FFMA roofline."""
    c = _ffma2_ceiling(dev)
    roof["ffma2_ceiling"] = {
        "value": c, "unit": UNIT, "frac": roof["achieved"] / c, "kernel": "ffma2_probe_kernel",
        "what": "register-only loop of fma.rn.f32x2 in the kernels' operand form ((q_r, q_r+1) x (k, k)), runs of "
                "eight sharing the register pair as in the kernels, 148 CTAs x 256 threads, timed in this run: the "
                "attainable rate of the instruction itself (frac above is against the nominal 128 lanes x 2 flop "
                "x clock)"}
    return roof


class ClockSampler:
    """Samples SM clock and throttle reasons with nvidia-smi while the timed region runs."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id):
        self.gpu_id = gpu_id
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu_id), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                smax = float(parts[1])
            except ValueError:
                continue
            for n, v in zip(names, parts[4:8]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["not sampled"]}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": smax, "reasons": sorted(reasons), "samples": len(sm)}


def _workload(name):
    try:
        return workloads.by_name(name)
    except KeyError as e:
        raise SystemExit(str(e)) from None


def _segment_ids(w):
    if w.branches:
        nb, bl = w.branches
        return inputs.branch_ids(w.q_pos_offset, nb, bl)
    if w.segments:
        ids = inputs.segment_ids(w.segments)
        return ids, ids
    return None, None


def _make_inputs(w, dev, seed_offset=0):
    seeds = (inputs.SEED_Q + seed_offset, inputs.SEED_K + seed_offset, inputs.SEED_V + seed_offset)
    big = w.Lq * w.Hq * w.d > (1 << 28)
    gen_dev = dev if big else "cpu"  # host generation for the sizes the oracle checks
    q, k, v = inputs.qkv(w.B, w.Hq, w.Hkv, w.Lq, w.Lk, w.d, dtype=w.dtype, device=gen_dev, seeds=seeds)
    sq, skv = _segment_ids(w)
    to = lambda x: None if x is None else torch.as_tensor(x, dtype=torch.int32).to(dev)
    return q.to(dev), k.to(dev), v.to(dev), to(sq), to(skv)


# ----------------------------------------------------------------------------- oracle arms
def _oracle_sample(w, budget_s, q, k, v, seg_q, seg_kv):
    """Times the fp64 oracle on seeded sampled rows until ~budget_s; returns (flops, seconds, rows)."""
    import numpy as np

    import oracle

    rng = np.random.default_rng(inputs.SEED_ROWS)
    order = rng.permutation(w.Lq)
    done, flops, t_total = 0, 0, 0.0
    mask = oracle.MASK_PREFIX_BRANCH if w.mask_kind == "prefix_branch" else oracle.MASK_CAUSAL
    sq = None if seg_q is None else seg_q
    skv = None if seg_kv is None else seg_kv
    while t_total < budget_s and done < w.Lq:
        rows = np.sort(order[done:done + 64])
        t0 = time.perf_counter()
        oracle.attention(q, k, v, mask_kind=mask, q_pos_offset=w.q_pos_offset, seg_q=sq, seg_kv=skv, rows=rows)
        t_total += time.perf_counter() - t0
        vis = oracle.visible(rows, w.Lk, mask_kind=mask, q_pos_offset=w.q_pos_offset, seg_q=sq, seg_kv=skv)
        flops += 4 * w.d * w.Hq * w.B * int(vis.sum())
        done += len(rows)
    return flops, t_total, done


def _blas_threads():
    try:
        from threadpoolctl import threadpool_info

        info = [i for i in threadpool_info() if i.get("user_api") == "blas"]
        if info:
            return int(info[0]["num_threads"])
    except Exception:
        pass
    return len(os.sched_getaffinity(0))


def _cpu_inputs(w):
    """Host copies of the workload's inputs (rows are sampled, so Q may be generated in full on host)."""
    q, k, v = inputs.qkv(w.B, w.Hq, w.Hkv, w.Lq, w.Lk, w.d, dtype=w.dtype, device="cpu")
    sq, skv = _segment_ids(w)
    return q, k, v, sq, skv


def run_reference(args, w, rank, world):
    if rank != 0:
        return
    q, k, v, sq, skv = _cpu_inputs(w)
    budget = max(2.0, 60.0 / max(1, args.steps + args.warmup))
    for _ in range(args.warmup):
        _oracle_sample(w, budget / 4, q, k, v, sq, skv)
    vals, secs = [], []
    rows_total = 0
    for _ in range(args.steps):
        f, t, n = _oracle_sample(w, budget, q, k, v, sq, skv)
        vals.append(f / t / 1e12)
        secs.append(t)
        rows_total += n
    value = statistics.median(vals)
    cores = _blas_threads()
    sample = f"{rows_total // max(1, args.steps)} seeded sampled query rows x {w.Hq} heads per step of {w.name}"
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": 1e3 * statistics.median(secs), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic N(0,1), seeds 1/2/3",
        "config": _config(w, world),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def _config(w, world):
    c = {"workload": w.name, "B_per_gpu": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "d": w.d, "Lq": w.Lq, "Lk": w.Lk,
         "mask": w.mask_kind, "q_pos_offset": w.q_pos_offset,
         "global_batch": w.B * world, "parallelism": f"replicas x{world} (one batch entry per GPU)",
         "l2": "inputs larger than L2 (no flush)" if w.io_bytes() >= 4 * 126e6
         else "L2 flushed between steps (512 MiB write outside the timed events)"}
    if w.segments:
        c["segments"] = len(w.segments)
    if w.branches:
        c["branches"] = list(w.branches)
    return c


# ----------------------------------------------------------------------------- GPU arm
def _max_over_ranks(x, dist, device):
    """Largest value of `x` over all ranks: one all-reduce of a scalar (timing only, not
    on the data path).  With no process group it returns `x`."""
    if dist is None:
        return x
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def _seed_offset(rank):
    """Each rank runs its own replica on its own batch entry: seeds shift by 10 per rank."""
    return 10 * rank


def _time_steps(fn, steps, stream, flush=None):
    """Per-step CUDA events on `stream`; `flush` (if any) runs between steps, outside the events."""
    start = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    end = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    for i in range(steps):
        if flush is not None:
            flush()
        start[i].record(stream)
        fn()
        end[i].record(stream)
    torch.cuda.synchronize()
    return [s.elapsed_time(e) for s, e in zip(start, end)]


SWEEP_L = (512, 4096, 15_231, 30_468, 60_926, 131_072, 262_144, 524_288, 1_048_576)


def memory_point(w, dev, fp32_path="ffma"):
    """Device memory one forward call needs beyond its inputs and outputs, for workload w:
    (peak bytes allocated over q/k/v/out/lse/ids, cudaMemGetInfo delta over the call)."""
    torch.cuda.synchronize(dev)
    torch.cuda.empty_cache()
    q, k, v, sq, skv = _make_inputs(w, dev)
    out = torch.empty_like(q)
    lse = torch.empty((w.B, w.Hq, w.Lq), device=dev, dtype=torch.float32)
    torch.cuda.synchronize(dev)
    io = torch.cuda.memory_allocated(dev)
    torch.cuda.reset_peak_memory_stats(dev)
    # The workspace (the caller's, through the binding) is the only memory beyond the
    # inputs and outputs; the library itself must allocate nothing during the call.
    code = gqa.GQA_F32_TC if fp32_path == "tc" else w.dtype
    need = gqa.workspace_bytes(w.B, w.Hq, w.Hkv, w.Lq, w.Lk, w.d, code, w.mask_kind, sq is not None)
    ws = torch.empty(max(need, 256), dtype=torch.uint8, device=dev)
    torch.cuda.synchronize(dev)
    free0, _ = torch.cuda.mem_get_info(dev)
    gqa.fwd(q, k, v, mask_kind=w.mask_kind, q_pos_offset=w.q_pos_offset, seg_q=sq, seg_kv=skv, out=out, lse=lse,
            workspace=ws, fp32_path=fp32_path)
    torch.cuda.synchronize(dev)
    free1, _ = torch.cuda.mem_get_info(dev)
    peak = torch.cuda.max_memory_allocated(dev) - io
    del q, k, v, out, lse, sq, skv, ws
    return int(peak), int(free0 - free1)


def memory_sweep(dev):
    """Peak device memory over inputs against L (causal; fp32 up to 60,926 tokens, bf16
    above; the fp32 tensor-core path at 60,926) and for the 1M-token packed configuration,
    beside the L x L score matrix of the math path (16 * L^2 * 4 bytes per batch entry)."""
    points = []

    def add(w, fp32_path="ffma", **extra):
        peak, delta = memory_point(w, dev, fp32_path)
        dt = "bf16" if w.dtype == torch.bfloat16 else ("f32_tc" if fp32_path == "tc" else "f32")
        io = w.io_bytes()
        points.append(dict({"L": w.Lq, "dtype": dt, "peak_bytes_over_inputs": peak,
                            "peak_over_io_ratio": peak / io, "io_bytes": io, "mem_get_info_delta_bytes": delta,
                            "math_path_score_matrix_bytes": 16 * w.Lq * w.Lk * 4}, **extra))

    for L in SWEEP_L:
        add(workloads.causal(L, torch.float32 if L <= 60_926 else torch.bfloat16))
    add(workloads.causal(60_926, torch.float32), fp32_path="tc")
    w = workloads.by_name("segmented_1M_bf16")
    add(w, segments=len(w.segments))
    causal_pts = [pt for pt in points if "segments" not in pt and pt["dtype"] != "f32_tc"]
    # linear fit of the causal points (bytes = a * L + b) and its largest residual
    n = len(causal_pts)
    xs = [pt["L"] for pt in causal_pts]
    ys = [pt["peak_bytes_over_inputs"] for pt in causal_pts]
    mx, my = sum(xs) / n, sum(ys) / n
    sxx = sum((x - mx) ** 2 for x in xs)
    a = sum((x - mx) * (y - my) for x, y in zip(xs, ys)) / sxx
    b = my - a * mx
    return {"unit": "bytes", "points": points,
            "max_over_inputs_bytes": max(pt["peak_bytes_over_inputs"] for pt in points),
            "L_range": [min(xs), max(xs)],
            "causal_linear_fit": {"bytes_per_token": a, "intercept_bytes": b,
                                  "max_residual_bytes": max(abs(y - (a * x + b)) for x, y in zip(xs, ys))},
            "quarter_score_matrix_per_head_bytes_at_max_L": max(xs) ** 2 * 4 // 4}


def run_memory_sweep(args, rank, local_rank):
    if rank != 0:
        return
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    print(json.dumps(dict({"metric": "peak device memory over inputs vs L"}, **memory_sweep(dev))), flush=True)


def _gpu_id(dev, local_rank):
    gpu_id = torch.cuda.get_device_properties(dev).uuid
    gpu_id = f"GPU-{gpu_id}" if gpu_id and not str(gpu_id).startswith("GPU-") else gpu_id
    return gpu_id if gpu_id else local_rank


def _timed_region(step, steps, warmup, stream, gpu_id, flush=None):
    """W warm-up calls, then K calls timed one by one with CUDA events while the SM
    clocks are sampled (`flush`, if any, runs between calls outside the events);
    returns (per-step ms, clock summary)."""
    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    with ClockSampler(gpu_id) as clocks:
        per = _time_steps(step, steps, stream, flush)
    return per, clocks.summary()


def _tensor_roofline(achieved, peaks, src, kernel, executed=None):
    """Roofline of a tensor-core kernel against both measured cuBLAS bf16 peaks."""
    burst = float(peaks["bf16_tflops"])
    sustained = float(peaks.get("bf16_tflops_sustained") or burst)
    roof = {"bound": "tensor", "achieved": achieved, "peak": burst, "unit": UNIT, "frac": achieved / burst,
            "peak_sustained": sustained, "frac_sustained": achieved / sustained,
            "reading": "frac against the burst peak (each call is one kernel timed alone); frac_sustained "
                       "against the seconds-long cuBLAS loop under the power cap, the closer match when "
                       "the clocks show sw_power_cap during the timed calls",
            "peak_source": f"{src} bf16_tflops / bf16_tflops_sustained (cuBLAS) of MEASURED_PEAKS.json",
            "kernel": kernel, "traffic": None}
    if executed is not None:
        roof["executed_tflops"] = executed
        roof["executed_frac"] = executed / burst
    return roof


def run_extras(args, dev, local_rank):
    """The rest of the metric, measured in the same process after the headline line's
    timing: the bf16 forward at L = 60,926 (the second dtype of the headline), the
    backward at L = 16,384 in both dtypes, and peak device memory over inputs against L."""
    peaks, src = _peaks()
    stream = torch.cuda.current_stream(dev)
    gpu_id = _gpu_id(dev, local_rank)
    ex = {}

    w = workloads.by_name("causal_60926_bf16")
    q, k, v, _, _ = _make_inputs(w, dev)
    out = torch.empty_like(q)
    lse = torch.empty((w.B, w.Hq, w.Lq), device=dev, dtype=torch.float32)
    ws = torch.empty(256, dtype=torch.uint8, device=dev)
    per, clk = _timed_region(lambda: gqa.fwd(q, k, v, out=out, lse=lse, workspace=ws, stream=stream), args.steps,
                             args.warmup, stream, gpu_id)
    assert gqa.status(ws) == 0, "device-side wait ran out"
    ms = statistics.mean(per)
    achieved = w.flops() / (ms * 1e-3) / 1e12
    roof = _tensor_roofline(achieved, peaks, src, "fwd_bf16_kernel")
    roof["traffic"] = _traffic("fwd_bf16_kernel", w.name)
    ex["bf16"] = {"workload": w.name, "value": achieved, "unit": UNIT, "ms_per_step": ms, "steps": args.steps,
                  "warmup": args.warmup, "algorithmic_tflop_per_step": w.flops() / 1e12, "roofline": roof,
                  "clocks": clk, "gpu_launches": args.steps,
                  "timed": "CUDA events around each forward call (attention kernel + a 256-byte status memset)"}
    del q, k, v, out, lse

    ex["bwd"] = {}
    for dtype, name in ((torch.bfloat16, "bf16"), (torch.float32, "f32")):
        w = workloads.causal(16_384, dtype)
        q, k, v, _, _ = _make_inputs(w, dev)
        out, lse = gqa.fwd(q, k, v, stream=stream)
        gen = torch.Generator(device=dev).manual_seed(inputs.SEED_V + 100)
        dout = torch.randn(q.shape, generator=gen, device=dev, dtype=torch.float32).to(dtype)
        dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
        bws = torch.empty(max(256, gqa.bwd_workspace_bytes(w.B, w.Hq, w.Hkv, w.Lq, w.Lk, w.d, dtype)),
                          dtype=torch.uint8, device=dev)
        scratch = torch.empty(512 << 20, dtype=torch.uint8, device=dev)

        def step():
            gqa.bwd(q, k, v, out, lse, dout, dq=dq, dk=dk, dv=dv, workspace=bws, stream=stream)

        # inputs below 4x the L2 here: a 512 MiB write evicts it between calls, outside the events
        steps = args.steps if dtype == torch.bfloat16 else max(1, min(args.steps, 5))
        per, clk = _timed_region(step, steps, min(args.warmup, 3) if dtype == torch.float32 else args.warmup,
                                 stream, gpu_id, flush=lambda: scratch.fill_(1))
        assert gqa.status(bws) == 0, "device-side wait ran out"
        ms = statistics.mean(per)
        flops = 2.5 * w.flops()
        achieved = flops / (ms * 1e-3) / 1e12
        if dtype == torch.bfloat16:
            roof = _tensor_roofline(achieved, peaks, src, "bwd_tc_kernel dV + dK + dQ (+ bwd_rowstate_kernel)",
                                    executed=achieved * 8 / 5)
            launches = 3
        else:
            sm_max = clk.get("sm_max_mhz") or peaks.get("sm_max_mhz", 1965.0)
            peak = _fp32_peak_tflops(SM_COUNT_B200, sm_max)
            roof = {"bound": "alu", "achieved": achieved, "peak": peak, "unit": UNIT, "frac": achieved / peak,
                    "traffic": None, "kernel": "bwd_dq_kernel + bwd_dkv_kernel (+ bwd_rowdot_kernel)",
                    "peak_source": f"derived: {SM_COUNT_B200} SMs x {FP32_LANES_PER_SM} FP32 lanes x 2 flop x "
                                   f"{sm_max:.0f} MHz (max SM clock)"}
            _with_ffma2_ceiling(roof, dev)
            launches = 3
        ex["bwd"][name] = {"workload": w.name, "value": achieved, "unit": UNIT, "ms_per_step": ms, "steps": steps,
                           "algorithmic_tflop_per_step": flops / 1e12, "roofline": roof, "clocks": clk,
                           "gpu_launches": launches * steps,
                           "timed": "CUDA events around each backward call (row-state + gradient kernels + "
                                    "a 256-byte status memset); L2 flushed between calls (512 MiB write "
                                    "outside the events)"}
        del q, k, v, out, lse, dout, dq, dk, dv, bws, scratch

    torch.cuda.empty_cache()
    ex["memory_sweep"] = memory_sweep(dev)
    return ex


# ----------------------------------------------------------------------------- one problem over N ranks
SHARD_DEFAULTS = {"heads": "causal_60926_f32", "ring": "causal_1M_bf16"}


def sharded_setup(mode, w, rank, world, device, *, layout="zigzag", group=None, gather=False, attention=None,
                  block=None, accumulator=None, dtype=None, backward=False, backward_fn=None, block_bwd=None):
    """This rank's share of ONE problem (workload ``w``) and the step that computes it.

    ``mode="heads"``: rank r holds the key/value heads ``heads.head_range(r, world,
    Hkv)`` and their query heads (no exchange; ``gather=True`` adds an all-gather of
    out / lse to the step).  ``mode="ring"``: rank r holds the sequence shard of
    ``layout`` (``ring.shard``) and the step is ``ring.ring_attention`` (key/value
    shards passed around the ring by point-to-point sends).  The inputs are the
    workload's seeded tensors, generated whole and cut, so every rank's share is a
    piece of the same problem.  ``attention`` (heads) and ``block`` / ``accumulator``
    (ring) replace the CUDA library's calls (CPU ranks in tests); ``dtype`` overrides
    the workload's.  Returns ``(step, shard)``: ``step()`` -> (out, lse) of this
    rank's share, ``shard`` = (q, k, v) of this rank.  With ``backward`` the forward
    runs once in the setup and ``step()`` is the backward of this rank's share ->
    (dq, dk, dv), from a seeded upstream gradient of the whole problem cut the same way
    (``backward_fn`` for heads, ``block_bwd`` for the ring replace the CUDA calls)."""
    from long_context_causal_flash_b200 import heads, ring

    dt = dtype or w.dtype
    gen_dev = device if (device.type == "cuda" and w.Lq * w.Hq * w.d > (1 << 28)) else "cpu"
    q, k, v = inputs.qkv(w.B, w.Hq, w.Hkv, w.Lq, w.Lk, w.d, dtype=dt, device=gen_dev)
    dout = None
    if backward:
        gen = torch.Generator(device=gen_dev).manual_seed(inputs.SEED_V + 100)
        dout = torch.randn(q.shape, generator=gen, device=gen_dev, dtype=torch.float32).to(dt)
    if w.segments or w.branches or w.q_pos_offset:
        raise SystemExit("the sharded modes take a causal self-attention workload")
    if mode == "heads":
        if gather and w.Hkv % world:
            raise SystemExit("--gather needs Hkv divisible by the number of ranks")
        qs, ks, vs = (x.to(device) for x in heads.shard_heads(q, k, v, rank, world))
        ds = None if dout is None else heads.shard_query_heads(dout, rank, world, w.Hkv).to(device)
        del q, k, v, dout

        def step():
            return heads.fwd_head_sharded(qs, ks, vs, group=group, gather=gather, attention=attention,
                                          presharded=True)
        if backward:  # this rank's own out / lse (not gathered) feed its backward
            out, lse = heads.fwd_head_sharded(qs, ks, vs, group=group, gather=False, attention=attention,
                                              presharded=True)

            def step():  # noqa: F811
                return heads.bwd_head_sharded(qs, ks, vs, out, lse, ds, group=group, gather=gather,
                                              backward=backward_fn, presharded=True)
    elif mode == "ring":
        n_chunks = world * len(ring.chunks_of(0, world, layout))
        if w.Lq % n_chunks:
            raise SystemExit(f"L = {w.Lq} does not split into {n_chunks} equal chunks")
        qs, ks, vs = (ring.shard(x, rank, world, layout).to(device) for x in (q, k, v))
        ds = None if dout is None else ring.shard(dout, rank, world, layout).to(device)
        del q, k, v, dout

        def step():
            return ring.ring_attention(qs, ks, vs, group=group, layout=layout, block=block, accumulator=accumulator)
        if backward:
            out, lse = step()

            def step():  # noqa: F811
                return ring.ring_attention_backward(qs, ks, vs, out, lse, ds, group=group, layout=layout,
                                                    block_bwd=block_bwd)
    else:
        raise SystemExit(f"unknown shard mode {mode}")
    return step, (qs, ks, vs)


def run_sharded(args, w, rank, world, local_rank):
    """Strong scaling: one problem split over the ranks (``--shard heads|ring``); the time
    of a step is the slowest rank's, and ``value`` is the whole problem's work over it."""
    import datetime

    import torch.distributed as dist

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
    os.environ.setdefault("MASTER_PORT", "29533")
    os.environ.setdefault("RANK", str(rank))
    os.environ.setdefault("WORLD_SIZE", str(world))
    dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    try:
        backward = args.pass_ == "bwd"
        step, _ = sharded_setup(args.shard, w, rank, world, dev, layout=args.layout, gather=args.gather,
                                backward=backward)
        flops = w.flops() * (2.5 if backward else 1.0)  # backward: 5 GEMMs of 2 d flops per visible pair
        stream = torch.cuda.current_stream(dev)
        for _ in range(args.warmup):
            step()
        torch.cuda.synchronize()
        dist.barrier()
        torch.cuda.synchronize()
        with ClockSampler(_gpu_id(dev, local_rank)) as clocks:
            per = _time_steps(step, args.steps, stream)
        dist.barrier()
        total_ms = _max_over_ranks(sum(per), dist, dev)
        if rank == 0:
            ms = total_ms / args.steps
            value = flops / (ms * 1e-3) / 1e12
            what = (f"key/value head groups x{world}" + (" + all-gather of out/lse" if args.gather else "")
                    if args.shard == "heads" else f"ring context parallelism x{world} ({args.layout})")
            line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
                    "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "strong",
                    "vs_baseline": None, "dtype": "f32" if w.dtype == torch.float32 else "bf16",
                    "data": "synthetic N(0,1), seeds 1/2/3",
                    "config": dict(_config(w, 1), parallelism=what, shard=args.shard,
                                   **({"pass": "backward"} if backward else {})),
                    "gpu_launches": None, "clocks": clocks.summary(),
                    "algorithmic_tflop_per_step": flops / 1e12,
                    "timed": "CUDA events around each step on every rank (its kernels and its NCCL calls), "
                             "max over ranks"}
            print(json.dumps(line), flush=True)
    finally:
        dist.destroy_process_group()


def run_ours(args, w, rank, world, local_rank):
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    dist = None
    if world > 1:
        import datetime

        import torch.distributed as dist

        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    torch.cuda.reset_peak_memory_stats(dev)
    base_alloc = torch.cuda.memory_allocated(dev)
    q, k, v, sq, skv = _make_inputs(w, dev, seed_offset=_seed_offset(rank))
    out = torch.empty_like(q)
    lse = torch.empty((w.B, w.Hq, w.Lq), device=dev, dtype=torch.float32)
    has_seg = sq is not None
    tc = args.fp32_path == "tc"
    if tc and w.dtype != torch.float32:
        raise SystemExit("--fp32-path tc needs an fp32 workload")
    code = gqa.GQA_F32_TC if tc else w.dtype
    splits = gqa.split_hint(w.B, w.Hq, w.Hkv, w.Lq, w.Lk, code, w.mask_kind, has_seg) if args.splits == "auto" \
        else int(args.splits)
    ws_bytes = max(256, gqa.split_workspace_bytes(w.B, w.Hq, w.Hkv, w.Lq, w.Lk, splits, w.d, code, w.mask_kind,
                                                  has_seg))
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    io_alloc = torch.cuda.memory_allocated(dev) - base_alloc

    def step():
        gqa.fwd(q, k, v, mask_kind=w.mask_kind, q_pos_offset=w.q_pos_offset, seg_q=sq, seg_kv=skv, out=out, lse=lse,
                workspace=ws, stream=stream, splits=splits, fp32_path=args.fp32_path)

    backward = args.pass_ == "bwd"
    if backward and tc:
        raise SystemExit("the backward has no tensor-core fp32 path")
    flops = w.flops() * (2.5 if backward else 1.0)  # backward: 5 GEMMs of 2 d flops per visible pair
    if backward:
        # The forward's out / lse are inputs of the timed backward; dout is seeded.
        step()
        gen = torch.Generator(device=dev).manual_seed(inputs.SEED_V + 100)
        dout = torch.randn(q.shape, generator=gen, device=dev, dtype=torch.float32).to(q.dtype)
        dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
        bws = torch.empty(max(256, gqa.bwd_workspace_bytes(w.B, w.Hq, w.Hkv, w.Lq, w.Lk, w.d, w.dtype, w.mask_kind,
                                                           has_seg)), dtype=torch.uint8, device=dev)
        # memory over inputs for the backward: its own workspace beyond q, k, v, out, lse,
        # dout and the gradients (the fp32 draw behind dout is gone before the peak reset)
        del gen
        torch.cuda.synchronize(dev)
        torch.cuda.reset_peak_memory_stats(dev)
        io_alloc = torch.cuda.memory_allocated(dev) - base_alloc - bws.numel()
        ws_bytes = bws.numel()

        def step():  # noqa: F811
            gqa.bwd(q, k, v, out, lse, dout, mask_kind=w.mask_kind, q_pos_offset=w.q_pos_offset, seg_q=sq,
                    seg_kv=skv, dq=dq, dk=dk, dv=dv, workspace=bws, stream=stream)

    status_ws = bws if backward else ws  # the timed call's status word
    # small inputs: evict L2 between steps (a 512 MiB write); the bench's buffer, not
    # the library's, so it is left out of the memory figures below
    flush, flush_bytes = None, 0
    if w.io_bytes() < 4 * 126e6:
        scratch = torch.empty(512 << 20, dtype=torch.uint8, device=dev)
        flush, flush_bytes = (lambda: scratch.fill_(1)), scratch.numel()
        flush()  # its kernel's first launch (lazy module loading) before the memory baseline
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    assert gqa.status(status_ws) == 0, "device-side wait ran out during warm-up"
    free_before, _ = torch.cuda.mem_get_info(dev)
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    gpu_id = torch.cuda.get_device_properties(dev).uuid
    gpu_id = f"GPU-{gpu_id}" if gpu_id and not str(gpu_id).startswith("GPU-") else gpu_id
    with ClockSampler(gpu_id if gpu_id else local_rank) as clocks:
        per_step = _time_steps(step, args.steps, stream, flush)
    if dist:
        dist.barrier()
    total_ms = sum(per_step)
    free_after, _ = torch.cuda.mem_get_info(dev)
    assert gqa.status(status_ws) == 0, "device-side wait ran out"
    peak_over_inputs = torch.cuda.max_memory_allocated(dev) - base_alloc - io_alloc + ws_bytes - flush_bytes
    total_ms = _max_over_ranks(total_ms, dist, dev)

    # end to end through the public host API: pinned host inputs -> device -> host results
    e2e = None
    if not args.no_e2e and not backward:
        hq, hk, hv = (x.cpu().pin_memory() for x in (q, k, v))
        hsq = None if sq is None else sq.cpu()
        hskv = None if skv is None else skv.cpu()
        hout = torch.empty(out.shape, dtype=out.dtype, pin_memory=True)
        hlse = torch.empty(lse.shape, dtype=lse.dtype, pin_memory=True)

        def host_step():
            gqa.fwd_host(hq, hk, hv, device=dev, mask_kind=w.mask_kind, q_pos_offset=w.q_pos_offset, seg_q=hsq,
                         seg_kv=hskv, out=hout, lse=hlse, stream=stream, fp32_path=args.fp32_path)

        host_step()
        e_steps = max(1, min(args.steps, 3))
        if dist:
            dist.barrier()
        torch.cuda.synchronize()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(e_steps):
            host_step()
        e1.record(stream)
        torch.cuda.synchronize()
        e_ms = e0.elapsed_time(e1) / e_steps
        e_ms = _max_over_ranks(e_ms, dist, dev)
        h2d = sum(x.numel() * x.element_size() for x in (hq, hk, hv)) + \
            (0 if hsq is None else (hsq.numel() + hskv.numel()) * 4)
        d2h = hout.numel() * hout.element_size() + hlse.numel() * 4
        e2e = {"value": flops * world / (e_ms * 1e-3) / 1e12, "unit": UNIT, "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h, "ms_per_step": e_ms}

    if rank != 0:
        if dist:
            dist.destroy_process_group()
        return
    ms_per_step = total_ms / args.steps
    value = flops * world / (ms_per_step * 1e-3) / 1e12
    per_launch_ms = statistics.mean(per_step)
    achieved = flops / (per_launch_ms * 1e-3) / 1e12
    peaks, src = _peaks()
    clk = clocks.summary()
    if tc:
        # fp32 on the tensor cores: three fp16 MMAs per product (hi*hi + hi*lo + lo*hi);
        # `achieved` counts the algorithmic fp32 work, `executed_tflops` the tensor work.
        peak = float(peaks["bf16_tflops"])
        roof = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": UNIT, "frac": achieved / peak,
                "traffic": None, "executed_tflops": 3 * achieved, "executed_frac": 3 * achieved / peak,
                "peak_source": f"{src} bf16_tflops (cuBLAS burst) of MEASURED_PEAKS.json; fp16 MMAs run at the "
                               "bf16 rate"}
    elif w.dtype == torch.float32:
        sm_max = clk.get("sm_max_mhz") or peaks.get("sm_max_mhz", 1965.0)
        peak = _fp32_peak_tflops(SM_COUNT_B200, sm_max)
        roof = {"bound": "alu", "achieved": achieved, "peak": peak, "unit": UNIT, "frac": achieved / peak,
                "traffic": None,
                "peak_source": f"derived: {SM_COUNT_B200} SMs x {FP32_LANES_PER_SM} FP32 lanes x 2 flop x "
                               f"{sm_max:.0f} MHz (max SM clock)"}
    else:
        peak = float(peaks["bf16_tflops"])
        roof = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": UNIT, "frac": achieved / peak,
                "traffic": None, "peak_source": f"{src} bf16_tflops (cuBLAS burst) of MEASURED_PEAKS.json"}
    roof["kernel"] = ("fwd_f32_tc_kernel" if tc else "fwd_f32_kernel") if w.dtype == torch.float32 \
        else "fwd_bf16_kernel"
    roof["traffic"] = _traffic(roof["kernel"], w.name)
    if w.dtype == torch.float32 and not tc:
        _with_ffma2_ceiling(roof, dev)
    if backward and w.dtype == torch.float32:
        roof["kernel"] = "bwd_dq_kernel + bwd_dkv_kernel (+ bwd_rowdot_kernel)"
        roof["traffic"] = None
    elif backward:
        # The three tensor-core kernels execute 8 GEMM-equivalents per visible block (S
        # and dP twice, S once more for dV); `achieved` counts the algorithmic 5.
        roof["kernel"] = "bwd_tc_kernel dV + dK + dQ (+ bwd_rowstate_kernel)"
        roof["traffic"] = None
        roof["executed_tflops"] = achieved * 8 / 5
    roof["timed"] = ("CUDA events around each forward call (attention kernel + a 256-byte status memset"
                     + (", operand-split kernels and their memset" if tc else "")
                     + (", plan kernels" if has_seg else "") + (", merge kernel" if splits > 1 else "") + ")")
    if backward:
        roof["timed"] = ("CUDA events around each backward call (row-state, " +
                         ("dQ and dK/dV" if w.dtype == torch.float32 else "dV, dK and dQ") +
                         " kernels + a 256-byte status memset" + (", plan kernels" if has_seg else "") + ")")
    n_bwd = 3 if w.dtype == torch.float32 else 4  # fp32: row dot, dQ, dK+dV; bf16: row state, dV, dK, dQ
    kernels_per_step = (n_bwd if backward else 1 + (1 if splits > 1 else 0) + (2 if tc else 0)) + \
        (2 if sq is not None else 0)
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f32" if w.dtype == torch.float32 else "bf16", "data": "synthetic N(0,1), seeds 1/2/3 (+10/rank)",
        "config": dict(_config(w, world), splits=splits, **({"pass": "backward"} if backward else {}),
                       **({"fp32_path": "tc: per-head scaled two-term fp16 split, 3 tcgen05 MMAs per product, "
                                        "fp32 accumulation"} if tc else {})),
        "roofline": roof, "e2e": e2e, "gpu_launches": kernels_per_step * args.steps,
        "tiles": _tile_summary(w, code, sq, skv, dev) if not backward else None,
        "clocks": clk, "peak_gib_over_inputs": peak_over_inputs / 2 ** 30,
        "mem_get_info_delta_bytes": int(free_before - free_after),
        "math_path_score_matrix_gib": 16 * w.Lq * w.Lk * 4 / 2 ** 30,
        "algorithmic_tflop_per_step": flops / 1e12,
    }
    if world == 1 and not args.no_extras and not backward and w.name == "causal_60926_f32" and not tc:
        line.update(run_extras(args, dev, local_rank))
    if world == 1 and not args.no_cpu_baseline and not backward:
        qc, kc, vc, sqc, skvc = _cpu_inputs(w) if w.Lq * w.Hq * w.d <= (1 << 28) else (None,) * 5
        if qc is not None:
            f, t, n = _oracle_sample(w, args.cpu_seconds, qc, kc, vc, sqc, skvc)
            line["cpu_baseline"] = {"value": f / t / 1e12, "unit": UNIT, "cores": _blas_threads(), "kind": "oracle",
                                    "sample": f"{n} seeded sampled query rows x {w.Hq} heads of {w.name}, "
                                              f"{t:.1f} s of fp64 numpy on the host"}
    print(json.dumps(line), flush=True)
    if dist:
        dist.destroy_process_group()


def run_fp32_probe(local_rank):
    """One JSON line: the rate of each operand form of the register-only FMA probe, with
    the SM clocks sampled while it runs."""
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    forms = {0: "packed (q_r, q_r+1) x (k, k), runs sharing the duplicated k",
             1: "packed (q_r, q_r+1) x (k, k), runs sharing the (q_r, q_r+1) pair: the kernels' order",
             2: "packed, no duplicated operand", 3: "scalar fma.rn.f32"}
    _ffma2_ceiling(dev, 1)  # first launches of the process outside the sampled region
    _FFMA2_CEILING.clear()
    with ClockSampler(_gpu_id(dev, local_rank)) as clocks:
        time.sleep(0.3)  # the sampler's first line
        rates = {str(f): _ffma2_ceiling(dev, f) for f in forms}
        time.sleep(0.3)
    nominal = _fp32_peak_tflops(SM_COUNT_B200, clocks.summary().get("sm_max_mhz") or 1965.0)
    print(json.dumps({"fp32_probe": {f: {"form": forms[int(f)], "value": v, "unit": UNIT, "frac_of_nominal": v / nominal}
                                     for f, v in rates.items()},
                      "nominal_fp32_tflops": nominal, "clocks": clocks.summary()}), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default="causal_60926_f32")
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--shard", choices=["heads", "ring"], default=None,
                    help="strong scaling: split ONE problem over the ranks by key/value head group or by "
                         "sequence (ring); default workloads causal_60926_f32 / causal_1M_bf16")
    ap.add_argument("--layout", choices=["contiguous", "zigzag"], default="zigzag",
                    help="ring shard layout (--shard ring)")
    ap.add_argument("--gather", action="store_true", help="--shard heads: all-gather out / lse in each step")
    ap.add_argument("--no-extras", action="store_true",
                    help="skip the bf16 / backward / memory-sweep sub-objects of the default line")
    ap.add_argument("--splits", default="auto", help="key splits: 'auto' (the library's hint) or a count")
    ap.add_argument("--memory-sweep", action="store_true",
                    help="print peak device memory over inputs against L instead of timing")
    ap.add_argument("--fp32-path", dest="fp32_path", choices=["ffma", "tc"], default="ffma",
                    help="fp32 workloads: the FFMA kernel (default) or the tensor cores on split operands")
    ap.add_argument("--pass", dest="pass_", choices=["fwd", "bwd"], default="fwd",
                    help="time the forward (default) or the backward from the forward's out / lse")
    ap.add_argument("--fp32-probe", action="store_true",
                    help="print the register-only FMA rate of each probe operand form instead of timing")
    args = ap.parse_args()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus and "RANK" in os.environ:
        print(f"warning: --gpus {args.gpus} but WORLD_SIZE {world}", file=sys.stderr)
    if args.shard and args.workload == ap.get_default("workload"):
        args.workload = SHARD_DEFAULTS[args.shard]
    w = _workload(args.workload)
    if args.shard and args.impl == "ours":
        run_sharded(args, w, rank, world, local_rank)
    elif args.memory_sweep:
        run_memory_sweep(args, rank, local_rank)
    elif args.fp32_probe:
        run_fp32_probe(local_rank)
    elif args.impl == "reference":
        run_reference(args, w, rank, world)
    else:
        run_ours(args, w, rank, world, local_rank)


if __name__ == "__main__":
    main()
