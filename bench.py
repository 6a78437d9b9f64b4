"""Benchmark of the BPT layer forward on B200: tokens/s and TFLOP/s.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

One step is one whole layer forward (QKV projection, blockwise attention over
every query block, output projection, residuals and FFN) over one batch of
synthetic inputs already resident in HBM. N > 1 runs under torchrun, one rank
per GPU: every rank runs its own sequence(s) (independent units, no collective
on the data path); the timed region is bracketed by a barrier and a device
sync on every rank and the reported time is the max over ranks.

--impl reference times the fp64 CPU oracle (a deliberately slow program) on a
bounded sample of the same workload, on the host cores, rank 0 only.
"""

from __future__ import annotations

import argparse
import json
import math
import os
import re
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import bpt_inputs as bi  # noqa: E402

METRIC = "BPT layer fwd tokens/s and TFLOP/s (% BF16 peak) on 1 B200, vs fp64 oracle"
DEFAULT_WORKLOAD = "gpt7b_s32768_h4096"
L2_BYTES = 126 * 1024 * 1024


# ---------------------------------------------------------------------------
# work accounting (matmul flops; causal attention counted as half)
# ---------------------------------------------------------------------------

def layer_flops(shape: bi.LayerShape) -> dict:
    b, s, h = shape.b, shape.s, shape.h
    tok = b * s
    att = 4.0 * b * s * s * h * (0.5 if shape.causal else 1.0)
    return {
        "gemm_qkv": 2.0 * tok * h * 3 * h,
        "attention": att,
        "gemm_outproj": 2.0 * tok * h * h,
        "gemm_ffn_up": 2.0 * tok * h * 4 * h,
        "gemm_ffn_down": 2.0 * tok * 4 * h * h,
    }


def profiled_traffic(workload: str, kernel: str):
    """DRAM bytes per launch of the dominant kernel from the committed ncu
    summary, or None when there is none for this workload or the kernel's
    source changed since the counters were taken."""
    if kernel != "attention":
        return None
    import hashlib
    path = os.path.join(ROOT, "profiles", "attention_s16384_h2048_causal.md")
    if not os.path.exists(path):
        return None
    text = open(path).read()
    m_t = re.search(rf"traffic_per_launch_{re.escape(workload)}_bytes: (\d+)", text)
    m_h = re.search(r"kernel_source_sha256_16: ([0-9a-f]+)", text)
    if not (m_t and m_h):
        return None
    h = hashlib.sha256()
    for f in ("attention.cuh", "ptx.cuh"):
        with open(os.path.join(ROOT, "blockwise_attn_ffn_bpt_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return int(m_t.group(1)) if h.hexdigest()[:16] == m_h.group(1) else None


def measured_peaks() -> tuple[dict, str]:
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            return json.load(f), "measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


# ---------------------------------------------------------------------------
# distributed plumbing
# ---------------------------------------------------------------------------

def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def init_dist(backend: str, world: int):
    import datetime

    import torch.distributed as dist
    if world > 1 and not dist.is_initialized():
        dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=120))
    return dist if world > 1 else None


def barrier(dist, device=None):
    if dist is not None:
        if device is not None and dist.get_backend() == "nccl":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


def max_over_ranks(value: float, dist, device=None) -> float:
    """Max of a float over all ranks (every rank takes this step)."""
    if dist is None:
        return value
    import torch
    t = torch.tensor([value], dtype=torch.float64,
                     device=device if (device is not None and dist.get_backend() == "nccl") else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def rank_seed(rank: int) -> int:
    """Each rank draws its own sequence(s): independent units of work."""
    return rank


def whole_job_throughput(tokens_per_rank: int, steps: int, world: int, ms_max: float) -> float:
    """Tokens/s of the whole job: every rank's tokens over the slowest rank's time."""
    return tokens_per_rank * steps * world / (ms_max / 1e3)


# ---------------------------------------------------------------------------
# clocks
# ---------------------------------------------------------------------------

class ClockSampler:
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(prefix="bpt_clocks_", suffix=".csv")
        os.close(fd)
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.QUERY}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=self.f, stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.f.close()

    def summary(self) -> dict:
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        try:
            for line in open(self.path):
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm.append(float(parts[1]))
                    mx = float(parts[2])
                except ValueError:
                    continue
                for n, v in zip(names, parts[5:9]):
                    if v.lower() == "active":
                        reasons.add(n)
            os.unlink(self.path)
        except OSError:
            pass
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"]}
        return {"sm_mhz": float(np.median(sm)), "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------------------
# CPU baseline: the oracle on a bounded sample
# ---------------------------------------------------------------------------

def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        info = threadpool_info()
        if info:
            return int(max(i.get("num_threads", 1) for i in info))
    except Exception:
        pass
    return os.cpu_count() or 1


def oracle_sample(shape: bi.LayerShape, inp: dict, budget_s: float = 10.0, max_rows: int | None = None):
    """Time the oracle on the first n rows of sequence 0 (n doubled until the
    budget is spent). Returns (tokens/s, rows, seconds)."""
    import oracle
    args = bi.oracle_args(inp)
    n = 64
    cap = min(shape.s, max_rows or shape.s)
    best = None
    while True:
        rows = np.arange(min(n, cap), dtype=np.int64)
        t0 = time.perf_counter()
        oracle.layer_rows(*args, heads=shape.heads, causal=shape.causal, rows=rows)
        dt = time.perf_counter() - t0
        best = (rows.size / dt, int(rows.size), dt)
        if dt >= budget_s or rows.size >= cap:
            return best
        n = min(cap, max(n * 2, int(n * budget_s / max(dt, 1e-3) * 0.6)))


def reference_arm(args, shape, name):
    world, rank, _ = dist_env()
    if rank != 0:
        return 0
    inp = bi.make_inputs(shape, seed=0)
    per_step = []
    for _ in range(args.warmup):
        oracle_sample(shape, inp, budget_s=2.0, max_rows=256)
    for _ in range(args.steps):
        per_step.append(oracle_sample(shape, inp, budget_s=args.ref_budget))
    tps = float(np.mean([p[0] for p in per_step]))
    rows = per_step[-1][1]
    secs = float(sum(p[2] for p in per_step))
    cores = blas_threads()
    sample = (f"oracle rows t=0..{rows - 1} of sequence 0 (their keys/values projected), fp64 numpy/BLAS; "
              f"early causal rows attend to short prefixes, so this favours the CPU")
    line = {
        "impl": "reference", "metric": METRIC, "value": tps, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": secs / max(1, args.steps) * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded N(0,1) x, N(0,1/fan_in) weights, N(0,0.02^2) biases)",
        "config": config_of(shape, name),
        "cpu_baseline": {"value": tps, "unit": "tokens/s", "cores": cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": tps, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line))
    return 0


def config_of(shape: bi.LayerShape, name: str) -> dict:
    return {"workload": name, "batch": shape.b, "seq_len": shape.s, "d_model": shape.h, "heads": shape.heads,
            "head_dim": shape.dh, "ffn_hidden": shape.f, "causal": shape.causal, "q_block": shape.q_block,
            "kv_block": shape.kv_block, "input_dtype": shape.dtype,
            "l2": "inputs larger than L2 (x, K/V and weights each exceed 126 MB)"
            if shape.b * shape.s * shape.h * 2 > L2_BYTES else "L2 flushed between steps",
            "parallelism": "independent sequences per GPU"}


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------

def our_arm(args, shape, name):
    import torch

    import blockwise_attn_ffn_bpt_b200 as bpt

    world, rank, local = dist_env()
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    dist = init_dist("nccl", world)

    inp = bi.make_inputs(shape, seed=rank_seed(rank))
    x = bi.to_torch(inp["x"], device)
    params = {k: bi.to_torch(inp[k], device) for k in bi.PARAM_NAMES}
    out = torch.empty((shape.b, shape.s, shape.h), dtype=torch.float32, device=device)
    dtype_code = bpt.BPT_DTYPE_F32 if shape.dtype == "f32" else bpt.BPT_DTYPE_BF16
    ws_bytes = bpt.workspace_bytes(dtype_code, shape.b, shape.s, shape.h, shape.heads, shape.q_block,
                                   shape.kv_block)
    flush = None
    if shape.b * shape.s * shape.h * 2 <= L2_BYTES:
        flush = torch.empty(2 * L2_BYTES // 4, dtype=torch.float32, device=device)
    stream = torch.cuda.current_stream(device)

    def step():
        if flush is not None:
            flush.zero_()
        bpt.layer_forward(x, params, shape.heads, shape.q_block, shape.kv_block, shape.causal, out=out,
                          stream=stream)

    # device memory the library takes (its pool keeps the workspace between
    # calls): free memory before the first call minus free memory after warm-up
    torch.cuda.synchronize(device)
    free_pre, _ = torch.cuda.mem_get_info(device)
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(device)
    if bpt.device_status() != 0:
        raise RuntimeError("device error during warm-up")
    free_post, _ = torch.cuda.mem_get_info(device)

    # ---- timed region (device time, CUDA events on the launching stream)
    torch.cuda.reset_peak_memory_stats(device)
    mem0 = torch.cuda.memory_allocated(device)
    free0, _ = torch.cuda.mem_get_info(device)
    bpt.set_kernel_timing(True)
    bpt.kernel_times()
    launches0 = bpt.launch_count()
    ev0 = torch.cuda.Event(enable_timing=True)
    ev1 = torch.cuda.Event(enable_timing=True)
    with ClockSampler(device.index if "CUDA_VISIBLE_DEVICES" not in os.environ else
                      int(os.environ["CUDA_VISIBLE_DEVICES"].split(",")[local])) as clocks:
        barrier(dist, device)
        torch.cuda.synchronize(device)
        ev0.record(stream)
        for _ in range(args.steps):
            step()
        ev1.record(stream)
        torch.cuda.synchronize(device)
        barrier(dist, device)
    launches = bpt.launch_count() - launches0
    ktimes = bpt.kernel_times()
    bpt.set_kernel_timing(False)
    if bpt.device_status() != 0:
        raise RuntimeError("device error during the timed region")
    ms = ev0.elapsed_time(ev1)
    ms_max = max_over_ranks(ms, dist, device)

    # ---- end to end through the C ABI's host-memory entry (bpt_layer_forward_host):
    # every step copies its input from pinned host memory and its result back;
    # the library overlaps step i's copies with the compute of steps i -/+ 1
    x_host = torch.empty(x.shape, dtype=x.dtype, pin_memory=True)
    x_host.copy_(x)
    out_host = torch.empty(out.shape, dtype=torch.float32, pin_memory=True)
    torch.cuda.synchronize(device)
    bpt.layer_forward_host(x_host, params, shape.heads, shape.q_block, shape.kv_block, shape.causal,
                           out_host=out_host, n_inputs=max(1, args.warmup // 2), stream=stream)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    barrier(dist, device)
    torch.cuda.synchronize(device)
    e2e_steps = max(1, args.steps)
    e0.record(stream)
    bpt.layer_forward_host(x_host, params, shape.heads, shape.q_block, shape.kv_block, shape.causal,
                           out_host=out_host, n_inputs=e2e_steps, stream=stream)
    e1.record(stream)
    torch.cuda.synchronize(device)
    barrier(dist, device)
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), dist, device)

    peak_bytes = torch.cuda.max_memory_allocated(device) - mem0

    # ---- CPU baseline (rank 0, N = 1 only)
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        tps, rows, secs = oracle_sample(shape, inp, budget_s=args.ref_budget)
        cpu = {"value": tps, "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle",
               "sample": f"first {rows} rows of sequence 0 with their keys/values, fp64 numpy/BLAS, {secs:.1f} s"}

    if dist is not None:
        barrier(dist, device)
    if rank != 0:
        if dist is not None:
            dist.destroy_process_group()
        return 0

    tokens = shape.b * shape.s
    flops = layer_flops(shape)
    total_flops = sum(flops.values())
    value = whole_job_throughput(tokens, args.steps, world, ms_max)
    tflops = total_flops * args.steps * world / (ms_max / 1e3) / 1e12
    peaks, peak_src = measured_peaks()
    peak = peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"])

    # dominant kernel: largest share of the timed kernel time
    dom = max(ktimes.items(), key=lambda kv: kv[1][1]) if ktimes else None
    roof = None
    if dom is not None:
        kname, (nl, kms) = dom
        kflops = flops.get(kname, 0.0) * args.steps
        achieved = kflops / (kms / 1e3) / 1e12 if kms > 0 else 0.0
        roof = {"bound": "tensor", "kernel": kname, "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                "frac": achieved / peak, "traffic": profiled_traffic(name, kname), "launches": nl,
                "avg_launch_ms": kms / nl,
                "peak_source": f"{peak_src} bf16_tflops_sustained (kernel timed inside a long step)"}
    kernel_table = {k: {"launches": n, "ms": t, "share": t / sum(v[1] for v in ktimes.values())}
                    for k, (n, t) in ktimes.items()}

    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_max / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded N(0,1) x, N(0,1/fan_in) weights, N(0,0.02^2) biases; random-init layer)",
        "config": config_of(shape, name),
        "tflops": tflops, "frac_of_bf16_peak": tflops / peak,
        "roofline": roof,
        "cpu_baseline": cpu,
        "e2e": {"value": tokens * e2e_steps * world / (e2e_ms / 1e3), "unit": "tokens/s",
                "h2d_bytes_per_step": int(x.numel() * x.element_size()),
                "d2h_bytes_per_step": int(out.numel() * out.element_size()),
                "steps": e2e_steps, "api": "bpt_layer_forward_host (pinned host buffers)"},
        "gpu_launches": int(launches),
        "kernels": kernel_table,
        "clocks": clocks.summary(),
        "memory": {"workspace_bytes": ws_bytes, "ratio_bytes_vs_2bsh": ws_bytes / (2 * tokens * shape.h),
                   "ratio_elems_vs_2bsh": ws_bytes / 2 / (2 * tokens * shape.h),
                   "peak_torch_alloc_bytes_in_step": int(peak_bytes),
                   "device_bytes_taken_by_library": int(free_pre - free_post),
                   "free_bytes_before": int(free0)},
    }
    print(json.dumps(line))
    if dist is not None:
        dist.destroy_process_group()
    return 0


def largest_fitting(need, budget: int, unit: int) -> int:
    """The largest multiple n * unit (n >= 1) with need(n * unit) <= budget, for
    a need that grows with its argument; unit when even that does not fit."""
    lo, hi = 1, 2
    while need(hi * unit) <= budget:
        lo, hi = hi, hi * 2
    while hi - lo > 1:
        mid = (lo + hi) // 2
        lo, hi = (mid, hi) if need(mid * unit) <= budget else (lo, mid)
    return lo * unit


def max_context_arm(args):
    """The longest single sequence one 7B-class BPT layer forward (h 4096, 32
    heads, causal, q_block 1024, kv_block 2048) fits on this GPU, measured by
    running it: the budget is the free device memory minus the weights and a
    margin, the need per length is x (bf16) + out (fp32) + the library's exact
    workspace. Inputs are seeded synthetic tensors drawn on the device; the
    first rows are checked against the oracle (a causal row depends only on
    its prefix)."""
    import torch
    import blockwise_attn_ffn_bpt_b200 as bpt
    import oracle

    h, heads, qb, kvb = 4096, 32, 1024, 2048
    device = torch.device("cuda", 0)
    torch.cuda.set_device(device)
    g = torch.Generator(device=device).manual_seed(0)
    std = {"Wqkv": 1 / math.sqrt(h), "Wo": 1 / math.sqrt(h), "W1": 1 / math.sqrt(h), "W2": 1 / math.sqrt(4 * h)}
    shapes = {"Wqkv": (h, 3 * h), "bqkv": (3 * h,), "Wo": (h, h), "bo": (h,), "W1": (h, 4 * h), "b1": (4 * h,),
              "W2": (4 * h, h), "b2": (h,)}
    params = {k: (torch.randn(shp, generator=g, device=device) * std.get(k, 0.02)).to(torch.bfloat16)
              for k, shp in shapes.items()}
    # load the kernels and the library's pool on a short prefix first
    warm = torch.randn((1, 8192, h), generator=g, device=device).to(torch.bfloat16)
    bpt.layer_forward(warm, params, heads, qb, kvb, True)
    del warm
    torch.cuda.synchronize(device)
    torch.cuda.empty_cache()
    free, total = torch.cuda.mem_get_info(device)
    margin = 3 << 30  # input generation chunks, the library's own allocations, fragmentation

    def need(s):
        return s * h * 2 + s * h * 4 + bpt.workspace_bytes(0, 1, s, h, heads, qb, kvb)

    s = largest_fitting(need, free - margin, kvb)
    x = torch.empty((1, s, h), dtype=torch.bfloat16, device=device)
    chunk = 1 << 16
    for r0 in range(0, s, chunk):
        r1 = min(s, r0 + chunk)
        x[0, r0:r1] = torch.randn((r1 - r0, h), generator=g, device=device).to(torch.bfloat16)
    out = torch.empty((1, s, h), dtype=torch.float32, device=device)
    torch.cuda.synchronize(device)
    torch.cuda.empty_cache()
    free_before, _ = torch.cuda.mem_get_info(device)
    stream = torch.cuda.current_stream(device)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(0 if "CUDA_VISIBLE_DEVICES" not in os.environ else
                      int(os.environ["CUDA_VISIBLE_DEVICES"].split(",")[0])) as clocks:
        ev0.record(stream)
        bpt.layer_forward(x, params, heads, qb, kvb, True, out=out, stream=stream)
        ev1.record(stream)
        torch.cuda.synchronize(device)
    ms = ev0.elapsed_time(ev1)
    free_after, _ = torch.cuda.mem_get_info(device)
    status = bpt.device_status()
    # oracle check of the first rows, and finiteness of rows spread over the sequence
    R = 256
    p64 = {k: v.float().cpu().numpy().astype(np.float64) for k, v in params.items()}
    x0 = x[0, :R].float().cpu().numpy().astype(np.float64)[None]
    ref = oracle.layer_rows(x0, *(p64[k] for k in bi.PARAM_NAMES), heads=heads, causal=True, rows=np.arange(R))
    got = out[0, :R].cpu().numpy().astype(np.float64)
    d = got - ref
    spread = torch.linspace(0, s - 1, 64, device=device).long()
    finite = bool(torch.isfinite(out[0, spread]).all().item())
    shape = bi.LayerShape(1, s, h, heads, qb, kvb, True)
    flops = sum(layer_flops(shape).values())
    ws = bpt.workspace_bytes(0, 1, s, h, heads, qb, kvb)
    line = {
        "metric": "longest single sequence of one 7B-class BPT layer forward on one GPU",
        "value": s, "unit": "tokens", "n_gpus": 1, "dtype": "bf16", "data": "synthetic (seeded on the device)",
        "config": {"workload": "max_context_h4096", "d_model": h, "heads": heads, "q_block": qb, "kv_block": kvb,
                   "causal": True, "ffn_hidden": 4 * h},
        "ms": ms, "tokens_per_s": s / (ms / 1e3), "tflops": flops / (ms / 1e3) / 1e12,
        "memory": {"device_total_bytes": total, "free_before_bytes": free_before, "free_after_bytes": free_after,
                   "x_bytes": s * h * 2, "out_bytes": s * h * 4, "workspace_bytes": ws,
                   "workspace_vs_2bsh_elements": ws / (2 * s * h * 2)},
        "parity_first_rows": {"rows": R, "max_abs": float(np.abs(d).max()),
                              "rel_l2": float(np.linalg.norm(d) / np.linalg.norm(ref))},
        "finite_at_64_spread_rows": finite, "device_status": status,
        "clocks": clocks.summary(),
    }
    print(json.dumps(line))
    return 0 if (status == 0 and finite) else 1


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD,
                    help="one of: " + ", ".join(list(bi.WORKLOADS) + ["sweep_<block>_<causal|noncausal>"]))
    ap.add_argument("--ref-budget", type=float, default=10.0, help="seconds of oracle work per sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--max-context", action="store_true",
                    help="instead: the longest sequence one 7B-class layer forward fits on the GPU, run once")
    args = ap.parse_args(argv)
    if args.max_context:
        return max_context_arm(args)
    if args.warmup < 3 and args.impl == "ours":
        print("warning: fewer than 3 warm-up steps", file=sys.stderr)
    name = args.workload
    if name.startswith("sweep_"):
        _, blk, c = name.split("_")
        shape = bi.sweep_shape(int(blk), c == "causal")
    else:
        shape = bi.WORKLOADS[name]
    world, _, _ = dist_env()
    if world != args.gpus:
        print(f"note: --gpus {args.gpus} but WORLD_SIZE={world}; using WORLD_SIZE", file=sys.stderr)
    if args.impl == "reference":
        return reference_arm(args, shape, name)
    return our_arm(args, shape, name)


if __name__ == "__main__":
    sys.exit(main())
