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
# wave_rows values of the library's FFN-side schedules (BPT_WAVE_* in include/bpt.h)
FFN_SCHEDULES = {"default": 0, "chained": -1, "waves": -2, "mega": -3}
L2_BYTES = 126 * 1024 * 1024


# ---------------------------------------------------------------------------
# work accounting (matmul flops; causal attention counted as half)
# ---------------------------------------------------------------------------

def layer_flops(shape: bi.LayerShape) -> dict:
    """Matmul flops of one forward per kernel name of the library's timing log
    (ffn_chain runs the three FFN-side GEMMs in one launch)."""
    b, s, h, f = shape.b, shape.s, shape.h, shape.f
    tok = b * s
    att = 4.0 * b * s * s * h * (0.5 if shape.causal else 1.0)
    return {
        "gemm_qkv": 2.0 * tok * h * 3 * h,
        "attention": att,
        "gemm_outproj": 2.0 * tok * h * h,
        "gemm_ffn_up": 2.0 * tok * h * f,
        "gemm_ffn_down": 2.0 * tok * f * h,
    }


def kernel_flops(shape: bi.LayerShape) -> dict:
    f = layer_flops(shape)
    f["ffn_chain"] = f["gemm_outproj"] + f["gemm_ffn_up"] + f["gemm_ffn_down"]
    f["layer_mega"] = f["attention"] + f["ffn_chain"]  # attention and the FFN side in one launch
    return f


TRAFFIC_FILE = os.path.join(ROOT, "profiles", "attention_traffic.json")


def kernel_source_hash(files=("attention.cuh", "ptx.cuh")) -> str:
    import hashlib
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, "blockwise_attn_ffn_bpt_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def profiled_traffic(workload: str, kernel: str, path: str = TRAFFIC_FILE):
    """DRAM bytes per launch of the dominant kernel, from the data file written
    beside its ncu summary; None when there is none for this workload or the
    kernel's source changed since the counters were taken."""
    if kernel != "attention" or not os.path.exists(path):
        return None
    with open(path) as f:
        d = json.load(f)
    if d.get("kernel_source_sha256_16") != kernel_source_hash():
        return None
    v = d.get("traffic_per_launch_bytes", {}).get(workload)
    return int(v) if v is not None else None


FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                  "bf16_tflops_sustained_sm_mhz": 1300.0}


def measured_peaks() -> tuple[dict, str]:
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            return json.load(f), "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def sustained_clock_mhz(peaks: dict):
    """SM clock (MHz) at which the sustained bf16 peak was taken: a key of the
    peaks record that names both 'sustain' and a clock, else the fallback's."""
    stack = [peaks]
    while stack:
        d = stack.pop()
        for k, v in d.items():
            if isinstance(v, dict):
                stack.append(v)
            elif isinstance(v, (int, float)) and "sustain" in k.lower() and ("mhz" in k.lower() or "clock" in k.lower()):
                return float(v)
    return FALLBACK_PEAKS["bf16_tflops_sustained_sm_mhz"]


def tensor_roofline(kernel: str, achieved: float, peaks: dict, src: str, sm_mhz, traffic) -> dict:
    """Roofline object of a tensor-core kernel timed with CUDA events.

    frac is against the burst bf16 peak (the denominator of a kernel that runs
    at full clock, as this one does inside a step of tens of ms); the
    sustained peak, scaled from the clock it was taken at to the clock sampled
    during this run, is reported beside it."""
    burst = float(peaks["bf16_tflops"])
    sus = float(peaks.get("bf16_tflops_sustained", burst))
    sus_mhz = sustained_clock_mhz(peaks)
    scaled = sus * (sm_mhz / sus_mhz) if sm_mhz else None
    return {"bound": "tensor", "kernel": kernel, "achieved": achieved, "peak": burst, "unit": "TFLOP/s",
            "frac": achieved / burst, "traffic": traffic,
            "peak_source": f"{src} bf16_tflops (burst, cuBLAS bf16 GEMM timed alone)",
            "peak_sustained_at_sampled_clock": scaled,
            "frac_vs_sustained_at_sampled_clock": (achieved / scaled) if scaled else None,
            "sustained_peak_note": f"{src} bf16_tflops_sustained {sus} taken at {sus_mhz:.0f} MHz, scaled by the "
                                   f"median SM clock sampled in this run ({sm_mhz} MHz)"}


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
    """SM clock and clock-event reasons during a timed region: read every 20 ms
    through NVML (read-only queries) in a thread, only while the region runs;
    nvidia-smi at its 200 ms interval where NVML is not available."""

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    REASON_BITS = {"sw_power_cap": 0x4, "hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40}
    PERIOD_S = 0.02

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None
        self.nvml = None
        self.samples = []  # (sm MHz, reasons bitmask)
        self.watts = []    # board power draw, where NVML reports it
        self.max_mhz = None
        self.limit_w = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.handle = pynvml.nvmlDeviceGetHandleByIndex(gpu_index)
            self.max_mhz = float(pynvml.nvmlDeviceGetMaxClockInfo(self.handle, pynvml.NVML_CLOCK_SM))
            self.nvml = pynvml
        except Exception:
            self.nvml = None
        if self.nvml is not None:
            try:  # read-only: the limit the power cap enforces, in mW
                self.limit_w = float(self.nvml.nvmlDeviceGetEnforcedPowerLimit(self.handle)) / 1000.0
            except Exception:
                self.limit_w = None

    def _reasons(self):
        nv = self.nvml
        get = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or nv.nvmlDeviceGetCurrentClocksThrottleReasons
        return int(get(self.handle))

    def _instant_watts(self):
        # the instantaneous board power (NVML field POWER_INSTANT, mW): the
        # plain power query averages over about a second, longer than the
        # timed region, so it is not used
        nv = self.nvml
        try:
            v = nv.nvmlDeviceGetFieldValues(self.handle, [nv.NVML_FI_DEV_POWER_INSTANT])[0]
            if v.nvmlReturn != 0:
                return None
            kinds = {0: "dVal", 1: "uiVal", 2: "ulVal", 3: "ullVal", 4: "sllVal", 5: "siVal"}
            return float(getattr(v.value, kinds[int(v.valueType)])) / 1000.0
        except Exception:
            return None

    def _run(self):
        nv = self.nvml
        while not self.stop.is_set():
            try:
                self.samples.append((float(nv.nvmlDeviceGetClockInfo(self.handle, nv.NVML_CLOCK_SM)), self._reasons()))
            except Exception:
                pass
            w = self._instant_watts()
            if w is not None:
                self.watts.append(w)
            self.stop.wait(self.PERIOD_S)

    def __enter__(self):
        if self.nvml is not None:
            import threading
            self.stop = threading.Event()
            self.thread = threading.Thread(target=self._run, daemon=True)
            self.thread.start()
            return self
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
        if self.nvml is not None:
            self.stop.set()
            self.thread.join(timeout=5)
            try:
                self.nvml.nvmlShutdown()
            except Exception:
                pass
            return
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.f.close()

    def summary(self) -> dict:
        if self.nvml is not None:
            if not self.samples:
                return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unavailable"]}
            reasons = sorted(n for n, bit in self.REASON_BITS.items() if any(r & bit for _, r in self.samples))
            out = {"sm_mhz": float(np.median([c for c, _ in self.samples])), "sm_max_mhz": self.max_mhz,
                   "reasons": reasons, "samples": len(self.samples), "source": "NVML every 20 ms in the timed region"}
            if self.watts:
                out["power_w"] = float(np.median(self.watts))
                out["power_source"] = "NVML instantaneous board power, median of the samples"

            if self.limit_w is not None:
                out["power_limit_w"] = self.limit_w
            return out
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
        return {"sm_mhz": float(np.median(sm)), "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sm),
                "source": "nvidia-smi every 200 ms"}


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


def spread_rows(s: int, n: int, offset: int = 0) -> np.ndarray:
    """n query positions spread evenly over [0, s), the last one always s - 1
    (so the oracle projects the keys/values of the whole sequence)."""
    n = max(1, min(n, s))
    idx = (np.arange(n, dtype=np.int64) * s) // n + (offset % max(1, s // n))
    idx = np.minimum(idx, s - 1)
    idx[-1] = s - 1
    return np.unique(idx)


class OracleTimer:
    """Time of the fp64 oracle on one whole layer forward of a workload,
    extrapolated from rows spread over the sequence.

    The oracle's row function (layer_rows) costs a fixed part, the key/value
    projection of the visible prefix (the whole sequence once the last row is
    asked for), plus a part per row (its query projection, its scores against
    every projected key with the invisible ones masked, the output projection
    and the FFN), as its plain whole-sequence forward does. A calibration call
    on the last row alone (after one untimed warm-up call) gives fixed + one
    row; a call on n rows spread evenly over the sequence gives fixed + n rows;
    the whole forward of one sequence is then fixed + s rows, and b sequences
    take b times that."""

    def __init__(self, shape: bi.LayerShape, inp: dict):
        import oracle
        self.oracle = oracle
        self.shape = shape
        self.args = bi.oracle_args(inp)
        last = np.array([shape.s - 1], dtype=np.int64)
        self._time(last)  # warm-up: BLAS threads, page faults of the fp64 copies
        self.t_one = self._time(last)

    def _time(self, rows: np.ndarray) -> float:
        t0 = time.perf_counter()
        self.oracle.layer_rows(*self.args, heads=self.shape.heads, causal=self.shape.causal, rows=rows)
        return time.perf_counter() - t0

    # host memory the oracle's score matrices of one call may take: it holds,
    # per head and worker thread, a few fp64 arrays of (rows x visible keys)
    MEM_BUDGET = 4 << 30

    def max_rows(self) -> int:
        threads = max(1, min(self.shape.heads, os.cpu_count() or 1))
        per_row = self.shape.s * 8 * 4 * threads
        return int(max(2, min(self.shape.s, self.MEM_BUDGET // per_row)))

    def rows_for_budget(self, budget_s: float) -> int:
        """How many spread rows take about budget_s beyond the fixed part
        (never more than the memory bound allows)."""
        probe = spread_rows(self.shape.s, min(64, self.max_rows()))
        per_row = max((self._time(probe) - self.t_one) / max(1, probe.size - 1), 1e-6)
        return int(max(2, min(self.max_rows(), budget_s / per_row)))

    def sample(self, n: int, offset: int = 0):
        """(tokens/s of the whole forward, rows timed, seconds spent, est. seconds of one forward)."""
        s = self.shape.s
        rows = spread_rows(s, min(n, self.max_rows()), offset)
        t_n = self._time(rows)
        if rows.size >= s:
            t_seq = t_n
        else:
            per_row = max(t_n - self.t_one, 0.0) / max(1, rows.size - 1)
            t_seq = self.t_one + (s - 1) * per_row
        t_full = self.shape.b * t_seq
        return self.shape.b * s / t_full, int(rows.size), t_n, t_full


def sample_text(timer: OracleTimer, rows: int) -> str:
    s = timer.shape.s
    return (f"fp64 numpy/BLAS oracle (layer_rows) on {rows} query rows spread evenly over sequence 0 (s={s}, "
            f"incl. row {s - 1}, so the whole key/value projection), after a calibration call on row {s - 1} "
            f"alone ({timer.t_one:.2f} s); the whole forward of all {timer.shape.b} sequence(s) is extrapolated "
            f"as b * (fixed + s * per-row)")


def reference_arm(args, shape, name):
    world, rank, _ = dist_env()
    if rank != 0:
        return 0
    inp = bi.make_inputs(shape, seed=0)
    # warm-up: the oracle on a short prefix (its threads and BLAS come up)
    for _ in range(args.warmup):
        import oracle
        oracle.layer_rows(*bi.oracle_args(inp), heads=shape.heads, causal=shape.causal,
                          rows=np.arange(min(shape.s, 64), dtype=np.int64))
    timer = OracleTimer(shape, inp)
    n = timer.rows_for_budget(args.ref_budget)
    per_step = [timer.sample(n, offset=i) for i in range(args.steps)]
    tps = float(np.mean([p[0] for p in per_step]))
    secs = float(sum(p[2] for p in per_step))
    cores = blas_threads()
    line = {
        "impl": "reference", "metric": METRIC, "value": tps, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": float(np.mean([p[3] for p in per_step])) * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded N(0,1) x, N(0,1/fan_in) weights, N(0,0.02^2) biases)",
        "config": config_of(shape, name),
        "cpu_baseline": {"value": tps, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                         "sample": sample_text(timer, per_step[-1][1]) + f"; {secs:.1f} s timed over the steps"},
        "e2e": {"value": tps, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line))
    return 0


def config_of(shape: bi.LayerShape, name: str) -> dict:
    return {"workload": name, "batch": shape.b, "seq_len": shape.s, "d_model": shape.h, "heads": shape.heads,
            "head_dim": shape.dh, "ffn_hidden": shape.f, "causal": shape.causal, "q_block": shape.q_block,
            "kv_block": shape.kv_block, "input_dtype": shape.dtype,
            "block_sizes": "q_block sets the FFN wave (a whole number of query blocks); kv_block is validated but "
                           "does not change the GPU schedule (attention tiles keys by 128)",
            "l2": "inputs larger than L2 (x, K/V and weights each exceed 126 MB)"
            if shape.b * shape.s * shape.h * 2 > L2_BYTES else
            "L2 flushed between steps (a 252 MB write, outside each step's event pair)",
            "parallelism": "independent sequences per GPU"}


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------

class Layer:
    """Device-resident inputs of one workload and the call that runs it."""

    def __init__(self, shape: bi.LayerShape, seed: int, device, inp: dict | None = None, wave_rows: int = 0):
        import torch
        import blockwise_attn_ffn_bpt_b200 as bpt
        self.bpt = bpt
        self.shape = shape
        self.wave_rows = wave_rows
        self.inp = inp if inp is not None else bi.make_inputs(shape, seed=seed)
        self.x = bi.to_torch(self.inp["x"], device)
        self.params = {k: bi.to_torch(self.inp[k], device) for k in bi.PARAM_NAMES}
        self.out = torch.empty((shape.b, shape.s, shape.h), dtype=torch.float32, device=device)
        self.flush = None
        if shape.b * shape.s * shape.h * 2 <= L2_BYTES:
            self.flush = torch.empty(2 * L2_BYTES // 4, dtype=torch.float32, device=device)

    def run(self, stream):
        sh = self.shape
        self.bpt.layer_forward(self.x, self.params, sh.heads, sh.q_block, sh.kv_block, sh.causal, out=self.out,
                               wave_rows=self.wave_rows, stream=stream)

    def timed_steps(self, steps: int, stream) -> float:
        """Device milliseconds of `steps` layer forwards: each forward between
        its own pair of CUDA events on the launching stream (an L2 flush, when
        the inputs fit in L2, runs between the pairs and is not counted)."""
        import torch
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
        for e0, e1 in evs:
            if self.flush is not None:
                self.flush.zero_()
            e0.record(stream)
            self.run(stream)
            e1.record(stream)
        torch.cuda.synchronize(stream.device)
        return float(sum(e0.elapsed_time(e1) for e0, e1 in evs))


def gpu_index(local: int) -> int:
    if "CUDA_VISIBLE_DEVICES" in os.environ:
        return int(os.environ["CUDA_VISIBLE_DEVICES"].split(",")[local])
    return local


def kernel_split(layer: Layer, steps: int, stream) -> dict:
    """Per-kernel device time over `steps` forwards, in a pass of its own with
    the library's per-launch CUDA-event log on (never the headline pass)."""
    bpt = layer.bpt
    bpt.set_kernel_timing(True)
    bpt.kernel_times()
    for _ in range(steps):
        if layer.flush is not None:
            layer.flush.zero_()
        layer.run(stream)
    kt = bpt.kernel_times()
    bpt.set_kernel_timing(False)
    return kt


def measure(args, shape: bi.LayerShape, name: str, layer: Layer, device, dist, steps: int) -> dict:
    """Headline timing of one workload: warm-up, then `steps` forwards timed
    with the kernel log off, barrier + sync on both sides, max over ranks;
    clocks sampled during the timed region; then the per-kernel split in a
    second pass."""
    import torch
    bpt = layer.bpt
    world, rank, local = dist_env()
    stream = torch.cuda.current_stream(device)
    for _ in range(args.warmup):
        layer.run(stream)
    if bpt.stream_status(stream) != 0:
        raise RuntimeError("device error during warm-up")
    launches0 = bpt.launch_count()
    with ClockSampler(gpu_index(local)) as clocks:
        barrier(dist, device)
        torch.cuda.synchronize(device)
        ms = layer.timed_steps(steps, stream)
        torch.cuda.synchronize(device)
        barrier(dist, device)
    launches = bpt.launch_count() - launches0
    if bpt.stream_status(stream) != 0:
        raise RuntimeError("device error during the timed region")
    ms_max = max_over_ranks(ms, dist, device)
    ksteps = max(1, min(steps, 10))
    ktimes = kernel_split(layer, ksteps, stream)
    if bpt.stream_status(stream) != 0:
        raise RuntimeError("device error during the kernel-split pass")
    flops = layer_flops(shape)
    kflops = kernel_flops(shape)
    clk = clocks.summary()
    peaks, src = measured_peaks()
    tokens = shape.b * shape.s
    value = whole_job_throughput(tokens, steps, world, ms_max)
    tflops = sum(flops.values()) * steps * world / (ms_max / 1e3) / 1e12
    total_k = sum(v[1] for v in ktimes.values()) or 1.0
    kernels = {}
    for k, (n, t) in ktimes.items():
        kf = kflops.get(k, 0.0) * ksteps
        kernels[k] = {"launches": n, "ms": t, "share": t / total_k, "avg_launch_ms": t / n,
                      "tflops": (kf / (t / 1e3) / 1e12) if (kf and t > 0) else None}
    roof = None
    if ktimes:
        kname = max(ktimes.items(), key=lambda kv: kv[1][1])[0]
        kn, kms = ktimes[kname]
        achieved = kflops.get(kname, 0.0) * ksteps / (kms / 1e3) / 1e12 if kms > 0 else 0.0
        roof = tensor_roofline(kname, achieved, peaks, src, clk.get("sm_mhz"), profiled_traffic(name, kname))
        roof.update({"launches": kn, "avg_launch_ms": kms / kn,
                     "timing": f"per-launch CUDA events on the launching stream, in a separate pass of {ksteps} "
                               f"forwards after the headline pass"})
    return {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": steps,
        "warmup": args.warmup, "ms_per_step": ms_max / steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16" if shape.dtype == "bf16" else "f32-in/bf16-mma",
        "data": "synthetic (seeded N(0,1) x, N(0,1/fan_in) weights, N(0,0.02^2) biases; random-init layer)",
        "config": dict(config_of(shape, name), ffn_schedule=args.ffn),
        "tflops": tflops, "frac_of_bf16_peak": tflops / float(peaks["bf16_tflops"]),
        "peak_source": f"{src} bf16_tflops (burst)",
        "roofline": roof,
        "gpu_launches": int(launches),
        "kernels": kernels,
        "kernels_pass": f"separate pass of {ksteps} forwards with per-launch CUDA events",
        "clocks": clk,
    }


def our_arm(args, shape, name):
    import torch

    world, rank, local = dist_env()
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    dist = init_dist("nccl", world)
    layer = Layer(shape, rank_seed(rank), device, wave_rows=FFN_SCHEDULES[args.ffn])
    bpt = layer.bpt
    dtype_code = bpt.BPT_DTYPE_F32 if shape.dtype == "f32" else bpt.BPT_DTYPE_BF16
    ws_bytes = bpt.workspace_bytes(dtype_code, shape.b, shape.s, shape.h, shape.heads, shape.q_block,
                                   shape.kv_block)
    stream = torch.cuda.current_stream(device)

    # device memory the library takes (its pool keeps the workspace between
    # calls): free memory before the first call minus free memory after it
    torch.cuda.synchronize(device)
    free_pre, _ = torch.cuda.mem_get_info(device)
    layer.run(stream)
    torch.cuda.synchronize(device)
    free_post, _ = torch.cuda.mem_get_info(device)
    torch.cuda.reset_peak_memory_stats(device)
    mem0 = torch.cuda.memory_allocated(device)

    line = measure(args, shape, name, layer, device, dist, args.steps)
    peak_bytes = torch.cuda.max_memory_allocated(device) - mem0

    # ---- end to end through the C ABI's host-memory entry (bpt_layer_forward_host):
    # every step copies its input from pinned host memory and its result back;
    # the library overlaps step i's copies with the compute of steps i -/+ 1
    x, out = layer.x, layer.out
    x_host = torch.empty(x.shape, dtype=x.dtype, pin_memory=True)
    x_host.copy_(x)
    out_host = torch.empty(out.shape, dtype=torch.float32, pin_memory=True)
    torch.cuda.synchronize(device)
    bpt.layer_forward_host(x_host, layer.params, shape.heads, shape.q_block, shape.kv_block, shape.causal,
                           out_host=out_host, n_inputs=max(1, args.warmup // 2), stream=stream)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    barrier(dist, device)
    torch.cuda.synchronize(device)
    e2e_steps = max(1, args.steps)
    e0.record(stream)
    bpt.layer_forward_host(x_host, layer.params, shape.heads, shape.q_block, shape.kv_block, shape.causal,
                           out_host=out_host, n_inputs=e2e_steps, stream=stream)
    e1.record(stream)
    torch.cuda.synchronize(device)
    barrier(dist, device)
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), dist, device)
    if bpt.stream_status(stream) != 0:
        raise RuntimeError("device error during the end-to-end pass")

    # ---- CPU baseline (rank 0, N = 1 only): the oracle as it stands
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        timer = OracleTimer(shape, layer.inp)
        n = timer.rows_for_budget(args.ref_budget)
        tps, rows, secs, _ = timer.sample(n)
        cpu = {"value": tps, "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle",
               "sample": sample_text(timer, rows) + f"; {secs:.1f} s for the spread rows"}

    if dist is not None:
        barrier(dist, device)
    if rank != 0:
        if dist is not None:
            dist.destroy_process_group()
        return 0

    tokens = shape.b * shape.s
    line["cpu_baseline"] = cpu
    line["e2e"] = {"value": tokens * e2e_steps * world / (e2e_ms / 1e3), "unit": "tokens/s",
                   "h2d_bytes_per_step": int(x.numel() * x.element_size()),
                   "d2h_bytes_per_step": int(out.numel() * out.element_size()),
                   "steps": e2e_steps, "api": "bpt_layer_forward_host (pinned host buffers)"}
    two_bsh_bytes = 2 * tokens * shape.h
    line["memory"] = {
        "workspace_bytes": ws_bytes, "ratio_bytes_vs_2bsh": ws_bytes / two_bsh_bytes,
        "ratio_elems_vs_2bsh": ws_bytes / 2 / two_bsh_bytes,
        "reading": "target: 2bsh read as elements (<= 1.5x); read as bf16 bytes the bound is not met (2.0x), "
                   "which is inherent to materialising K and V (Algorithm 1 step 1: 4bsh bytes)",
        "peak_torch_alloc_bytes_in_step": int(peak_bytes),
        "device_bytes_taken_by_library": int(free_pre - free_post),
    }
    print(json.dumps(line))
    if dist is not None:
        dist.destroy_process_group()
    return 0


def all_configs_arm(args):
    """One JSON line per configuration of the layer's workloads (the four
    fixed workloads and every point of the block-size sweep, causal and not):
    device time, tokens/s, TFLOP/s, fraction of the bf16 peak, kernel split,
    SM clock. One GPU; no e2e or CPU legs."""
    import torch
    device = torch.device("cuda", 0)
    torch.cuda.set_device(device)
    names = list(bi.WORKLOADS) + [f"sweep_{blk}_{c}" for c in ("causal", "noncausal") for blk in bi.SWEEP_BLOCKS]
    if args.only:
        names = [n for n in names if any(o in n for o in args.only.split(","))]
    cache = {}
    for name in names:
        shape = shape_of(name)
        key = ("sweep", shape.causal) if name.startswith("sweep_") else name
        if key not in cache:
            cache.clear()
            cache[key] = bi.make_inputs(shape, seed=0)
        layer = Layer(shape, 0, device, inp=cache[key], wave_rows=FFN_SCHEDULES[args.ffn])
        steps = args.steps if shape.s * shape.b >= 32768 else max(args.steps, 20)
        line = measure(args, shape, name, layer, device, None, steps)
        line["cpu_baseline"] = None
        line["e2e"] = None
        print(json.dumps(line), flush=True)
        del layer
        torch.cuda.empty_cache()
    return 0


def shape_of(name: str) -> bi.LayerShape:
    if name.startswith("sweep_"):
        _, blk, c = name.split("_")
        return bi.sweep_shape(int(blk), c == "causal")
    return bi.WORKLOADS[name]


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
    status = bpt.stream_status(stream)
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


def ffn_backward_arm(args):
    """Throughput of the FFN block's backward (bpt_ffn_backward) at the 7B-class
    layer's shapes (rows 32768, h 4096, ffn 16384; 16384-row chunks): five
    products of 2 rows h ffn flops each (the recomputed intermediate, da,
    dhid, dW1, dW2). Seeded synthetic inputs drawn on the device."""
    import torch
    import blockwise_attn_ffn_bpt_b200 as bpt
    rows, h, f = 32768, 4096, 16384
    device = torch.device("cuda", 0)
    torch.cuda.set_device(device)
    g = torch.Generator(device=device).manual_seed(0)
    hid = torch.randn((rows, h), generator=g, device=device)
    dy = torch.randn((rows, h), generator=g, device=device)
    W1 = (torch.randn((h, f), generator=g, device=device) / math.sqrt(h)).to(torch.bfloat16)
    b1 = (torch.randn(f, generator=g, device=device) * 0.02).to(torch.bfloat16)
    W2 = (torch.randn((f, h), generator=g, device=device) / math.sqrt(f)).to(torch.bfloat16)
    stream = torch.cuda.current_stream(device)
    for _ in range(args.warmup):
        bpt.ffn_backward(hid, W1, b1, W2, dy, stream=stream)
    torch.cuda.synchronize(device)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    with ClockSampler(gpu_index(0)) as clocks:
        for e0, e1 in evs:
            e0.record(stream)
            bpt.ffn_backward(hid, W1, b1, W2, dy, stream=stream)
            e1.record(stream)
        torch.cuda.synchronize(device)
    status = bpt.stream_status(stream)
    ms = float(np.mean([e0.elapsed_time(e1) for e0, e1 in evs]))
    flops = 5 * 2.0 * rows * h * f
    peaks, src = measured_peaks()
    line = {"metric": "FFN block backward (bpt_ffn_backward) TFLOP/s on 1 B200", "value": flops / (ms / 1e3) / 1e12,
            "unit": "TFLOP/s", "ms": ms, "steps": args.steps, "warmup": args.warmup, "dtype": "bf16",
            "config": {"workload": "ffn_backward_rows32768_h4096_f16384", "chunk_rows": 16384},
            "frac_of_bf16_peak": flops / (ms / 1e3) / 1e12 / float(peaks["bf16_tflops"]),
            "peak_source": f"{src} bf16_tflops (burst)", "device_status": status, "clocks": clocks.summary(),
            "data": "synthetic (torch generator on the device)"}
    print(json.dumps(line))
    return 0 if status == 0 else 1


def layer_backward_flops(shape: bi.LayerShape) -> dict:
    """Matmul flops of one layer backward (bpt_layer_backward) per kernel name:
    the forward it recomputes (projection, attention, out-projection), the FFN
    block's five products, the out-projection's two, the attention backward's
    five s x s products (S, dP, dV, dK, dQ; causal counted as half) and the
    projection's two."""
    b, s, h, f = shape.b, shape.s, shape.h, shape.f
    tok = b * s
    half = 0.5 if shape.causal else 1.0
    return {
        "forward recompute": 2.0 * tok * h * 3 * h + 4.0 * b * s * s * h * half + 2.0 * tok * h * h,
        "ffn backward": 5 * 2.0 * tok * h * f,
        "out-projection backward": 2 * 2.0 * tok * h * h,
        "attention_bwd": 5 * 2.0 * b * s * s * h * half,
        "projection backward": 2 * 2.0 * tok * h * 3 * h,
    }


def layer_backward_arm(args):
    """Throughput of the whole layer's backward (bpt_layer_backward) on one
    workload: the recomputed forward, the FFN block, the out-projection, the
    attention backward kernel and the projection, one call per step; then the
    per-kernel split in a pass of its own. Seeded synthetic inputs drawn on the
    device (x and dy N(0, 1), weights N(0, 1/fan_in), biases N(0, 0.02^2))."""
    import torch
    import blockwise_attn_ffn_bpt_b200 as bpt
    shape = shape_of(args.workload)
    b, s, h, f, heads = shape.b, shape.s, shape.h, shape.f, shape.heads
    device = torch.device("cuda", 0)
    torch.cuda.set_device(device)
    g = torch.Generator(device=device).manual_seed(0)
    x = torch.randn((b, s, h), generator=g, device=device).to(torch.bfloat16)
    dy = torch.randn((b, s, h), generator=g, device=device)
    params = {}
    for name, shp in bi.tensor_shapes(shape).items():
        if name != "x":
            params[name] = (torch.randn(shp, generator=g, device=device) * bi.tensor_std(name, shape)).to(
                torch.bfloat16)
    stream = torch.cuda.current_stream(device)
    for _ in range(args.warmup):
        bpt.layer_backward(x, params, dy, heads, shape.causal, stream=stream)
    torch.cuda.synchronize(device)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    with ClockSampler(gpu_index(0)) as clocks:
        for e0, e1 in evs:
            e0.record(stream)
            bpt.layer_backward(x, params, dy, heads, shape.causal, stream=stream)
            e1.record(stream)
        torch.cuda.synchronize(device)
    status = bpt.stream_status(stream)
    ms = float(np.mean([e0.elapsed_time(e1) for e0, e1 in evs]))
    fl = layer_backward_flops(shape)
    total = sum(fl.values())
    # per-kernel split, in a pass of its own with the launch log on
    bpt.set_kernel_timing(True)
    bpt.kernel_times()
    for _ in range(args.steps):
        bpt.layer_backward(x, params, dy, heads, shape.causal, stream=stream)
    kt = bpt.kernel_times()
    bpt.set_kernel_timing(False)
    kernels = {}
    split_total = sum(ms_ for _, ms_ in kt.values()) or 1.0
    for name, (n_, ms_) in sorted(kt.items(), key=lambda kv: -kv[1][1]):
        kernels[name] = {"launches": n_, "ms_per_step": ms_ / args.steps, "share": ms_ / split_total}
    att = kt.get("attention_bwd")
    att_tflops = fl["attention_bwd"] / (att[1] / args.steps / 1e3) / 1e12 if att else None
    # the same backward from the forward's saved O and statistics (bpt_layer_forward_save once, untimed):
    # no attention recomputation
    _, o_sv, lse_sv = bpt.layer_forward_save(x, params, heads, shape.q_block, shape.kv_block, shape.causal,
                                             stream=stream)
    for _ in range(args.warmup):
        bpt.layer_backward(x, params, dy, heads, shape.causal, stream=stream, saved=(o_sv, lse_sv))
    torch.cuda.synchronize(device)
    evs2 = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    for e0, e1 in evs2:
        e0.record(stream)
        bpt.layer_backward(x, params, dy, heads, shape.causal, stream=stream, saved=(o_sv, lse_sv))
        e1.record(stream)
    torch.cuda.synchronize(device)
    status = status or bpt.stream_status(stream)
    ms_sv = float(np.mean([e0.elapsed_time(e1) for e0, e1 in evs2]))
    total_sv = total - 4.0 * b * s * s * h * (0.5 if shape.causal else 1.0)
    saved = {"ms_per_step": ms_sv, "tokens_per_s": b * s / (ms_sv / 1e3), "tflops": total_sv / (ms_sv / 1e3) / 1e12,
             "api": "bpt_layer_forward_save, then bpt_layer_backward_saved (the attention is not recomputed)"}
    peaks, src = measured_peaks()
    line = {"metric": "BPT layer backward (bpt_layer_backward) tokens/s and TFLOP/s on 1 B200",
            "value": b * s / (ms / 1e3), "unit": "tokens/s", "ms_per_step": ms, "tflops": total / (ms / 1e3) / 1e12,
            "frac_of_bf16_peak": total / (ms / 1e3) / 1e12 / float(peaks["bf16_tflops"]),
            "peak_source": f"{src} bf16_tflops (burst)", "steps": args.steps, "warmup": args.warmup,
            "dtype": "bf16", "config": config_of(shape, args.workload),
            "flops_per_step": fl, "attention_bwd_tflops": att_tflops, "kernels": kernels,
            "from_saved_forward": saved,
            "device_status": status, "clocks": clocks.summary(),
            "data": "synthetic (torch generator on the device)"}
    print(json.dumps(line))
    return 0 if status == 0 else 1


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD,
                    help="one of: " + ", ".join(list(bi.WORKLOADS) + ["sweep_<block>_<causal|noncausal>"]))
    ap.add_argument("--ref-budget", type=float, default=4.0, help="seconds of oracle work per sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--max-context", action="store_true",
                    help="instead: the longest sequence one 7B-class layer forward fits on the GPU, run once")
    ap.add_argument("--all-configs", action="store_true",
                    help="instead: one line per workload and block-size sweep point (one GPU)")
    ap.add_argument("--only", default="", help="with --all-configs: comma-separated name fragments to keep")
    ap.add_argument("--ffn", choices=list(FFN_SCHEDULES), default="default",
                    help="FFN-side schedule: the library's default, one chained launch, or per-GEMM waves")
    ap.add_argument("--ffn-backward", action="store_true",
                    help="instead: throughput of the FFN block's backward at the 7B-class layer's shapes")
    ap.add_argument("--layer-backward", action="store_true",
                    help="instead: throughput of the whole layer's backward on --workload")
    args = ap.parse_args(argv)
    if args.max_context:
        return max_context_arm(args)
    if args.ffn_backward:
        return ffn_backward_arm(args)
    if args.layer_backward:
        return layer_backward_arm(args)
    if args.warmup < 3 and args.impl == "ours":
        print("warning: fewer than 3 warm-up steps", file=sys.stderr)
    if args.all_configs:
        return all_configs_arm(args)
    name = args.workload
    shape = shape_of(name)
    world, _, _ = dist_env()
    if world != args.gpus:
        print(f"note: --gpus {args.gpus} but WORLD_SIZE={world}; using WORLD_SIZE", file=sys.stderr)
    if args.impl == "reference":
        return reference_arm(args, shape, name)
    return our_arm(args, shape, name)


if __name__ == "__main__":
    sys.exit(main())
