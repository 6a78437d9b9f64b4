"""Host-side logic of bench.py without a GPU: the multi-rank plumbing on gloo
(world size 2), the whole-job throughput formula, and the reference arm (the
fp64 oracle on a bounded sample) on the CPU."""

import json
import os
import subprocess
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    dist = bench.init_dist("gloo", world)
    try:
        w, r, _ = bench.dist_env()
        bench.barrier(dist)
        # each rank "measured" a different time; the job time is the slowest rank's
        ms = 10.0 + 5.0 * r
        ms_max = bench.max_over_ranks(ms, dist)
        q.put((r, w, ms_max, bench.rank_seed(r)))
        bench.barrier(dist)
    finally:
        dist.destroy_process_group()


def test_two_ranks_agree_on_the_slowest_time_and_draw_different_data():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29500 + (os.getpid() % 1000)
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    assert [r[0] for r in res] == [0, 1]
    assert all(r[1] == 2 for r in res)
    assert all(r[2] == 15.0 for r in res)           # max over ranks, seen by every rank
    assert res[0][3] != res[1][3]                    # independent sequences per rank


def test_single_rank_needs_no_process_group():
    assert bench.init_dist("gloo", 1) is None
    assert bench.max_over_ranks(3.5, None) == 3.5


def test_whole_job_throughput_is_weak_scaling():
    one = bench.whole_job_throughput(32768, 10, 1, 200.0)
    assert one == pytest.approx(32768 * 10 / 0.2)
    # N ranks with the same per-rank time do N times the work
    assert bench.whole_job_throughput(32768, 10, 4, 200.0) == pytest.approx(4 * one)


def test_layer_flops_counts_causal_attention_as_half():
    import bpt_inputs as bi
    f = bench.layer_flops(bi.WORKLOADS["gpt7b_s32768_h4096"])
    assert sum(f.values()) == pytest.approx(2.1990e13, rel=1e-3)
    nc = bench.layer_flops(bi.sweep_shape(1024, False))
    assert sum(nc.values()) == pytest.approx(3.8483e12, rel=1e-3)


def run_bench(args, env=None):
    e = dict(os.environ)
    e.update(env or {})
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], capture_output=True, text=True,
                       env=e, timeout=600)
    return r


def test_reference_arm_prints_one_json_line():
    r = run_bench(["--impl", "reference", "--workload", "small_fp32_s256_h256", "--steps", "1", "--warmup", "0",
                   "--ref-budget", "0.5"])
    assert r.returncode == 0, r.stderr
    lines = [l for l in r.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["unit"] == "tokens/s" and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0
    assert d["config"]["workload"] == "small_fp32_s256_h256"


def test_reference_arm_runs_on_rank_zero_only():
    r = run_bench(["--impl", "reference", "--workload", "small_fp32_s256_h256", "--steps", "1", "--warmup", "0"],
                  env={"RANK": "1", "WORLD_SIZE": "2", "LOCAL_RANK": "1"})
    assert r.returncode == 0
    assert r.stdout.strip() == ""


@pytest.mark.parametrize("unit", [1, 7, 2048])
def test_largest_fitting_length_is_the_largest_that_fits(unit):
    # need grows with the length, like the layer's bytes (x + out + workspace)
    def need(s):
        return 10 * s + (s // 3) * 2 + 1000

    for budget in (1000, 1010 + 10 * unit, 5_000, 123_457, 10_000_000):
        s = bench.largest_fitting(need, budget, unit)
        assert s % unit == 0 and s >= unit
        if need(unit) <= budget:
            assert need(s) <= budget < need(s + unit)
        else:
            assert s == unit  # nothing fits: the smallest length is reported


def test_spread_rows_cover_the_sequence_and_end_on_its_last_row():
    for s, n in [(256, 8), (32768, 100), (1000, 1), (64, 500), (5, 3)]:
        r = bench.spread_rows(s, n)
        assert r[-1] == s - 1 and r.min() >= 0 and np.all(np.diff(r) > 0)
        assert r.size == min(n, s) or r.size == min(n, s) - 1  # the last slot moved onto s - 1
        if n < s:
            # evenly spread: the mean position is near the middle, so causal
            # rows average a prefix of about s/2
            assert abs(r.mean() - (s - 1) / 2) <= s / n + 1


def test_oracle_timer_extrapolates_a_whole_forward():
    import bpt_inputs as bi
    shape = bi.LayerShape(2, 128, 128, 2, 64, 64, True)
    inp = bi.make_inputs(shape, seed=0)
    timer = bench.OracleTimer(shape, inp)
    assert timer.t_one > 0
    tps, rows, secs, t_full = timer.sample(16)
    assert rows == 16 and secs > 0 and t_full > 0
    assert tps == pytest.approx(shape.b * shape.s / t_full)
    # asking for every row times the whole sequence directly
    assert timer.max_rows() == shape.s  # a tiny problem is never memory-bound
    tps_all, rows_all, secs_all, t_all = timer.sample(10_000)
    assert rows_all == shape.s and t_all == pytest.approx(shape.b * secs_all)


def test_traffic_comes_from_the_data_file_only_while_the_source_matches(tmp_path):
    p = tmp_path / "traffic.json"
    good = {"kernel_source_sha256_16": bench.kernel_source_hash(), "traffic_per_launch_bytes": {"w": 123}}
    p.write_text(json.dumps(good))
    assert bench.profiled_traffic("w", "attention", str(p)) == 123
    assert bench.profiled_traffic("other", "attention", str(p)) is None
    assert bench.profiled_traffic("w", "gemm_qkv", str(p)) is None
    p.write_text(json.dumps(dict(good, kernel_source_sha256_16="0" * 16)))
    assert bench.profiled_traffic("w", "attention", str(p)) is None
    assert bench.profiled_traffic("w", "attention", str(tmp_path / "missing.json")) is None


def test_roofline_frac_is_against_the_burst_peak():
    peaks = {"bf16_tflops": 1600.0, "bf16_tflops_sustained": 1300.0, "bf16_tflops_sustained_sm_mhz": 1300.0}
    r = bench.tensor_roofline("attention", 1000.0, peaks, "measured", 1950.0, None)
    assert r["peak"] == 1600.0 and r["frac"] == pytest.approx(1000.0 / 1600.0)
    # the sustained figure scaled to the sampled clock
    assert r["peak_sustained_at_sampled_clock"] == pytest.approx(1300.0 * 1950.0 / 1300.0)
    assert r["frac_vs_sustained_at_sampled_clock"] == pytest.approx(1000.0 / 1950.0)
    # without a clock key the fallback's clock is used
    assert bench.sustained_clock_mhz({"bf16_tflops": 1.0}) == bench.FALLBACK_PEAKS["bf16_tflops_sustained_sm_mhz"]
    assert bench.sustained_clock_mhz({"x": {"sustained_clock_mhz": 1234}}) == 1234.0


def test_clock_sampler_reads_nvml_only_inside_the_timed_region(monkeypatch):
    # a fake NVML: SM clock 1500 then 1900 MHz, the power-cap bit from the third read on
    import sys
    import time
    import types
    reads = {"n": 0}

    def clock(handle, kind):
        reads["n"] += 1
        return 1500 if reads["n"] <= 2 else 1900

    fake = types.SimpleNamespace(
        NVML_CLOCK_SM=1,
        nvmlInit=lambda: None, nvmlShutdown=lambda: None,
        nvmlDeviceGetHandleByIndex=lambda i: ("gpu", i),
        nvmlDeviceGetMaxClockInfo=lambda h, k: 1965,
        nvmlDeviceGetClockInfo=clock,
        nvmlDeviceGetCurrentClocksEventReasons=lambda h: 0x4 if reads["n"] >= 3 else 0x0,
        NVML_FI_DEV_POWER_INSTANT=186,
        nvmlDeviceGetFieldValues=lambda h, ids: [types.SimpleNamespace(
            nvmlReturn=0, valueType=1, value=types.SimpleNamespace(uiVal=998000))],  # mW
        nvmlDeviceGetEnforcedPowerLimit=lambda h: 1000000)
    monkeypatch.setitem(sys.modules, "pynvml", fake)
    import bench
    c = bench.ClockSampler(3)
    assert reads["n"] == 0  # nothing read before the region starts
    with c:
        time.sleep(0.25)
    n_in = reads["n"]
    time.sleep(0.1)
    assert reads["n"] == n_in  # and nothing after it ends
    s = c.summary()
    assert s["samples"] == n_in >= 5 and s["sm_max_mhz"] == 1965.0
    assert s["sm_mhz"] == 1900.0 and s["reasons"] == ["sw_power_cap"]
    assert s["power_w"] == 998.0 and s["power_limit_w"] == 1000.0


def test_every_forward_kernel_of_each_schedule_has_its_flops():
    # the kernels one forward launches under each FFN schedule (the library's
    # timing-log names) all have a flop count, and the fused launches count
    # exactly the steps they run
    import bench
    import bpt_inputs as bi
    shape = bi.WORKLOADS["gpt7b_s32768_h4096"]
    f = bench.kernel_flops(shape)
    for name in ("gemm_qkv", "attention", "gemm_outproj", "gemm_ffn_up", "gemm_ffn_down", "ffn_chain", "layer_mega"):
        assert f[name] > 0, name
    assert f["ffn_chain"] == f["gemm_outproj"] + f["gemm_ffn_up"] + f["gemm_ffn_down"]
    assert f["layer_mega"] == f["attention"] + f["ffn_chain"]
    assert sum(bench.layer_flops(shape).values()) == f["gemm_qkv"] + f["layer_mega"]
