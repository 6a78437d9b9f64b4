"""Host-side logic of bench.py without a GPU: the multi-rank plumbing on gloo
(world size 2), the whole-job throughput formula, and the reference arm (the
fp64 oracle on a bounded sample) on the CPU."""

import json
import os
import subprocess
import sys

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
