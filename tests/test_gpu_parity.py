"""GPU parity: the CUDA library (through its C ABI) against the fp64 oracle.

Both sides consume the same seeded inputs (bpt_inputs); the expected values
come only from oracle/. Tolerance for the layer output (fp32) against the
fp64 oracle: max-abs <= 2e-2 and relative L2 <= 1e-2, on every case. Steps
checked alone use tolerances derived from their single rounding (stated at
each test). Fixed points whose result is exact in the GPU's arithmetic are
checked for equality.
"""

import json
import os

import numpy as np
import pytest
import torch

import blockwise_attn_ffn_bpt_b200 as bpt
import bpt_inputs as bi
import oracle

pytestmark = pytest.mark.gpu

MAX_ABS = 2e-2
REL_L2 = 1e-2


def errors(got: np.ndarray, ref: np.ndarray):
    d = got.astype(np.float64) - ref
    return float(np.abs(d).max()), float(np.linalg.norm(d) / max(np.linalg.norm(ref), 1e-300))


def log_errors(what, mx, rl2):
    path = os.environ.get("BPT_PARITY_LOG")
    if path:
        with open(path, "a") as f:
            f.write(json.dumps({"case": what, "max_abs": mx, "rel_l2": rl2}) + "\n")


def assert_parity(got, ref, what):
    assert np.isfinite(got).all(), f"{what}: non-finite output"
    mx, rl2 = errors(got, ref)
    log_errors(what, mx, rl2)
    assert mx <= MAX_ABS and rl2 <= REL_L2, f"{what}: max-abs {mx:.3e}, rel-L2 {rl2:.3e}"
    return mx, rl2


def device_params(inp):
    return {k: bi.to_torch(inp[k]) for k in bi.PARAM_NAMES}


def run_layer(shape, inp, wave_rows=0, workspace=False):
    x = bi.to_torch(inp["x"])
    params = device_params(inp)
    if workspace:
        nbytes = bpt.workspace_bytes(bpt.BPT_DTYPE_F32 if shape.dtype == "f32" else bpt.BPT_DTYPE_BF16,
                                     shape.b, shape.s, shape.h, shape.heads, shape.q_block, shape.kv_block, wave_rows,
                                     ffn=shape.f)
        ws = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
        out = bpt.layer_forward(x, params, shape.heads, shape.q_block, shape.kv_block, shape.causal,
                                workspace=ws, wave_rows=wave_rows)
    else:
        out = bpt.layer_forward(x, params, shape.heads, shape.q_block, shape.kv_block, shape.causal,
                                wave_rows=wave_rows)
    torch.cuda.synchronize()
    assert bpt.stream_status() == 0
    return out.cpu().numpy()


def oracle_full(shape, inp):
    return oracle.layer_forward(*bi.oracle_args(inp), heads=shape.heads, causal=shape.causal)


# ---------------------------------------------------------------------------
# single steps
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("b,s,h", [(1, 256, 256), (2, 200, 512), (1, 77, 1024)])
def test_qkv_projection_matches_oracle(b, s, h):
    shp = bi.LayerShape(b, s, h, h // 64, 1, 1, False)
    inp = bi.make_inputs(shp, seed=1)
    q, k, v = bpt.qkv_projection(bi.to_torch(inp["x"]), bi.to_torch(inp["Wqkv"]), bi.to_torch(inp["bqkv"]))
    torch.cuda.synchronize()
    Q, K, V = oracle.qkv_projection(*(bi.to_f64(inp[n]) for n in ("x", "Wqkv", "bqkv")))
    for got, ref in ((q, Q), (k, K), (v, V)):
        g = got.float().cpu().numpy().astype(np.float64)
        # one bf16 rounding of an fp32-accumulated sum: |err| <= 2^-8 |ref| + 1e-4
        assert np.all(np.abs(g - ref) <= 2.0 ** -8 * np.abs(ref) + 1e-4)


def seeded_qkv(b, s, h, seed, q_scale=1.0):
    """Seeded bf16 Q, K, V drawn directly (std 1; Q scaled to sharpen the softmax)."""
    out = []
    for i, sc in enumerate((q_scale, 1.0, 1.0)):
        v = bi.normal_f64(seed, 20 + i, b * s * h) * sc
        out.append(bi.f32_to_bf16_bits(v.astype(np.float32)).reshape(b, s, h))
    return out


@pytest.mark.parametrize("b,s,h,heads", [(1, 256, 256, 2), (2, 384, 256, 4), (1, 200, 512, 4), (3, 130, 128, 1)])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("q_scale", [1.0, 4.0])
def test_attention_matches_oracle(b, s, h, heads, causal, q_scale):
    qb, kb = (s, s) if s % 64 else (64, 64)
    qkv = seeded_qkv(b, s, h, seed=2, q_scale=q_scale)
    o = bpt.attention(*(bi.to_torch(a) for a in qkv), heads, qb, kb, causal)
    torch.cuda.synchronize()
    ref = oracle.attention(*(bi.to_f64(a) for a in qkv), heads, causal)
    got = o.float().cpu().numpy()
    # P and O are rounded to bf16: |err| stays below 2e-2 for weighted means of unit-scale V
    assert_parity(got, ref, f"attention b{b} s{s} h{h} H{heads} causal{causal} qx{q_scale}")


def test_attention_rows_sum_to_one_exactly():
    b, s, h, heads = 2, 300, 256, 2
    q, k, _ = seeded_qkv(b, s, h, seed=3, q_scale=6.0)
    ones = np.full((b, s, h), 0x3F80, dtype=np.uint16)  # bf16 1.0
    for causal in (False, True):
        o = bpt.attention(bi.to_torch(q), bi.to_torch(k), bi.to_torch(ones), heads, 1, 1, causal)
        torch.cuda.synchronize()
        assert torch.equal(o.float().cpu(), torch.ones(b, s, h)), f"causal={causal}"


def test_attention_first_causal_row_is_its_own_value():
    b, s, h, heads = 2, 256, 256, 2
    q, k, v = seeded_qkv(b, s, h, seed=4, q_scale=3.0)
    o = bpt.attention(bi.to_torch(q), bi.to_torch(k), bi.to_torch(v), heads, 128, 128, True)
    torch.cuda.synchronize()
    got = o[:, 0].cpu().view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(got, v[:, 0])


def test_attention_zero_queries_average_the_visible_values():
    b, s, h, heads = 1, 512, 256, 2
    _, k, v = seeded_qkv(b, s, h, seed=5)
    zq = np.zeros((b, s, h), dtype=np.uint16)
    V = bi.to_f64(v)
    for causal in (False, True):
        o = bpt.attention(bi.to_torch(zq), bi.to_torch(k), bi.to_torch(v), heads, 64, 128, causal)
        torch.cuda.synchronize()
        got = o.float().cpu().numpy()
        if causal:
            ref = np.cumsum(V, axis=1) / np.arange(1, s + 1)[None, :, None]
        else:
            ref = np.broadcast_to(V.mean(axis=1, keepdims=True), V.shape)
        # uniform weights are exact; one fp32 sum and one bf16 rounding remain
        assert np.all(np.abs(got - ref) <= 2.0 ** -8 * np.abs(ref) + 1e-5)


# ---------------------------------------------------------------------------
# the whole layer, small and ragged cases
# ---------------------------------------------------------------------------

SMALL = [
    bi.LayerShape(1, 128, 128, 2, 64, 64, True),        # one tile everywhere, dh 64
    bi.LayerShape(2, 256, 256, 2, 128, 64, False),      # dh 128, two batch items
    bi.LayerShape(1, 320, 256, 4, 64, 160, True),       # ragged: s % 128 != 0
    bi.LayerShape(3, 64, 128, 1, 64, 32, True),         # s below one tile
    bi.LayerShape(1, 1, 128, 2, 1, 1, True),            # a single token
    bi.LayerShape(1, 1000, 192, 3, 200, 125, True),     # ragged everything, h not a multiple of 128
    bi.LayerShape(2, 512, 384, 3, 128, 256, False, "f32"),
]


@pytest.mark.parametrize("shape", SMALL, ids=lambda s: f"b{s.b}s{s.s}h{s.h}H{s.heads}q{s.q_block}k{s.kv_block}"
                                                       f"{'c' if s.causal else 'n'}{s.dtype}")
def test_layer_small_matches_oracle(shape):
    inp = bi.make_inputs(shape, seed=0)
    ref = oracle_full(shape, inp)
    got = run_layer(shape, inp)
    assert_parity(got, ref, str(shape))


# FFN widths other than the pages' 4h (bpt_layer_forward_ffn): f = h, a width
# that leaves a partial 256-column tile and three 64-deep K steps, f = 8h, and
# the fp32 entry with f = 5h/3
FFN_SHAPES = [
    bi.LayerShape(1, 256, 256, 4, 64, 64, True, "bf16", ffn=256),
    bi.LayerShape(2, 200, 256, 2, 40, 100, False, "bf16", ffn=192),
    bi.LayerShape(1, 320, 256, 4, 64, 160, True, "bf16", ffn=2048),
    bi.LayerShape(1, 256, 384, 3, 128, 64, True, "f32", ffn=640),
]


@pytest.mark.parametrize("shape", FFN_SHAPES, ids=lambda s: f"f{s.f}h{s.h}{s.dtype}")
@pytest.mark.parametrize("workspace", [False, True])
def test_layer_any_ffn_width_matches_oracle(shape, workspace):
    inp = bi.make_inputs(shape, seed=5)
    got = run_layer(shape, inp, workspace=workspace)
    assert_parity(got, oracle_full(shape, inp), f"ffn {shape.f}: {shape}")


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_host_entry_equals_the_device_path(dtype):
    # three different inputs through bpt_layer_forward_host (pinned host
    # memory, copies overlapped with compute) give, bit for bit, what the
    # device entry gives for each; stride 0 repeats one input
    shape = bi.LayerShape(1, 320, 256, 4, 64, 64, True, dtype)
    inps = [bi.make_inputs(shape, seed=s) for s in (11, 12, 13)]
    params = device_params(inps[0])
    xs = [bi.to_torch(i["x"], device="cpu") for i in inps]
    x_host = torch.stack(xs).pin_memory()
    got = bpt.layer_forward_host(x_host, params, shape.heads, shape.q_block, shape.kv_block, shape.causal)
    assert bpt.stream_status() == 0
    for k in range(3):
        ref = bpt.layer_forward(xs[k].cuda(), params, shape.heads, shape.q_block, shape.kv_block, shape.causal)
        torch.cuda.synchronize()
        assert torch.equal(got[k], ref.cpu()), f"input {k}"
    one = bpt.layer_forward_host(xs[1].pin_memory(), params, shape.heads, shape.q_block, shape.kv_block,
                                 shape.causal, n_inputs=4)
    assert torch.equal(one, got[1])
    # and the result is the oracle's layer
    assert_parity(got[0].numpy(), oracle_full(shape, inps[0]), f"host entry {dtype}")


@pytest.mark.parametrize("b,s,h,heads,q_block,kv_block,causal", [
    (1, 4096, 256, 2, 512, 512, True),    # one sequence: attention wave by wave, last wave in halves
    (3, 1000, 256, 2, 200, 125, True),    # waves and row chunks that straddle sequence boundaries
    (1, 4096, 256, 2, 512, 512, False),   # not causal: one attention launch before the waves
    (1, 6000, 256, 2, 1000, 500, True),   # waves of whole 1000-row query blocks: rows start off the 128-row tiles
], ids=["causal_b1", "causal_b3_ragged", "full_b1", "causal_q1000"])
def test_host_entry_pipelining_keeps_every_row_bit_equal(b, s, h, heads, q_block, kv_block, causal):
    # With causal attention the host entry runs each FFN wave's attention just
    # before the wave (launches split at sequence boundaries, the first input's
    # row chunks projected as the waves need them) and the last input's last
    # wave in two halves; the launch counts show that it did, and every row
    # must still equal the device entry's bit for bit.
    shape = bi.LayerShape(b, s, h, heads, q_block, kv_block, causal)
    inp = bi.make_inputs(shape, seed=21)
    params = device_params(inp)
    x = bi.to_torch(inp["x"], device="cpu")
    bpt.set_kernel_timing(True)
    try:
        bpt.kernel_times()
        got = bpt.layer_forward_host(x.pin_memory(), params, heads, q_block, kv_block, causal)
        torch.cuda.synchronize()
        k_host = bpt.kernel_times()
        ref = bpt.layer_forward(x.cuda(), params, heads, q_block, kv_block, causal)
        torch.cuda.synchronize()
        k_dev = bpt.kernel_times()
    finally:
        bpt.set_kernel_timing(False)
    assert bpt.stream_status() == 0
    assert torch.equal(got, ref.cpu())
    n_att_host, n_att_dev = k_host["attention"][0], k_dev["attention"][0]
    op_host, op_dev = k_host["gemm_outproj"][0], k_dev["gemm_outproj"][0]
    assert n_att_dev == 1
    if causal:
        # at least one attention launch per wave (one per sequence piece of it)
        assert n_att_host >= op_dev, (k_host, k_dev)
    else:
        assert n_att_host == 1, k_host
    assert op_dev <= op_host <= op_dev + 1, (k_host, k_dev)
    if b == 1:
        assert op_host == op_dev + 1, (k_host, k_dev)
    if s * s * h <= 4096 * 4096 * 256:  # the device entry itself is checked against the oracle elsewhere
        assert_parity(got.numpy(), oracle_full(shape, inp), f"host pipeline {shape}")


def test_convert_rounds_to_nearest_even_like_torch():
    g = torch.Generator(device="cuda").manual_seed(7)
    src = torch.randn(1 << 20 | 3, generator=g, device="cuda") * 100.0
    src[:4] = torch.tensor([1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, -0.0, 3.0e38], device="cuda")  # ties, sign, range
    got = bpt.convert_f32_to_bf16(src)
    torch.cuda.synchronize()
    assert torch.equal(got.view(torch.int16), src.to(torch.bfloat16).view(torch.int16))


def test_two_layer_stack_matches_the_oracle_applied_twice():
    # layer 2 reads layer 1's fp32 output rounded to bf16
    s1 = bi.LayerShape(1, 256, 256, 4, 64, 128, True)
    p1, p2 = bi.make_inputs(s1, seed=21), bi.make_inputs(s1, seed=22)
    d1, d2 = device_params(p1), device_params(p2)
    x = bi.to_torch(p1["x"])
    got = bpt.stack_forward(x, [d1, d2], s1.heads, s1.q_block, s1.kv_block, s1.causal)
    # the stack is the composition of the library's calls, bit for bit
    y1 = bpt.layer_forward(x, d1, s1.heads, s1.q_block, s1.kv_block, s1.causal)
    x2 = bpt.convert_f32_to_bf16(y1).view(x.shape)
    y2 = bpt.layer_forward(x2, d2, s1.heads, s1.q_block, s1.kv_block, s1.causal)
    torch.cuda.synchronize()
    assert bpt.stream_status() == 0
    assert torch.equal(got, y2)
    # layer 2 on that bf16 input is the oracle's layer (the usual bound)
    x2_64 = x2.float().cpu().numpy().astype(np.float64)
    ref2 = oracle.layer_forward(x2_64, *bi.oracle_args(p2)[1:], heads=s1.heads, causal=s1.causal)
    assert_parity(got.cpu().numpy(), ref2, "stack, layer 2 on the GPU's bf16 intermediate")
    # against the oracle applied twice (its own intermediate rounded to bf16):
    # where the two layer-1 results straddle a bf16 rounding boundary the
    # intermediates differ by one bf16 ulp (up to 2^-8 |x|, ~0.03 at |x| ~ 8),
    # so elementwise max-abs is not a stable measure here; rel-L2 is
    r1 = oracle.layer_forward(*bi.oracle_args(p1), heads=s1.heads, causal=s1.causal)
    r2 = oracle.layer_forward(bi.to_f64(bi.f32_to_bf16_bits(r1.astype(np.float32))), *bi.oracle_args(p2)[1:],
                              heads=s1.heads, causal=s1.causal)
    mx, rl2 = errors(got.cpu().numpy(), r2)
    log_errors("two-layer stack vs oracle twice", mx, rl2)
    assert rl2 <= REL_L2, f"rel-L2 {rl2:.3e}"


@pytest.mark.parametrize("wave_rows", [64, 128, 384, 100000])
def test_layer_result_does_not_depend_on_the_wave(wave_rows):
    shape = bi.LayerShape(2, 768, 256, 2, 64, 128, True)
    inp = bi.make_inputs(shape, seed=6)
    ref = oracle_full(shape, inp)
    got = run_layer(shape, inp, wave_rows=wave_rows, workspace=True)
    assert_parity(got, ref, f"wave_rows={wave_rows}")


@pytest.mark.parametrize("schedule", [-1, -2, -3], ids=["chained", "default-waves", "one-launch"])
def test_both_ffn_schedules_match_the_oracle(schedule):
    # the FFN side in one launch (BPT_WAVE_CHAINED: four 2048-row groups here,
    # so both scratch slots are reused), in one launch per GEMM and wave
    # (BPT_WAVE_DEFAULT_WAVES) and attention with the FFN side in one launch
    # (BPT_WAVE_MEGA) compute the same layer
    shape = bi.LayerShape(2, 4096, 256, 2, 128, 256, True)
    inp = bi.make_inputs(shape, seed=9)
    got = run_layer(shape, inp, wave_rows=schedule, workspace=True)
    assert_parity(got, oracle_full(shape, inp), f"ffn schedule {schedule}")


MEGA_SHAPES = [
    bi.LayerShape(2, 4096, 256, 2, 128, 256, True),      # dh 128, row groups reusing the scratch slots
    bi.LayerShape(1, 1152, 256, 4, 128, 128, False),     # dh 64, an odd number of query tiles
    bi.WORKLOADS["gpt1b_s8192_h2048"],                   # the 1B-class workload
]


@pytest.mark.parametrize("shape", MEGA_SHAPES, ids=["b2_s4096", "s1152_dh64", "gpt1b"])
def test_one_launch_layer_equals_the_chained_schedule(shape):
    # attention and the FFN side in one persistent launch (BPT_WAVE_MEGA) run the
    # same arithmetic as attention followed by the chained FFN side: equal bit for
    # bit; and it is that kernel which ran
    inp = bi.make_inputs(shape, seed=21)
    chained = run_layer(shape, inp, wave_rows=-1, workspace=True)
    bpt.set_kernel_timing(True)
    bpt.kernel_times()
    mega = run_layer(shape, inp, wave_rows=-3, workspace=True)
    kinds = bpt.kernel_times()
    bpt.set_kernel_timing(False)
    assert "layer_mega" in kinds and "attention" not in kinds and "ffn_chain" not in kinds, kinds
    assert np.array_equal(mega, chained)


@pytest.mark.parametrize("q_scale,max_abs", [(2.0, MAX_ABS), (8.0, 0.1)])
def test_layer_sharp_attention_matches_oracle(q_scale, max_abs):
    # query weights scaled: attention far from uniform, so attention errors are
    # visible in the output. At x2 the full tolerance applies. At x8 the scores
    # have std ~8 and a CPU emulation that rounds only Q, K, V and O to bf16
    # (everything else exact) already moves the output by max-abs 0.068, so
    # there the bound is max-abs 0.1 with the usual rel-L2 1e-2.
    shape = bi.LayerShape(1, 1024, 512, 4, 128, 128, True)
    inp = bi.make_inputs(shape, seed=7)
    w = bi.to_f64(inp["Wqkv"])
    w[:, :512] *= q_scale
    inp["Wqkv"] = bi.f32_to_bf16_bits(w.astype(np.float32))
    ref = oracle_full(shape, inp)
    got = run_layer(shape, inp)
    assert np.isfinite(got).all()
    mx, rl2 = errors(got, ref)
    log_errors(f"sharp q x{q_scale}", mx, rl2)
    assert mx <= max_abs and rl2 <= REL_L2, f"q x{q_scale}: max-abs {mx:.3e}, rel-L2 {rl2:.3e}"


def test_layer_uniform_attention_closed_form():
    # Wq = 0: uniform attention over the visible keys. Wv = I, Wo = I, FFN off:
    # out = x + prefix-mean(x) (causal); all weights here are exact in bf16
    b, s, h, heads = 1, 384, 128, 2
    shape = bi.LayerShape(b, s, h, heads, 128, 128, True)
    inp = bi.make_inputs(shape, seed=8)
    eye = bi.f32_to_bf16_bits(np.eye(h, dtype=np.float32))
    wqkv = np.zeros((h, 3 * h), dtype=np.uint16)
    wqkv[:, h:2 * h] = inp["Wqkv"][:, h:2 * h]
    wqkv[:, 2 * h:] = eye
    inp.update(Wqkv=wqkv, bqkv=np.zeros(3 * h, np.uint16), Wo=eye, bo=np.zeros(h, np.uint16),
               W1=np.zeros((h, 4 * h), np.uint16), b1=np.zeros(4 * h, np.uint16),
               W2=np.zeros((4 * h, h), np.uint16), b2=np.zeros(h, np.uint16))
    x = bi.to_f64(inp["x"])
    ref = x + np.cumsum(x, axis=1) / np.arange(1, s + 1)[None, :, None]
    got = run_layer(shape, inp)
    pm = ref - x
    assert np.all(np.abs(got - ref) <= 2.0 ** -8 * np.abs(pm) + 1e-5)


# ---------------------------------------------------------------------------
# the workloads at full size
# ---------------------------------------------------------------------------

def sample_rows(shape, per_block=2, extra=16, cap=96, seed=0):
    """Rows spread over every query block: first and last row of each block
    (or of evenly spaced blocks when there are many) plus random rows."""
    rng = np.random.default_rng(seed)
    n_blocks = shape.s // shape.q_block
    blocks = np.unique(np.linspace(0, n_blocks - 1, min(n_blocks, cap // 2)).astype(int))
    rows = []
    for beta in range(shape.b):
        for blk in blocks:
            t0 = blk * shape.q_block
            rows += [beta * shape.s + t0, beta * shape.s + t0 + shape.q_block - 1][:per_block]
        rows += list(beta * shape.s + rng.integers(0, shape.s, extra))
    return np.unique(np.array(rows, dtype=np.int64))


def test_workload_small_fp32_full():
    shape = bi.WORKLOADS["small_fp32_s256_h256"]
    inp = bi.make_inputs(shape, seed=0)
    ref = oracle_full(shape, inp)
    got = run_layer(shape, inp)
    assert_parity(got, ref, "small fp32 workload")


def test_workload_causal_b2_s2048_full():
    shape = bi.WORKLOADS["causal_b2_s2048_h1024"]
    inp = bi.make_inputs(shape, seed=0)
    ref = oracle_full(shape, inp)
    got = run_layer(shape, inp)
    assert_parity(got, ref, "b2 s2048 h1024 causal")


def test_workload_gpt1b_s8192_every_row():
    # the 1B-class workload (s = 8192, h = 2048, causal) compared on every row
    shape = bi.WORKLOADS["gpt1b_s8192_h2048"]
    inp = bi.make_inputs(shape, seed=0)
    got = run_layer(shape, inp)
    assert_parity(got, oracle_full(shape, inp), "gpt1b s8192 h2048, every row")


def test_workload_gpt7b_s32768_first_and_last_query_blocks_and_sampled_rows():
    # the 7B-class workload: every row of the first and of the last query
    # block (rows 31744-32767 attend to the longest prefixes, where the running
    # max has moved most), plus rows spread over every other query block
    shape = bi.WORKLOADS["gpt7b_s32768_h4096"]
    inp = bi.make_inputs(shape, seed=0)
    got = run_layer(shape, inp)
    assert np.isfinite(got).all()
    qb = shape.q_block
    rows = np.unique(np.concatenate([np.arange(qb), np.arange(shape.s - qb, shape.s), sample_rows(shape)]))
    ref = oracle.layer_rows(*bi.oracle_args(inp), heads=shape.heads, causal=shape.causal, rows=rows)
    flat = got.reshape(-1, shape.h)
    assert_parity(flat[:qb], ref[:qb], "gpt7b first query block")
    assert_parity(flat[shape.s - qb:], ref[-qb:], "gpt7b last query block")
    assert_parity(flat[rows], ref, "gpt7b first, last and sampled rows")


@pytest.mark.parametrize("causal", [True, False])
def test_block_size_sweep_sampled_rows(causal):
    shapes = [bi.sweep_shape(blk, causal) for blk in bi.SWEEP_BLOCKS]
    inp = bi.make_inputs(shapes[0], seed=0)  # the inputs do not depend on the block size
    rows = sample_rows(bi.sweep_shape(64, causal), cap=64)
    ref = oracle.layer_rows(*bi.oracle_args(inp), heads=16, causal=causal, rows=rows)
    outs = []
    for shape in shapes:
        got = run_layer(shape, inp).reshape(-1, shape.h)
        assert np.isfinite(got).all()
        assert_parity(got[rows], ref, f"sweep block {shape.q_block} causal={causal}")
        outs.append(got)
    # every block size computes the same layer
    for o in outs[1:]:
        assert np.abs(o - outs[0]).max() <= MAX_ABS
    # and one sweep point (q_block = kv_block = 2048) on every row
    assert shapes[-1].q_block == 2048
    full = oracle_full(shapes[-1], inp).reshape(-1, shapes[-1].h)
    assert_parity(outs[-1], full, f"sweep block 2048 causal={causal}, every row")
