"""The C ABI without a GPU: the library loads, exports every function that
include/bpt.h declares, and rejects bad arguments synchronously (argument
checks run before any CUDA call, so these run on a CPU-only machine)."""

import os
import re

import numpy as np
import pytest

import blockwise_attn_ffn_bpt_b200 as bpt

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "bpt.h")

OK, NULL, SHAPE, BLOCK, ALIGN, ALIAS, NOMEM, DTYPE = 0, -1, -2, -3, -4, -5, -6, -10


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(bpt_[a-z0-9_]+)\s*\(", text)))


def test_library_exports_every_declared_function():
    L = bpt.lib()
    names = declared_functions()
    assert "bpt_layer_forward" in names and len(names) >= 10
    for n in names:
        assert hasattr(L, n), f"{n} declared in bpt.h but not exported"
    assert set(bpt.EXPORTED) == set(names)


def test_status_strings():
    for code in (OK, NULL, SHAPE, BLOCK, ALIGN, ALIAS, NOMEM, -7, -8, -9, DTYPE):
        assert bpt.status_string(code).startswith("BPT_")
    assert bpt.status_string(12345) == "unknown bpt status"


# fake, aligned, non-overlapping "device" addresses: the checks fail before any are used
BASE = 1 << 40
STEP = 1 << 36


def fake_ptrs(n):
    return [BASE + i * STEP for i in range(n)]


def call_layer(b=1, s=256, h=256, heads=4, qb=64, kb=64, causal=0, ptrs=None, out=None):
    p = ptrs or fake_ptrs(9)
    o = out if out is not None else BASE + 20 * STEP
    return bpt.lib().bpt_layer_forward(*p, b, s, h, heads, qb, kb, causal, o, None)


@pytest.mark.parametrize("kw,code", [
    (dict(h=256, heads=3), SHAPE),          # h % heads
    (dict(h=256, heads=8), SHAPE),          # dh = 32
    (dict(h=512, heads=2), SHAPE),          # dh = 256
    (dict(b=-1), SHAPE),
    (dict(s=-5), SHAPE),
    (dict(qb=0), BLOCK),
    (dict(qb=48), BLOCK),                   # 256 % 48
    (dict(kb=512), BLOCK),                  # > s
    (dict(kb=-64), BLOCK),
])
def test_layer_rejects_bad_shapes(kw, code):
    assert call_layer(**kw) == code


def test_empty_problem_is_a_noop():
    assert call_layer(b=0) == OK
    assert call_layer(s=0, qb=1, kb=1) == OK
    # empty problems need no pointers at all
    assert bpt.lib().bpt_layer_forward(*([None] * 9), 0, 128, 256, 4, 64, 64, 1, None, None) == OK


def test_layer_rejects_null_and_misaligned_pointers():
    p = fake_ptrs(9)
    for i in range(9):
        q = list(p)
        q[i] = None
        assert call_layer(ptrs=q) == NULL
        q[i] = p[i] + 8
        assert call_layer(ptrs=q) == ALIGN
    assert bpt.lib().bpt_layer_forward(*p, 1, 256, 256, 4, 64, 64, 0, None, None) == NULL


def test_layer_rejects_out_overlapping_an_input():
    p = fake_ptrs(9)
    assert call_layer(ptrs=p, out=p[0] + 256) == ALIAS      # inside x
    assert call_layer(ptrs=p, out=p[5] - 1024) == ALIAS     # runs into W1


def test_ws_entry_checks_dtype_and_workspace():
    L = bpt.lib()
    p = fake_ptrs(9)
    out = BASE + 20 * STEP
    ws = BASE + 30 * STEP
    need = bpt.workspace_bytes(0, 1, 256, 256, 4, 64, 64)
    args = [1, 256, 256, 4, 64, 64, 1, 0]
    assert L.bpt_layer_forward_ws(7, *p, *args, ws, need, out, None) == DTYPE
    assert L.bpt_layer_forward_ws(0, *p, *args, None, need, out, None) == NULL
    assert L.bpt_layer_forward_ws(0, *p, *args, ws + 16, need, out, None) == ALIGN
    assert L.bpt_layer_forward_ws(0, *p, *args, ws, need - 1, out, None) == NOMEM
    assert L.bpt_layer_forward_ws(0, *p, *args, p[3], need, out, None) == ALIAS


def _up(v):
    return (v + 1023) // 1024 * 1024


def chain_workspace(b, s, h, f):
    """Default bf16 workspace: one region holds K and V for the whole sequence
    during projection and attention, then the slots of the one-launch FFN side
    (3 slots of a row group's fp32 hid and bf16 hid copy, 2 of its bf16 U; the
    largest group of 16, 8, 4, 2 or 1 128-row tiles whose slots take at most
    1.5x the K/V bytes or 32 MiB), each piece rounded up to 1 KiB; then the
    chain's counters (three per group)."""
    M = b * s
    mt = -(-M // 128)
    kv = 2 * _up(M * h * 2)
    for gm in (16, 8, 4, 2, 1):
        groups = -(-mt // gm)
        hs, us, rows = min(3, groups), min(2, groups), gm * 128
        slots = _up(hs * rows * h * 4) + _up(hs * rows * h * 2) + _up(us * rows * f * 2)
        if slots <= max(kv // 2 * 3, 32 << 20):
            break
    return _up(max(kv, slots) + 3 * groups * 4), kv, slots


def chain_groups(b, s, h, f):
    """Row groups of the chained FFN side (the same choice as chain_workspace)."""
    mt = -(-(b * s) // 128)
    kv = 2 * _up(b * s * h * 2)
    for gm in (16, 8, 4, 2, 1):
        groups = -(-mt // gm)
        hs, us, rows = min(3, groups), min(2, groups), gm * 128
        if _up(hs * rows * h * 4) + _up(hs * rows * h * 2) + _up(us * rows * f * 2) <= max(kv // 2 * 3, 32 << 20):
            return groups
    return groups


def test_one_launch_layer_workspace_puts_the_slots_after_the_keys_and_values():
    # BPT_WAVE_MEGA: attention runs while the FFN side of earlier rows does, so
    # the chain's slots follow the K/V region instead of aliasing it; then the
    # counters (three per group for the chain, one per group for attention, one
    # ticket)
    for b, s, h, heads, qb, kvb in [(1, 32768, 4096, 32, 1024, 2048), (2, 4096, 256, 2, 128, 256),
                                    (1, 8192, 2048, 16, 512, 512), (1, 1152, 256, 4, 128, 128)]:
        _, kv, slots = chain_workspace(b, s, h, 4 * h)
        groups = chain_groups(b, s, h, 4 * h)
        assert bpt.workspace_bytes(0, b, s, h, heads, qb, kvb, -3) == _up(kv + slots + (4 * groups + 1) * 4)
    # at the 32k-token 7B shape that is 2048-row groups: 285 MiB more than the K/V region
    assert bpt.workspace_bytes(0, 1, 32768, 4096, 32, 1024, 2048, -3) - 2 * 32768 * 4096 * 2 < 300 << 20
    # s not a multiple of 128: as the chained schedule; fp32 inputs: per wave, as by default
    assert bpt.workspace_bytes(0, 3, 1000, 192, 3, 200, 125, -3) == chain_workspace(3, 1000, 192, 768)[0]
    assert bpt.workspace_bytes(1, 1, 256, 256, 4, 64, 64, -3) == bpt.workspace_bytes(1, 1, 256, 256, 4, 64, 64)


def test_workspace_bytes_follow_the_layout():
    def wave(b, s, h, wr):
        # explicit wave: K/V region, or one wave's fp32 hid, its bf16 copy and the bf16 U (wave rows x 4h)
        return max(_up(b * s * h * 2) * 2, _up(wr * h * 4) + _up(wr * h * 2) + _up(wr * 4 * h * 2))

    b, s, h = 1, 32768, 4096
    ws = bpt.workspace_bytes(0, b, s, h, 32, 1024, 2048)
    # the 32k-token 7B shape, default (per-GEMM waves): 8192-row waves (8 query
    # blocks) whose scratch fits inside the K/V region
    assert ws == wave(b, s, h, 8192) == 2 * b * s * h * 2
    assert ws / 2 / (2 * b * s * h) <= 1.0  # element ratio against 2bsh
    assert bpt.workspace_bytes(0, b, s, h, 32, 1024, 2048, -2) == ws  # BPT_WAVE_DEFAULT_WAVES
    assert bpt.workspace_bytes(0, b, s, h, 32, 1024, 2048, 12288) == wave(b, s, h, 12288) > ws
    # the chained schedule: its 2048-row slots fit inside the K/V region too
    exp, kv, slots = chain_workspace(b, s, h, 4 * h)
    assert bpt.workspace_bytes(0, b, s, h, 32, 1024, 2048, -1) == exp and slots < kv == ws
    assert exp / 2 / (2 * b * s * h) <= 1.0001  # the counters add a few KiB
    for args in [(2, 2048, 1024, 16, 128, 128), (1, 16384, 2048, 16, 2048, 2048), (1, 8192, 2048, 16, 512, 512),
                 (1, 256, 256, 4, 64, 64), (3, 1000, 192, 3, 200, 125)]:
        b_, s_, h_ = args[:3]
        assert bpt.workspace_bytes(0, *args, -1) == chain_workspace(b_, s_, h_, 4 * h_)[0], args
    assert bpt.workspace_bytes(0, 2, 2048, 1024, 16, 128, 128) == wave(2, 2048, 1024, 4096)
    assert bpt.workspace_bytes(0, 1, 8192, 2048, 16, 512, 512) == wave(1, 8192, 2048, 4096)
    # explicit waves: whole query blocks; a whole-sequence wave covers whole sequences
    assert bpt.workspace_bytes(0, 2, 2048, 1024, 16, 128, 128, 2048) == wave(2, 2048, 1024, 2048)
    assert bpt.workspace_bytes(0, 1, 16384, 2048, 16, 2048, 2048, 1000) == wave(1, 16384, 2048, 2048)
    assert bpt.workspace_bytes(0, 2, 2048, 1024, 16, 128, 128, 100000) == wave(2, 2048, 1024, 4096)
    # fp32 inputs keep one launch per GEMM and wave and add their bf16 parts: x
    # as [x_hi | x_lo] rows, Wqkv as [hi; lo; hi], Wo, W1 and W2 as [hi; lo]
    f = bpt.workspace_bytes(1, 1, 256, 256, 4, 64, 64)
    assert f == wave(1, 256, 256, 256) + _up(256 * 512 * 2) + _up(768 * 768 * 2) + _up(512 * 256 * 2) + \
        _up(512 * 1024 * 2) + _up(2048 * 256 * 2)
    assert bpt.workspace_bytes(0, 1, 256, 256, 3, 64, 64) == 0
    assert bpt.workspace_bytes(0, 0, 256, 256, 4, 64, 64) == 0


def test_ffn_width_entry_validates_and_sizes_its_workspace():
    L = bpt.lib()
    p = fake_ptrs(9)
    out = BASE + 20 * STEP

    def up(v):
        return (v + 1023) // 1024 * 1024

    # the FFN width must be a positive multiple of 64; refused before any CUDA call
    for bad in (0, -64, 32, 100):
        assert L.bpt_layer_forward_ffn(0, *p, 1, 256, 256, 4, bad, 64, 64, 1, 0, None, 0, out, None) == SHAPE
        assert bpt.workspace_bytes(0, 1, 256, 256, 4, 64, 64, ffn=bad) == 0
    # 4h through the general entry is the default layout
    for wr in (0, 128, 1000):
        assert bpt.workspace_bytes(0, 2, 512, 256, 4, 64, 64, wr, ffn=1024) == \
            bpt.workspace_bytes(0, 2, 512, 256, 4, 64, 64, wr)
    # one region: K and V, or the wave scratch with an ffn-wide U
    assert bpt.workspace_bytes(0, 1, 2048, 1024, 16, 128, 128, 512, ffn=192) == \
        max(2 * up(2048 * 1024 * 2), up(512 * 1024 * 4) + up(512 * 1024 * 2) + up(512 * 192 * 2))
    assert bpt.workspace_bytes(0, 1, 256, 256, 4, 64, 64, 256, ffn=4096) == \
        max(2 * up(256 * 256 * 2), up(256 * 256 * 4) + up(256 * 256 * 2) + up(256 * 4096 * 2))
    # fp32 inputs add the bf16 parts, W1 [h, f] and W2 [f, h] as [hi; lo]
    f32 = bpt.workspace_bytes(1, 1, 256, 256, 4, 64, 64, 256, ffn=640)
    b16 = bpt.workspace_bytes(0, 1, 256, 256, 4, 64, 64, 256, ffn=640)
    assert f32 == b16 + up(256 * 512 * 2) + up(768 * 768 * 2) + up(512 * 256 * 2) + up(512 * 640 * 2) + \
        up(1280 * 256 * 2)
    # a too-small caller workspace and a misaligned one are refused
    need = bpt.workspace_bytes(0, 1, 256, 256, 4, 64, 64, 0, ffn=512)
    ws = BASE + 30 * STEP
    assert L.bpt_layer_forward_ffn(0, *p, 1, 256, 256, 4, 512, 64, 64, 1, 0, ws, need - 1, out, None) == NOMEM
    assert L.bpt_layer_forward_ffn(0, *p, 1, 256, 256, 4, 512, 64, 64, 1, 0, ws + 16, need, out, None) == ALIGN


def test_host_entry_validates_before_touching_memory():
    L = bpt.lib()
    w = fake_ptrs(8)  # device weights (never dereferenced: every case fails validation first)
    xh, oh = BASE + 40 * STEP, BASE + 50 * STEP
    shp = [1, 256, 256, 4, 64, 64, 1]
    xb, ob = 256 * 256 * 2, 256 * 256 * 4
    assert L.bpt_layer_forward_host(0, xh, xb, *w, *shp, oh, ob, 0, None) == OK  # nothing to do
    assert L.bpt_layer_forward_host(0, xh, xb, *w, *shp, oh, ob, -1, None) == SHAPE
    assert L.bpt_layer_forward_host(0, None, xb, *w, *shp, oh, ob, 2, None) == NULL
    assert L.bpt_layer_forward_host(0, xh, xb, *w, *shp, None, ob, 2, None) == NULL
    assert L.bpt_layer_forward_host(0, xh, xb, *w[:7], None, *shp, oh, ob, 2, None) == NULL
    assert L.bpt_layer_forward_host(0, xh, xb, *w[:7], w[7] + 8, *shp, oh, ob, 2, None) == ALIGN
    assert L.bpt_layer_forward_host(0, xh, xb - 2, *w, *shp, oh, ob, 2, None) == SHAPE  # stride below one input
    assert L.bpt_layer_forward_host(0, xh, xb, *w, *shp, oh, ob - 4, 2, None) == SHAPE
    assert L.bpt_layer_forward_host(0, xh, xb, *w, *shp, xh + xb, ob, 2, None) == ALIAS  # out inside the inputs
    assert L.bpt_layer_forward_host(0, xh, 0, *w, *shp, xh, 0, 3, None) == ALIAS
    assert L.bpt_layer_forward_host(5, xh, xb, *w, *shp, oh, ob, 2, None) == DTYPE
    assert L.bpt_layer_forward_host(0, xh, 1 << 40, *w, *shp, oh, ob, 1 << 30, None) == SHAPE  # range overflows
    assert L.bpt_layer_forward_host(0, xh, xb, *w, 1, 256, 256, 3, 64, 64, 1, oh, ob, 2, None) == SHAPE
    assert L.bpt_layer_forward_host(0, xh, xb, *w, 1, 256, 256, 4, 48, 64, 1, oh, ob, 2, None) == BLOCK


def test_convert_entry_validates():
    L = bpt.lib()
    a, b = BASE, BASE + STEP
    assert L.bpt_convert_f32_to_bf16(a, b, 0, None) == OK
    assert L.bpt_convert_f32_to_bf16(a, b, -1, None) == SHAPE
    assert L.bpt_convert_f32_to_bf16(None, b, 8, None) == NULL
    assert L.bpt_convert_f32_to_bf16(a, None, 8, None) == NULL
    assert L.bpt_convert_f32_to_bf16(a + 4, b, 8, None) == ALIGN
    assert L.bpt_convert_f32_to_bf16(a, b + 8, 8, None) == ALIGN
    assert L.bpt_convert_f32_to_bf16(a, a + 16, 8, None) == ALIAS
    assert L.bpt_convert_f32_to_bf16(a, b, (1 << 60) + 1, None) == SHAPE


def test_stage_entry_points_validate():
    L = bpt.lib()
    p = fake_ptrs(6)
    assert L.bpt_qkv_projection(p[0], p[1], p[2], 1, 128, 100, p[3], p[4], p[5], None) == SHAPE
    assert L.bpt_qkv_projection(p[0], None, p[2], 1, 128, 128, p[3], p[4], p[5], None) == NULL
    assert L.bpt_attention(p[0], p[1], p[2], 1, 128, 256, 2, 128, 64, 1, None, None) == NULL
    assert L.bpt_attention(p[0], p[1], p[2], 1, 128, 256, 2, 96, 64, 1, p[3], None) == BLOCK
    assert L.bpt_attention(p[0], p[1], p[2] + 4, 1, 128, 256, 2, 64, 64, 1, p[3], None) == ALIGN


def test_status_entry_points_without_a_gpu():
    # bpt_stream_status synchronises the stream it is given before it reads
    # that stream's word: with no GPU the synchronisation fails, which it
    # reports as BPT_ERR_CUDA instead of a status word (and it must not crash)
    L = bpt.lib()
    import torch
    if torch.cuda.is_available():
        pytest.skip("checks the no-GPU answer")
    assert L.bpt_stream_status(None) == -7
    assert L.bpt_stream_status(0x2) == -7  # the per-thread default stream handle
    assert L.bpt_device_status() == -7


def test_wait_flag_entry_validates():
    L = bpt.lib()
    f = BASE
    assert L.bpt_wait_flag(None, 1, 1000, None) == NULL
    assert L.bpt_wait_flag(f + 2, 1, 1000, None) == ALIGN
    assert L.bpt_wait_flag(f, 1, -1, None) == SHAPE
    assert L.bpt_wait_flag(f, 1, 10_000_001, None) == SHAPE


def test_kernel_timing_log_is_empty_without_launches():
    bpt.set_kernel_timing(True)
    assert bpt.kernel_times() == {}
    bpt.set_kernel_timing(False)
    assert bpt.launch_count() >= 0


def test_workspaces_keep_to_their_memory_budgets():
    # over many valid shapes: the default workspace (per-GEMM waves) holds K
    # and V, and its wave scratch stays within the larger of 1.5x the K/V
    # bytes and the scratch of a ~4096-row wave (whole query blocks, or whole
    # sequences); the chained schedule's slots stay within 1.5x the K/V region
    # (or 32 MiB) whenever a one-tile group does (otherwise the one-tile
    # group's slots set the size), and its counters add a few KiB
    rng = np.random.default_rng(0)
    for _ in range(300):
        heads = int(rng.integers(1, 9))
        h = heads * int(rng.choice([64, 128]))
        q_block = int(rng.choice([1, 16, 64, 128, 512, 1024]))
        s = q_block * int(rng.integers(1, 65))
        b = int(rng.integers(1, 5))
        f = 64 * int(rng.integers(1, 4 * h // 64 + 9))
        ws_waves = bpt.workspace_bytes(0, b, s, h, heads, q_block, q_block, ffn=f)
        kv = 2 * _up(b * s * h * 2)
        floor_rows = max(q_block, 4096 // q_block * q_block) if s >= 4096 else min(b, 4096 // s) * s
        wave_budget = max(kv // 2 * 3, _up(floor_rows * h * 4) + _up(floor_rows * h * 2) + _up(floor_rows * f * 2))
        assert kv <= ws_waves <= max(kv, wave_budget + 3 * 1024), (b, s, h, heads, q_block, f)
        assert ws_waves >= bpt.workspace_bytes(0, b, s, h, heads, q_block, q_block, q_block, ffn=f)
        ws = bpt.workspace_bytes(0, b, s, h, heads, q_block, q_block, -1, ffn=f)
        exp, kv, slots = chain_workspace(b, s, h, f)
        assert ws == exp, (b, s, h, heads, q_block, f)
        assert ws >= kv
        mt = -(-b * s // 128)
        one_tile = min(3, mt) * 128 * h * 6 + min(2, mt) * 128 * f * 2 + 3 * 1024
        assert ws <= max(kv // 2 * 3, 32 << 20, one_tile) + _up(3 * mt * 4) + 1024, (b, s, h, heads, q_block, f)
        assert bpt.workspace_bytes(0, b, s, h, heads, q_block, q_block, -2, ffn=f) == ws_waves


def test_binding_checks_parameters_before_calling_the_library():
    # shape and dtype checks run in Python, before any pointer reaches the C ABI
    import torch

    b, s, h = 1, 8, 64
    x = torch.zeros((b, s, h), dtype=torch.bfloat16)
    good = {"Wqkv": (h, 3 * h), "bqkv": (3 * h,), "Wo": (h, h), "bo": (h,), "W1": (h, 4 * h), "b1": (4 * h,),
            "W2": (4 * h, h), "b2": (h,)}
    params = {k: torch.zeros(shp, dtype=torch.bfloat16) for k, shp in good.items()}
    bad = dict(params, W2=torch.zeros((4 * h, h + 64), dtype=torch.bfloat16))
    with pytest.raises(ValueError, match="W2"):
        bpt.layer_forward(x, bad, 1, 8, 8, True, out=torch.empty((b, s, h)))
    bad = dict(params, bo=torch.zeros((h,), dtype=torch.float32))
    with pytest.raises(TypeError, match="bo"):
        bpt.layer_forward(x, bad, 1, 8, 8, True, out=torch.empty((b, s, h)))
    with pytest.raises(TypeError):
        bpt.layer_forward(x.to(torch.float16), params, 1, 8, 8, True, out=torch.empty((b, s, h)))
    # the host entry wants host inputs and CUDA weights
    with pytest.raises(ValueError):
        bpt.layer_forward_host(x, params, 1, 8, 8, True, out_host=torch.empty((b, s, h)))
    with pytest.raises(TypeError):
        bpt.convert_f32_to_bf16(torch.zeros(4))


def test_ffn_backward_entry_validates_before_touching_memory():
    L = bpt.lib()
    p = fake_ptrs(11)
    hid, W1, b1, W2, dy, dhid, dW1, db1, dW2, db2, ws = p
    rows, h, f = 1000, 256, 1024
    need = L.bpt_ffn_backward_workspace_bytes(rows, h, f, 384)
    # chunk of 384 rows: bf16 copies of hid and dy, the intermediate and da
    assert need == 2 * _up(384 * h * 2) + 2 * _up(384 * f * 2)
    assert L.bpt_ffn_backward_workspace_bytes(rows, h, f, 0) == 2 * _up(1000 * h * 2) + 2 * _up(1000 * f * 2)
    assert L.bpt_ffn_backward_workspace_bytes(rows, h, f, 100) == 2 * _up(128 * h * 2) + 2 * _up(128 * f * 2)
    assert L.bpt_ffn_backward_workspace_bytes(rows, 100, f, 0) == 0

    def call(**kw):
        a = dict(hid=hid, W1=W1, b1=b1, W2=W2, dy=dy, rows=rows, h=h, f=f, chunk=384, dhid=dhid, dW1=dW1, db1=db1,
                 dW2=dW2, db2=db2, ws=ws, nbytes=need)
        a.update(kw)
        return L.bpt_ffn_backward(a["hid"], a["W1"], a["b1"], a["W2"], a["dy"], a["rows"], a["h"], a["f"],
                                  a["chunk"], a["dhid"], a["dW1"], a["db1"], a["dW2"], a["db2"], a["ws"],
                                  a["nbytes"], None)

    assert call(rows=0) == OK
    assert call(h=100) == SHAPE and call(f=1000) == SHAPE and call(rows=-1) == SHAPE and call(chunk=-5) == SHAPE
    assert call(W2=None) == NULL and call(ws=None) == NULL
    assert call(dy=dy + 8) == ALIGN
    assert call(nbytes=need - 1) == NOMEM
    assert call(dW1=hid) == ALIAS  # an output over an input
    assert call(db1=dW2 + 16) == ALIAS  # two outputs overlapping


def test_backward_entries_validate_and_size_their_workspaces():
    L = bpt.lib()

    def up(v):
        return (v + 1023) // 1024 * 1024

    b, s, h, heads, f = 2, 256, 256, 2, 512
    rows = b * s
    # attention backward: D and the fp32 dQ sums
    assert L.bpt_attention_backward_workspace_bytes(b, s, h, heads) == up(b * heads * s * 4) + up(rows * h * 4)
    assert L.bpt_attention_backward_workspace_bytes(b, s, 192, 2) == 0  # dh 96
    p = fake_ptrs(10)
    ws_att = L.bpt_attention_backward_workspace_bytes(b, s, h, heads)
    assert L.bpt_attention_backward(*p[:6], b, s, 192, 2, 1, *p[6:9], p[9], ws_att, None) == SHAPE
    assert L.bpt_attention_backward(*p[:6], b, s, h, heads, 1, *p[6:9], None, ws_att, None) == NULL
    assert L.bpt_attention_backward(*p[:6], b, s, h, heads, 1, *p[6:9], p[9], ws_att - 1, None) == NOMEM
    assert L.bpt_attention_backward(*p[:6], b, s, h, heads, 1, p[6] + 8, *p[7:9], p[9], ws_att, None) == ALIGN
    assert L.bpt_attention_backward(*p[:6], b, s, h, heads, 1, p[0], *p[7:9], p[9], ws_att, None) == ALIAS
    assert L.bpt_attention_backward(*p[:6], 0, s, h, heads, 1, *p[6:9], p[9], 0, None) == OK  # nothing to do
    assert L.bpt_attention_lse(*p[:3], b, s, h, heads, 1, p[3], None, None) == NULL
    assert L.bpt_attention_lse(*p[:3], b, s, h, heads, 1, p[3], p[3], None) == ALIAS
    # layer backward: the recomputed forward, the gradients on the way, the FFN chunk buffers
    need = L.bpt_layer_backward_workspace_bytes(b, s, h, heads, f)
    act, act32, stat = up(rows * h * 2), up(rows * h * 4), up(b * heads * s * 4)
    ffn_ws = L.bpt_ffn_backward_workspace_bytes(rows, h, f, 0)
    assert need == 7 * act + 2 * act32 + 2 * stat + up(rows * 3 * h * 2) + ffn_ws  # Q K V O hb dhb dO
    for bad in (0, 32, 100):
        assert L.bpt_layer_backward_workspace_bytes(b, s, h, heads, bad) == 0
    q = fake_ptrs(20)
    assert L.bpt_layer_backward(*q[:10], b, s, h, heads, 100, 1, *q[10:19], q[19], need, None) == SHAPE
    assert L.bpt_layer_backward(*q[:10], b, s, h, heads, f, 1, *q[10:19], q[19], need - 1, None) == NOMEM
    assert L.bpt_layer_backward(*q[:9], None, b, s, h, heads, f, 1, *q[10:19], q[19], need, None) == NULL
    assert L.bpt_layer_backward(*q[:10], b, s, h, heads, f, 1, q[0], *q[11:19], q[19], need, None) == ALIAS


def test_saved_forward_and_backward_entries_validate_before_touching_memory():
    L = bpt.lib()
    b, s, h, heads, f = 2, 256, 256, 2, 512
    rows = b * s
    # forward with saved O and statistics: the layer's own checks, then the two extra buffers
    p = fake_ptrs(13)  # x, 8 weights, out, o_save, lse2_save, (spare)
    w = p[1:9]
    assert L.bpt_layer_forward_save(p[0], *w, b, s, 192, 2, f, 64, 64, 1, p[9], p[10], p[11], None) == SHAPE
    assert L.bpt_layer_forward_save(p[0], *w, b, s, h, heads, f, 64, 64, 1, p[9], None, p[11], None) == NULL
    assert L.bpt_layer_forward_save(p[0], *w, b, s, h, heads, f, 64, 64, 1, p[9], p[10], None, None) == NULL
    assert L.bpt_layer_forward_save(p[0], *w, b, s, h, heads, f, 64, 64, 1, p[9], p[10] + 8, p[11], None) == ALIGN
    assert L.bpt_layer_forward_save(p[0], *w, b, s, h, heads, f, 64, 64, 1, p[9], p[9], p[11], None) == ALIAS
    assert L.bpt_layer_forward_save(p[0], *w, b, s, h, heads, f, 64, 64, 1, p[9], p[10], p[10], None) == ALIAS
    assert L.bpt_layer_forward_save(p[0], *w, b, s, h, heads, f, 64, 64, 1, p[9], p[10], p[0], None) == ALIAS
    assert L.bpt_layer_forward_save(p[0], *w, 0, s, h, heads, f, 64, 64, 1, p[9], None, None, None) == OK
    # backward from the saved inputs: the layer backward's checks plus the saved pair
    need = L.bpt_layer_backward_workspace_bytes(b, s, h, heads, f)
    q = fake_ptrs(22)  # x, 8 weights, o_saved, lse2_saved, dy, 9 gradients, workspace
    x, ws_, o, lse, dy, outs, ws = q[0], q[1:9], q[9], q[10], q[11], q[12:21], q[21]
    assert L.bpt_layer_backward_saved(x, *ws_, o, lse, dy, b, s, h, heads, f, 1, *outs, ws, need, None) != NULL
    assert L.bpt_layer_backward_saved(x, *ws_, None, lse, dy, b, s, h, heads, f, 1, *outs, ws, need, None) == NULL
    assert L.bpt_layer_backward_saved(x, *ws_, o, None, dy, b, s, h, heads, f, 1, *outs, ws, need, None) == NULL
    assert L.bpt_layer_backward_saved(x, *ws_, o + 8, lse, dy, b, s, h, heads, f, 1, *outs, ws, need, None) == ALIGN
    assert L.bpt_layer_backward_saved(x, *ws_, o, lse, dy, b, s, h, heads, f, 1, o, *outs[1:], ws, need,
                                      None) == ALIAS  # dx over the saved O
    assert L.bpt_layer_backward_saved(x, *ws_, o, lse, dy, b, s, h, heads, f, 1, *outs, lse, need,
                                      None) == ALIAS  # the workspace over the saved statistics
    assert L.bpt_layer_backward_saved(x, *ws_, o, lse, dy, b, s, h, heads, f, 1, *outs, ws, need - 1, None) == NOMEM
