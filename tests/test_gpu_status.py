"""Per-stream device status through the C ABI (bpt_stream_status).

A kernel of the library that gives up a bounded wait records BPT_ERR_TIMEOUT
in the status word of the stream it was launched on. These tests make a wait
run out on purpose with bpt_wait_flag (one thread waits, for a few
milliseconds, on a flag that nothing sets; the wait ends either way, so no
GPU hangs) and check that the status belongs to that stream alone: another
stream neither sees nor clears it, and reading another stream does not wait
for it.
"""

import time

import numpy as np
import pytest
import torch

import blockwise_attn_ffn_bpt_b200 as bpt
import bpt_inputs as bi

pytestmark = pytest.mark.gpu

TIMEOUT = -8


SHAPE = bi.LayerShape(1, 256, 256, 4, 64, 64, True)


def small_layer_inputs():
    """Device inputs of a small layer, copied before any wait is queued (a
    device-wide synchronisation later would wait for the other stream)."""
    inp = bi.make_inputs(SHAPE, seed=3)
    x = bi.to_torch(inp["x"])
    params = {k: bi.to_torch(inp[k]) for k in bi.PARAM_NAMES}
    torch.cuda.synchronize()
    return x, params


def small_layer(x, params, stream):
    return bpt.layer_forward(x, params, SHAPE.heads, SHAPE.q_block, SHAPE.kv_block, SHAPE.causal, stream=stream)


def test_a_status_on_one_stream_is_neither_seen_nor_cleared_through_another():
    a, b = torch.cuda.Stream(), torch.cuda.Stream()
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    x, params = small_layer_inputs()
    assert bpt.stream_status(a) == 0 and bpt.stream_status(b) == 0  # new streams start clean
    bpt.wait_flag(flag, 1, 20_000, stream=a)  # nothing sets the flag: gives up after 20 ms
    out = small_layer(x, params, b)
    assert bpt.stream_status(b) == 0
    assert np.isfinite(out.cpu().numpy()).all()
    assert bpt.stream_status(a) == TIMEOUT
    assert bpt.stream_status(a) == 0  # read once, then cleared
    # a wait whose flag is set records nothing
    flag.fill_(1)
    torch.cuda.synchronize()
    bpt.wait_flag(flag, 1, 1_000_000, stream=a)
    assert bpt.stream_status(a) == 0


def test_reading_one_stream_does_not_wait_for_another():
    a, b = torch.cuda.Stream(), torch.cuda.Stream()
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    x, params = small_layer_inputs()
    assert bpt.stream_status(a) == 0 and bpt.stream_status(b) == 0
    bpt.wait_flag(flag, 1, 2_000_000, stream=a)  # waits up to 2 s for the flag
    small_layer(x, params, b)
    t0 = time.perf_counter()
    assert bpt.stream_status(b) == 0  # synchronises b alone while a still waits
    dt = time.perf_counter() - t0
    with torch.cuda.stream(b):
        flag.fill_(1)  # lets a's wait end well before its limit
    assert bpt.stream_status(a) == 0
    assert dt < 1.0, f"reading stream b took {dt:.2f} s: it waited for stream a"
