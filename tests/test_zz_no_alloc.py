"""bpt_layer_forward_noalloc: the layer forward for callers that cannot allocate.

Some callers cannot call cudaMalloc (or any allocator) while they run, for
instance code inside an inference engine's execute hook where allocation is
forbidden, or a process whose device memory another manager reserved up front,
and they cannot lend the library a workspace either. For them the library
keeps one fixed scratch array in its own device memory. These tests call that
entry point through the C ABI and check that it gives, bit for bit, the result
of the allocating entry point (the same kernels on the same inputs), on two
calls in a row with different problems (so the second call cannot pass on
what the first one left in the shared scratch), that the first result is the
fp64 oracle's layer within the parity tolerance, and that a problem too large
for the scratch is refused before anything runs.
This file is collected last so that a failure here never hides another test.
"""

import ctypes

import numpy as np
import pytest
import torch

import blockwise_attn_ffn_bpt_b200 as bpt
import bpt_inputs as bi
import oracle

STATIC_WORKSPACE_BYTES = 64 << 20  # BPT_STATIC_WORKSPACE_BYTES in include/bpt.h
MAX_ABS = 2e-2
REL_L2 = 1e-2


def noalloc_fn():
    f = bpt.lib().bpt_layer_forward_noalloc
    f.restype = ctypes.c_int
    f.argtypes = [ctypes.c_void_p] * 9 + [ctypes.c_int] * 7 + [ctypes.c_void_p, ctypes.c_void_p]
    return f


def call_noalloc(shape, x, params, out, stream):
    ptrs = [x.data_ptr()] + [params[k].data_ptr() for k in bi.PARAM_NAMES]
    return noalloc_fn()(*ptrs, shape.b, shape.s, shape.h, shape.heads, shape.q_block, shape.kv_block,
                        int(shape.causal), out.data_ptr(), stream.cuda_stream)


@pytest.mark.gpu
def test_noalloc_matches_the_allocating_entry_point_on_two_calls_in_a_row():
    cases = [
        (bi.LayerShape(2, 1024, 512, 4, 128, 256, True), 0),
        (bi.LayerShape(1, 640, 256, 2, 64, 128, False), 1),
    ]
    stream = torch.cuda.current_stream()
    prepared = []
    for shape, seed in cases:
        need = bpt.workspace_bytes(bpt.BPT_DTYPE_BF16, shape.b, shape.s, shape.h, shape.heads, shape.q_block,
                                   shape.kv_block)
        assert 0 < need <= STATIC_WORKSPACE_BYTES
        inp = bi.make_inputs(shape, seed=seed)
        x = bi.to_torch(inp["x"])
        params = {k: bi.to_torch(inp[k]) for k in bi.PARAM_NAMES}
        ref = bpt.layer_forward(x, params, shape.heads, shape.q_block, shape.kv_block, shape.causal)
        out = torch.full((shape.b, shape.s, shape.h), float("nan"), dtype=torch.float32, device="cuda")
        prepared.append((shape, inp, x, params, ref, out))
    torch.cuda.synchronize()

    # the two calls, back to back on one stream
    for shape, _, x, params, _, out in prepared:
        assert call_noalloc(shape, x, params, out, stream) == 0
    torch.cuda.synchronize()
    assert bpt.stream_status(stream) == 0

    # the same kernels on the same inputs with the same wave plan: the result
    # is the allocating entry point's, bit for bit
    for shape, _, _, _, ref, out in prepared:
        assert torch.equal(out, ref), f"{shape}: differs from bpt_layer_forward"

    # and it is the layer: the first case against the fp64 oracle
    shape, inp, _, _, _, out = prepared[0]
    exp = oracle.layer_forward(*bi.oracle_args(inp), heads=shape.heads, causal=shape.causal)
    got = out.cpu().numpy().astype(np.float64)
    d = got - exp
    max_abs = float(np.abs(d).max())
    rel_l2 = float(np.linalg.norm(d) / np.linalg.norm(exp))
    assert max_abs <= MAX_ABS and rel_l2 <= REL_L2, f"{shape}: max-abs {max_abs:.3e} rel-L2 {rel_l2:.3e}"


def test_noalloc_refuses_a_problem_larger_than_its_scratch():
    # b=1, s=8192, h=2048 needs far more than the fixed scratch: refused with
    # BPT_ERR_NOMEM before any CUDA call (fake, aligned pointers are never touched)
    need = bpt.workspace_bytes(bpt.BPT_DTYPE_BF16, 1, 8192, 2048, 16, 512, 512)
    assert need > STATIC_WORKSPACE_BYTES
    base, step = 1 << 40, 1 << 36
    ptrs = [base + i * step for i in range(9)]
    out = base + 20 * step
    rc = noalloc_fn()(*ptrs, 1, 8192, 2048, 16, 512, 512, 1, out, None)
    assert rc == -6
    assert bpt.status_string(rc).startswith("BPT_ERR_NOMEM")
