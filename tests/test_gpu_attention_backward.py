"""GPU parity of the attention backward (bpt_attention_lse,
bpt_attention_backward) and of the whole layer's backward (bpt_layer_backward)
against the fp64 gradient oracle (oracle.bpt_oracle_backward), through the C
ABI.

Inputs are seeded bf16-representable values, so the oracle sees exactly the
operands the kernels see. Tolerances:

* lse2 (log2 units): |error| <= 4e-3. The forward's row sum adds bf16-rounded
  weights (relative rounding 2^-9 each, in both directions), so log2 of the
  sum is off by at most about 2^-9 / ln 2 = 2.8e-3 and far less on average.
* dQ, dK, dV: relative L2 error <= 1.5e-2 and max-abs error <= 4e-2 of the
  largest reference magnitude. P and dS enter their products as bf16 (2^-9
  relative each), D = rowsum(dO O) is taken from the bf16 O of the forward,
  and the results are rounded to bf16 (2^-9); sums over many keys keep the
  relative error near that. dS = P (dP - D) loses relative precision where dP
  and D nearly cancel, which the max-abs bound (relative to the largest
  gradient, not to each element) absorbs.
* The layer's gradients: each within 1.25x (plus 2e-3) of the relative L2
  error that PyTorch's own autograd of the same layer in bf16 makes against
  the oracle, and below a fixed cap (4e-2; 6e-2 for dW1, db1; 1e-2 for dW2,
  db2). Every gradient passes through several bf16-operand products in a row
  (the recomputed forward, the FFN block, the out-projection, the attention,
  the projection), and the ReLU's mask is decided on a pre-activation computed
  through them, so a bf16 training step lands 2-5% from the fp64 gradients on
  these inputs (measured: PyTorch bf16 autograd 2.2-5.1%, fp32 autograd below
  1e-5). Element-level checks of the parts are the FFN and attention tests.
"""

import numpy as np
import pytest
import torch

import blockwise_attn_ffn_bpt_b200 as bpt
import bpt_inputs as bi
from oracle import bpt_oracle_backward as obb

pytestmark = pytest.mark.gpu


def bf16_normal(seed: int, tensor_id: int, shape, std: float = 1.0) -> np.ndarray:
    n = int(np.prod(shape))
    bits = bi.f32_to_bf16_bits((bi.normal_f64(seed, tensor_id, n) * std).astype(np.float32))
    return bits.reshape(shape)


def rel_errors(got: torch.Tensor, ref: np.ndarray):
    g = got.float().cpu().numpy().astype(np.float64)
    assert np.isfinite(g).all()
    d = g - ref
    rl2 = float(np.linalg.norm(d) / max(np.linalg.norm(ref), 1e-300))
    mx = float(np.abs(d).max() / max(np.abs(ref).max(), 1e-300))
    return rl2, mx


def qkvo(b, s, h, seed):
    bits = {name: bf16_normal(seed, 60 + i, (b, s, h)) for i, name in enumerate(("q", "k", "v", "dO"))}
    return bits, {k: bi.to_torch(v) for k, v in bits.items()}, {k: bi.to_f64(v) for k, v in bits.items()}


ATT_CASES = [  # b, s, h, heads, causal
    (1, 256, 256, 2, True),     # dh 128, two tiles
    (2, 200, 128, 2, False),    # dh 64, ragged second tile
    (1, 384, 512, 4, True),     # dh 128, three tiles
    (1, 640, 256, 4, True),     # dh 64, five tiles
    (3, 130, 256, 2, False),    # dh 128, a two-row tail tile
]


@pytest.mark.parametrize("b,s,h,heads,causal", ATT_CASES)
def test_forward_lse_matches_the_oracle_and_leaves_o_unchanged(b, s, h, heads, causal):
    _, t, f = qkvo(b, s, h, seed=b * 1000 + s)
    o, lse2 = bpt.attention_lse(t["q"], t["k"], t["v"], heads, causal)
    o_plain = bpt.attention(t["q"], t["k"], t["v"], heads, s, s, causal)
    torch.cuda.synchronize()
    assert bpt.stream_status() == 0
    assert torch.equal(o, o_plain)
    ref = obb.attention_row_lse2(f["q"], f["k"], heads, causal)
    err = np.abs(lse2.cpu().numpy().astype(np.float64) - ref).max()
    assert err <= 4e-3, f"lse2 max error {err:.3e}"


@pytest.mark.parametrize("b,s,h,heads,causal", ATT_CASES)
def test_attention_backward_matches_the_gradient_oracle(b, s, h, heads, causal):
    _, t, f = qkvo(b, s, h, seed=b * 1000 + s)
    o, lse2 = bpt.attention_lse(t["q"], t["k"], t["v"], heads, causal)
    g = bpt.attention_backward(t["q"], t["k"], t["v"], o, t["dO"], lse2, heads, causal)
    torch.cuda.synchronize()
    assert bpt.stream_status() == 0
    dQ, dK, dV = obb.attention_backward(f["q"], f["k"], f["v"], f["dO"], heads, causal)
    for name, got, ref in (("dq", g["dq"], dQ), ("dk", g["dk"], dK), ("dv", g["dv"], dV)):
        rl2, mx = rel_errors(got, ref)
        assert rl2 <= 1.5e-2 and mx <= 4e-2, f"{name} b={b} s={s} h={h} heads={heads}: rel-L2 {rl2:.3e}, max {mx:.3e}"


def test_attention_backward_value_gradient_conserves_the_output_gradient():
    # every row of P sums to 1, so the column sums of dV = P^T dO equal those of dO
    b, s, h, heads = 1, 512, 256, 2
    _, t, f = qkvo(b, s, h, seed=77)
    o, lse2 = bpt.attention_lse(t["q"], t["k"], t["v"], heads, True)
    g = bpt.attention_backward(t["q"], t["k"], t["v"], o, t["dO"], lse2, heads, True)
    torch.cuda.synchronize()
    got = g["dv"].double().sum(dim=1).cpu().numpy()
    want = f["dO"].sum(axis=1)
    assert np.abs(got - want).max() <= 2e-2 * np.abs(want).max() + 0.5


LAYER_CASES = [  # b, s, h, heads, ffn, causal
    (1, 256, 256, 2, 512, True),
    (2, 192, 128, 2, 256, False),
]


@pytest.mark.parametrize("b,s,h,heads,f,causal", LAYER_CASES)
def test_layer_backward_matches_the_gradient_oracle(b, s, h, heads, f, causal):
    shape = bi.LayerShape(b, s, h, heads, s, s, causal, "bf16", ffn=f)
    inp = bi.make_inputs(shape, seed=s + h)
    dy_bits = bf16_normal(s + h, 41, (b, s, h))
    params = {k: bi.to_torch(inp[k]) for k in ("Wqkv", "bqkv", "Wo", "bo", "W1", "b1", "W2", "b2")}
    x = bi.to_torch(inp["x"])
    dy64 = bi.to_f64(dy_bits)
    g = bpt.layer_backward(x, params, torch.tensor(dy64, dtype=torch.float32, device="cuda"), heads, causal)
    torch.cuda.synchronize()
    assert bpt.stream_status() == 0
    args = bi.oracle_args(inp)
    ref = obb.layer_backward(*args, dy64, heads=heads, causal=causal)
    base = torch_bf16_layer_grads(x, params, torch.tensor(dy64, dtype=torch.float32, device="cuda"), heads, causal)
    caps = {"dW1": 6e-2, "db1": 6e-2, "dW2": 1e-2, "db2": 1e-2}
    for name in ("dx", "dWqkv", "dbqkv", "dWo", "dbo", "dW1", "db1", "dW2", "db2"):
        rl2, mx = rel_errors(g[name], ref[name])
        rl2_bf16, _ = rel_errors(base[name], ref[name])
        assert rl2 <= min(caps.get(name, 4e-2), 1.25 * rl2_bf16 + 2e-3), \
            f"{name} b={b} s={s} h={h}: rel-L2 {rl2:.3e} (bf16 autograd {rl2_bf16:.3e}, max {mx:.3e})"


def torch_bf16_layer_grads(x, params, dy, heads, causal):
    """The same layer's gradients by PyTorch autograd in bf16: the yardstick of
    what bf16 arithmetic reaches against the fp64 oracle."""
    b, s, h = x.shape
    dh = h // heads
    xx = x.detach().clone().requires_grad_(True)
    P = {k: v.detach().clone().requires_grad_(True) for k, v in params.items()}
    q, k, v = (xx @ P["Wqkv"] + P["bqkv"]).split(h, dim=-1)
    heads_of = lambda t: t.view(b, s, heads, dh).transpose(1, 2)
    o = torch.nn.functional.scaled_dot_product_attention(heads_of(q), heads_of(k), heads_of(v), is_causal=causal)
    hid = xx + o.transpose(1, 2).reshape(b, s, h) @ P["Wo"] + P["bo"]
    y = hid + torch.relu(hid @ P["W1"] + P["b1"]) @ P["W2"] + P["b2"]
    y.backward(dy.to(torch.bfloat16))
    return {"dx": xx.grad, **{"d" + name: t.grad for name, t in P.items()}}


def test_attention_backward_full_size_sampled_rows():
    # The 7B-class shape of the layer benchmarks (b1 s32768 h4096, 32 heads of 128,
    # causal: 256 key tiles, the dQ of a query tile summed from up to 256 partials,
    # dK and dV of key tile 0 over 256 query tiles). Rows of one head against the
    # row oracle, which takes every query row's softmax over all of its keys:
    # first, last and tile-edge rows of both kinds and a few inside.
    b, s, h, heads = 1, 32768, 4096, 32
    bits = {name: bf16_normal(11, 70 + i, (b, s, h)) for i, name in enumerate(("q", "k", "v", "dO"))}
    t = {k: bi.to_torch(v) for k, v in bits.items()}
    o, lse2 = bpt.attention_lse(t["q"], t["k"], t["v"], heads, True)
    g = bpt.attention_backward(t["q"], t["k"], t["v"], o, t["dO"], lse2, heads, True)
    torch.cuda.synchronize()
    assert bpt.stream_status() == 0
    head = 13
    c = slice(head * 128, (head + 1) * 128)
    f = {k: bi.to_f64(v[0, :, c]) for k, v in bits.items()}
    qr = [0, 1, 127, 128, 4095, 16383, 16384, 24577, 32766, 32767]
    kr = [0, 1, 127, 128, 8191, 16384, 30000, 32640, 32767]
    dQ, dK, dV = obb.attention_backward_rows(f["q"], f["k"], f["v"], f["dO"], True, qr, kr)
    for name, got, ref in (("dq", g["dq"][0, qr, c], dQ), ("dk", g["dk"][0, kr, c], dK), ("dv", g["dv"][0, kr, c], dV)):
        rl2, mx = rel_errors(got, ref)
        assert rl2 <= 1.5e-2 and mx <= 4e-2, f"{name} (s {s}, head {head}): rel-L2 {rl2:.3e}, max {mx:.3e}"


@pytest.mark.parametrize("b,s,h,heads,f,causal", LAYER_CASES + [(1, 1024, 256, 2, 1024, True)])
def test_layer_backward_from_saved_inputs_equals_the_rematerialising_backward(b, s, h, heads, f, causal):
    # the forward that keeps O and each row's log-sum-exp gives the same output
    # as the plain forward; the backward from them gives the same gradients, bit
    # for bit, as the backward that recomputes the attention (same kernels, same
    # operands)
    shape = bi.LayerShape(b, s, h, heads, s, s, causal, "bf16", ffn=f)
    inp = bi.make_inputs(shape, seed=s + h + 1)
    params = {k: bi.to_torch(inp[k]) for k in ("Wqkv", "bqkv", "Wo", "bo", "W1", "b1", "W2", "b2")}
    x = bi.to_torch(inp["x"])
    dy = torch.tensor(bi.to_f64(bf16_normal(s + h + 1, 41, (b, s, h))), dtype=torch.float32, device="cuda")
    out_s, o, lse2 = bpt.layer_forward_save(x, params, heads, s, s, causal)
    out = bpt.layer_forward(x, params, heads, s, s, causal)
    g_re = bpt.layer_backward(x, params, dy, heads, causal)
    g_sv = bpt.layer_backward(x, params, dy, heads, causal, saved=(o, lse2))
    torch.cuda.synchronize()
    assert bpt.stream_status() == 0
    assert torch.equal(out_s, out)
    for k in g_re:
        assert torch.equal(g_sv[k], g_re[k]), k
