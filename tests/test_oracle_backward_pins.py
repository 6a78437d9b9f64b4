"""Pins of the backward oracle (oracle/bpt_oracle_backward.py) against things
other than itself: central differences of the forward oracle, torch fp64
autograd of a forward written here with torch's own attention, a conservation
law of the value gradient, and the blockwise gradient equal to the plain one
for every block pair."""

import numpy as np
import pytest
import torch

import oracle
from oracle import bpt_oracle_backward as obb
from tests.test_oracle_pins import divisors, rand_layer

NAMES = ("x", "Wqkv", "bqkv", "Wo", "bo", "W1", "b1", "W2", "b2")


def grads(p, dy, heads, causal, **kw):
    return obb.layer_backward(*(p[k] for k in NAMES), dy, heads=heads, causal=causal, **kw)


def loss(p, dy, heads, causal):
    y = oracle.layer_forward(*(p[k] for k in NAMES), heads=heads, causal=causal, threads=1)
    return float(np.sum(y * dy))


def pre_activations(p, heads, causal):
    q, k, v = oracle.qkv_projection(p["x"], p["Wqkv"], p["bqkv"])
    o = oracle.attention(q, k, v, heads, causal, threads=1)
    hid = p["x"] + o @ p["Wo"] + p["bo"]
    return hid @ p["W1"] + p["b1"]


CASES = [(1, 3, 4, 2, 8, 3), (2, 4, 4, 1, 6, 4)]  # b, s, h, heads, ffn width, seed


@pytest.mark.parametrize("b,s,h,heads,f,seed", CASES)
@pytest.mark.parametrize("causal", [False, True])
def test_gradients_match_central_differences(b, s, h, heads, f, seed, causal):
    p = rand_layer(b, s, h, heads, seed=seed, f=f)
    dy = np.random.default_rng(seed + 100).standard_normal((b, s, h))
    # no ReLU pre-activation within reach of the step, so the loss is smooth there
    assert np.abs(pre_activations(p, heads, causal)).min() > 1e-4
    g = grads(p, dy, heads, causal)
    eps = 1e-6
    for name in NAMES:
        arr = p[name]
        num = np.zeros_like(arr)
        for idx in np.ndindex(arr.shape):
            old = arr[idx]
            arr[idx] = old + eps
            up = loss(p, dy, heads, causal)
            arr[idx] = old - eps
            down = loss(p, dy, heads, causal)
            arr[idx] = old
            num[idx] = (up - down) / (2 * eps)
        np.testing.assert_allclose(g["d" + name], num, rtol=1e-6, atol=1e-7, err_msg=name)


def torch_layer(p, heads, causal):
    """The layer in torch (fp64), attention by torch's scaled_dot_product_attention."""
    x = p["x"]
    b, s, h = x.shape
    dh = h // heads
    q, k, v = (x @ p["Wqkv"] + p["bqkv"]).split(h, dim=-1)

    def split(z):
        return z.reshape(b, s, heads, dh).transpose(1, 2)

    o = torch.nn.functional.scaled_dot_product_attention(split(q), split(k), split(v), is_causal=causal)
    o = o.transpose(1, 2).reshape(b, s, h)
    hid = x + o @ p["Wo"] + p["bo"]
    return hid + torch.relu(hid @ p["W1"] + p["b1"]) @ p["W2"] + p["b2"]


@pytest.mark.parametrize("b,s,h,heads,f", [(1, 5, 8, 2, 32), (2, 7, 16, 4, 24), (1, 16, 8, 1, 16)])
@pytest.mark.parametrize("causal", [False, True])
def test_gradients_match_torch_autograd(b, s, h, heads, f, causal):
    p = rand_layer(b, s, h, heads, seed=s + h, f=f)
    dy = np.random.default_rng(7).standard_normal((b, s, h))
    tp = {k: torch.tensor(v, dtype=torch.float64, requires_grad=True) for k, v in p.items()}
    y = torch_layer(tp, heads, causal)
    (y * torch.tensor(dy)).sum().backward()
    g = grads(p, dy, heads, causal)
    for name in NAMES:
        np.testing.assert_allclose(g["d" + name], tp[name].grad.numpy(), rtol=1e-9, atol=1e-10, err_msg=name)


@pytest.mark.parametrize("causal", [False, True])
def test_value_gradient_conserves_the_output_gradient(causal):
    # every row of P sums to 1, so per head the key rows of dV = P^T dO add up
    # to the query rows of dO
    rng = np.random.default_rng(3)
    Q, K, V, dO = (rng.standard_normal((2, 9, 8)) for _ in range(4))
    _, _, dV = obb.attention_backward(Q, K, V, dO, heads=2, causal=causal)
    np.testing.assert_allclose(dV.sum(axis=1), dO.sum(axis=1), rtol=0, atol=1e-12)


@pytest.mark.parametrize("s", [1, 2, 3, 8, 12])
@pytest.mark.parametrize("causal", [False, True])
def test_blockwise_attention_backward_equals_plain(s, causal):
    rng = np.random.default_rng(s)
    Q, K, V, dO = (rng.standard_normal((2, s, 8)) for _ in range(4))
    ref = obb.attention_backward(Q, K, V, dO, heads=2, causal=causal)
    for qb in divisors(s):
        for kb in divisors(s):
            got = obb.attention_backward_blockwise(Q, K, V, dO, heads=2, causal=causal, q_block=qb, kv_block=kb)
            for a, r in zip(got, ref):
                np.testing.assert_allclose(a, r, rtol=0, atol=1e-12)


def test_layer_backward_blockwise_equals_plain():
    p = rand_layer(2, 8, 8, 2, seed=11)
    dy = np.random.default_rng(12).standard_normal((2, 8, 8))
    ref = grads(p, dy, 2, True)
    got = grads(p, dy, 2, True, q_block=4, kv_block=2)
    for name in NAMES:
        np.testing.assert_allclose(got["d" + name], ref["d" + name], rtol=0, atol=1e-12, err_msg=name)


# ---------------------------------------------------------------------------
# the FFN block alone (ffn_backward): pinned to central differences of the
# forward oracle's FFN-with-residual (residual_ffn with O = 0, Wo = 0, bo = 0
# gives y = hid + max(0, hid W1 + b1) W2 + b2), and to torch fp64 autograd
# ---------------------------------------------------------------------------

def ffn_forward(hid, W1, b1, W2, b2):
    z = np.zeros_like(hid)
    return oracle.residual_ffn(hid, z, np.zeros((hid.shape[-1], hid.shape[-1])), np.zeros(hid.shape[-1]),
                               W1, b1, W2, b2)


@pytest.mark.parametrize("rows,h,f,seed", [(5, 4, 8, 1), (7, 6, 3, 2), (1, 3, 5, 3)])
def test_ffn_backward_matches_central_differences(rows, h, f, seed):
    rng = np.random.default_rng(seed)
    hid = rng.standard_normal((rows, h))
    W1, b1 = rng.standard_normal((h, f)), rng.standard_normal(f)
    W2, b2 = rng.standard_normal((f, h)), rng.standard_normal(h)
    dy = rng.standard_normal((rows, h))
    assert np.abs(hid @ W1 + b1).min() > 1e-4  # away from the ReLU kink
    g = obb.ffn_backward(hid, W1, b1, W2, dy)
    params = {"hid": hid, "W1": W1, "b1": b1, "W2": W2, "b2": b2}
    eps = 1e-6
    for name, arr in params.items():
        num = np.zeros_like(arr)
        for idx in np.ndindex(arr.shape):
            old = arr[idx]
            arr[idx] = old + eps
            up = float(np.sum(ffn_forward(**params) * dy))
            arr[idx] = old - eps
            down = float(np.sum(ffn_forward(**params) * dy))
            arr[idx] = old
            num[idx] = (up - down) / (2 * eps)
        np.testing.assert_allclose(g["d" + name], num, rtol=1e-6, atol=1e-7, err_msg=name)


def test_ffn_backward_matches_torch_autograd():
    rng = np.random.default_rng(11)
    rows, h, f = 37, 16, 48
    t = {k: torch.tensor(v, requires_grad=True) for k, v in {
        "hid": rng.standard_normal((rows, h)), "W1": rng.standard_normal((h, f)) / 4, "b1": rng.standard_normal(f),
        "W2": rng.standard_normal((f, h)) / 7, "b2": rng.standard_normal(h)}.items()}
    dy = rng.standard_normal((rows, h))
    y = t["hid"] + torch.relu(t["hid"] @ t["W1"] + t["b1"]) @ t["W2"] + t["b2"]
    y.backward(torch.tensor(dy))
    g = obb.ffn_backward(*(t[k].detach().numpy() for k in ("hid", "W1", "b1", "W2")), dy)
    for k in ("hid", "W1", "b1", "W2", "b2"):
        np.testing.assert_allclose(g["d" + k], t[k].grad.numpy(), rtol=1e-10, atol=1e-10, err_msg=k)


@pytest.mark.parametrize("causal", [False, True])
def test_row_lse_of_zero_queries_is_the_log_of_the_key_count(causal):
    # all scores 0: each row sums exp(0) once per visible key (closed form)
    b, s, h, heads = 2, 7, 8, 2
    rng = np.random.default_rng(5)
    Q, K = np.zeros((b, s, h)), rng.standard_normal((b, s, h))
    lse = obb.attention_row_lse2(Q, K, heads, causal)
    count = np.arange(1, s + 1) if causal else np.full(s, s)
    assert np.allclose(lse, np.broadcast_to(np.log2(count), (b, heads, s)), rtol=0, atol=1e-12)


def test_row_lse_of_the_first_causal_row_is_its_own_score():
    # causal row 0 sees key 0 alone: log2 exp(S_00) = S_00 log2(e)
    b, s, h, heads = 1, 5, 8, 2
    rng = np.random.default_rng(6)
    Q, K = rng.standard_normal((b, s, h)), rng.standard_normal((b, s, h))
    lse = obb.attention_row_lse2(Q, K, heads, True)
    for k in range(heads):
        c = slice(k * 4, (k + 1) * 4)
        s00 = float(Q[0, 0, c] @ K[0, 0, c]) / 2.0
        assert abs(lse[0, k, 0] - s00 / np.log(2.0)) < 1e-12


@pytest.mark.parametrize("causal", [False, True])
def test_row_lse_recovers_the_attention_weights_of_torch(causal):
    # exp(S - lse) reproduces torch's own softmax of the masked scores, row by row
    b, s, h, heads = 2, 6, 8, 2
    rng = np.random.default_rng(7)
    Q, K = rng.standard_normal((b, s, h)) * 2.0, rng.standard_normal((b, s, h))
    lse = obb.attention_row_lse2(Q, K, heads, causal)
    for k in range(heads):
        c = slice(k * 4, (k + 1) * 4)
        S = torch.tensor(Q[..., c]) @ torch.tensor(K[..., c]).transpose(-1, -2) / 2.0
        if causal:
            S = S.masked_fill(torch.triu(torch.ones(s, s, dtype=torch.bool), 1), float("-inf"))
        P = torch.softmax(S, dim=-1).numpy()
        P2 = np.where(np.isfinite(S.numpy()), np.exp2(S.numpy() / np.log(2.0) - lse[:, k, :, None]), 0.0)
        assert np.allclose(P2, P, rtol=1e-12, atol=1e-15)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("s,block", [(13, 4), (40, 16), (40, 40), (40, 64)])
def test_sampled_gradient_rows_equal_the_plain_gradient(s, block, causal):
    # the row-sampled gradient of one head (blocks of whole query rows, ragged
    # last block) is the plain gradient's rows, every row of either kind
    rng = np.random.default_rng(s + block)
    dh = 8
    Q, K, V, dO = (rng.standard_normal((1, s, dh)) for _ in range(4))
    dQ, dK, dV = obb.attention_backward(Q, K, V, dO, heads=1, causal=causal)
    rows = np.arange(s)[::-1]
    gq, gk, gv = obb.attention_backward_rows(Q[0], K[0], V[0], dO[0], causal, rows, rows[:5], block=block)
    np.testing.assert_allclose(gq, dQ[0, rows], rtol=0, atol=1e-12)
    np.testing.assert_allclose(gk, dK[0, rows[:5]], rtol=0, atol=1e-12)
    np.testing.assert_allclose(gv, dV[0, rows[:5]], rtol=0, atol=1e-12)


def test_sampled_gradient_rows_match_torch_autograd():
    # against PyTorch's autograd of its own attention (fp64), causal
    s, dh = 50, 16
    rng = np.random.default_rng(3)
    Q, K, V, dO = (rng.standard_normal((s, dh)) for _ in range(4))
    q, k, v = (torch.tensor(a, requires_grad=True) for a in (Q, K, V))
    o = torch.nn.functional.scaled_dot_product_attention(q[None], k[None], v[None], is_causal=True)[0]
    o.backward(torch.tensor(dO))
    rows = [0, 7, 31, 49]
    gq, gk, gv = obb.attention_backward_rows(Q, K, V, dO, True, rows, rows, block=16)
    np.testing.assert_allclose(gq, q.grad.numpy()[rows], rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(gk, k.grad.numpy()[rows], rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(gv, v.grad.numpy()[rows], rtol=1e-10, atol=1e-12)


def test_sampled_ffn_gradients_equal_the_whole_gradients():
    # the row/column-sampled FFN gradients are the corresponding parts of ffn_backward's
    rng = np.random.default_rng(11)
    R, h, f = 37, 16, 24
    hid, dy = rng.standard_normal((R, h)), rng.standard_normal((R, h))
    W1, b1, W2 = rng.standard_normal((h, f)) / 4, rng.standard_normal(f) * 0.1, rng.standard_normal((f, h)) / 5
    full = obb.ffn_backward(hid, W1, b1, W2, dy)
    rows, fc, hc = [0, 5, 36], [1, 7, 23], [0, 15, 3]
    got = obb.ffn_backward_samples(hid, W1, b1, W2, dy, rows, fc, hc)
    np.testing.assert_allclose(got["dhid"], full["dhid"][rows], rtol=0, atol=1e-12)
    np.testing.assert_allclose(got["dW1"], full["dW1"][:, fc], rtol=0, atol=1e-12)
    np.testing.assert_allclose(got["db1"], full["db1"][fc], rtol=0, atol=1e-12)
    np.testing.assert_allclose(got["dW2"], full["dW2"][np.ix_(fc, hc)], rtol=0, atol=1e-12)
    np.testing.assert_allclose(got["db2"], full["db2"], rtol=0, atol=1e-12)
    np.testing.assert_allclose(got["a_cols"], (hid @ W1 + b1)[:, fc], rtol=0, atol=1e-12)
