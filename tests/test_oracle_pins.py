"""Pins of the fp64 oracle against things other than itself.

Each test fixes the oracle to something the pages or the mathematics decide:
brute force on tiny inputs (scalar loops written here, not the oracle's code),
closed forms, the exactness of the blockwise algorithm (the BPT paper review
states the blockwise computation is exact, so its output must not depend on the
block sizes), and library special cases (torch's float64
nn.MultiheadAttention and nn.Linear, the validation pattern of the MHSA page,
section 6). test_oracle_mutations.py plants mistakes in the oracle and checks
that these pins catch them.
"""

import itertools
import math

import numpy as np
import pytest
import torch

import bpt_inputs as bi
import oracle


# ---------------------------------------------------------------------------
# helpers
# ---------------------------------------------------------------------------

def rand_layer(b, s, h, heads, seed=0, scale_q=1.0, f=None):
    """Random fp64 layer parameters (plain numpy RNG; exactness tests need no bf16);
    FFN width f (4h unless given)."""
    rng = np.random.default_rng(seed)
    f = 4 * h if f is None else f
    p = dict(
        x=rng.standard_normal((b, s, h)),
        Wqkv=rng.standard_normal((h, 3 * h)) / math.sqrt(h),
        bqkv=rng.standard_normal(3 * h) * 0.1,
        Wo=rng.standard_normal((h, h)) / math.sqrt(h),
        bo=rng.standard_normal(h) * 0.1,
        W1=rng.standard_normal((h, f)) / math.sqrt(h),
        b1=rng.standard_normal(f) * 0.1,
        W2=rng.standard_normal((f, h)) / math.sqrt(f),
        b2=rng.standard_normal(h) * 0.1,
    )
    p["Wqkv"][:, :h] *= scale_q
    return p


def args(p):
    return (p["x"], p["Wqkv"], p["bqkv"], p["Wo"], p["bo"], p["W1"], p["b1"], p["W2"], p["b2"])


def brute_force_layer(p, heads, causal):
    """Scalar-loop restatement of the layer, for tiny shapes only."""
    x = p["x"].tolist()
    b, s, h = len(x), len(x[0]), len(x[0][0])
    dh = h // heads
    f = len(p["b1"])
    Wqkv, bqkv = p["Wqkv"].tolist(), p["bqkv"].tolist()
    Wo, bo, W1, b1, W2, b2 = (p[k].tolist() for k in ("Wo", "bo", "W1", "b1", "W2", "b2"))

    def lin(vec, W, bias, n_out):
        return [bias[j] + sum(vec[i] * W[i][j] for i in range(len(vec))) for j in range(n_out)]

    y = []
    for beta in range(b):
        qkv = [lin(x[beta][t], Wqkv, bqkv, 3 * h) for t in range(s)]
        yb = []
        for t in range(s):
            o = [0.0] * h
            for k in range(heads):
                keys = range(t + 1) if causal else range(s)
                scores = []
                for u in keys:
                    dot = sum(qkv[t][k * dh + d] * qkv[u][h + k * dh + d] for d in range(dh))
                    scores.append(dot / math.sqrt(dh))
                mx = max(scores)
                ex = [math.exp(a - mx) for a in scores]
                tot = sum(ex)
                for d in range(dh):
                    o[k * dh + d] = sum(ex[i] / tot * qkv[u][2 * h + k * dh + d] for i, u in enumerate(keys))
            hid = [x[beta][t][j] + v for j, v in enumerate(lin(o, Wo, bo, h))]
            u1 = [max(0.0, v) for v in lin(hid, W1, b1, f)]
            ff = lin(u1, W2, b2, h)
            yb.append([hid[j] + ff[j] for j in range(h)])
        y.append(yb)
    return np.array(y)


def divisors(n):
    return [d for d in range(1, n + 1) if n % d == 0]


# ---------------------------------------------------------------------------
# brute force
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("b,s,h,heads", [(1, 1, 4, 1), (1, 3, 4, 2), (2, 5, 4, 2), (1, 4, 6, 3)])
@pytest.mark.parametrize("causal", [False, True])
def test_layer_equals_brute_force(b, s, h, heads, causal):
    p = rand_layer(b, s, h, heads, seed=s * 10 + h)
    ref = brute_force_layer(p, heads, causal)
    got = oracle.layer_forward(*args(p), heads=heads, causal=causal, threads=1)
    np.testing.assert_allclose(got, ref, rtol=0, atol=1e-12)


@pytest.mark.parametrize("f", [1, 3, 8, 20])
@pytest.mark.parametrize("causal", [False, True])
def test_layer_equals_brute_force_any_ffn_width(f, causal):
    # the oracle takes the FFN width from W1/W2, so widths other than 4h follow
    # the same definition
    p = rand_layer(2, 3, 4, 2, seed=f, f=f)
    ref = brute_force_layer(p, 2, causal)
    got = oracle.layer_forward(*args(p), heads=2, causal=causal, threads=1)
    np.testing.assert_allclose(got, ref, rtol=0, atol=1e-12)


# ---------------------------------------------------------------------------
# blockwise (Algorithm 1) equals the plain definition, for every block pair
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("s", [1, 2, 3, 8, 16, 64])
@pytest.mark.parametrize("causal", [False, True])
def test_blockwise_equals_naive_all_block_pairs(s, causal):
    b, h, heads = (2 if s <= 16 else 1), 8, 2
    p = rand_layer(b, s, h, heads, seed=s)
    ref = oracle.layer_forward(*args(p), heads=heads, causal=causal, threads=1)
    for qb, kb in itertools.product(divisors(s), divisors(s)):
        if s == 64 and (qb < 8 or kb < 8):
            continue
        got = oracle.layer_forward_blockwise(*args(p), heads=heads, causal=causal,
                                             q_block=qb, kv_block=kb, threads=1)
        np.testing.assert_allclose(got, ref, rtol=0, atol=1e-12, err_msg=f"q_block={qb} kv_block={kb}")


def test_blockwise_large_scores_stay_finite_and_exact():
    # query weights x30: scores of order 1e3, where an unshifted exp overflows
    p = rand_layer(1, 32, 8, 2, seed=5, scale_q=30.0)
    p["x"] *= 3.0
    ref = oracle.layer_forward(*args(p), heads=2, causal=True, threads=1)
    assert np.isfinite(ref).all()
    for qb, kb in [(4, 8), (8, 4), (32, 1), (1, 32)]:
        got = oracle.layer_forward_blockwise(*args(p), heads=2, causal=True, q_block=qb, kv_block=kb, threads=1)
        np.testing.assert_allclose(got, ref, rtol=0, atol=1e-10)
    Q, K, V = oracle.qkv_projection(p["x"], p["Wqkv"], p["bqkv"])
    assert np.abs(Q[..., :4] @ np.swapaxes(K[..., :4], -1, -2)).max() > 500


# ---------------------------------------------------------------------------
# closed forms
# ---------------------------------------------------------------------------

def identity_layer(b, s, h, heads, seed):
    """Zero query weights (uniform attention); Wo = I, value = x, no FFN."""
    p = rand_layer(b, s, h, heads, seed)
    p["Wqkv"][:, :h] = 0.0
    p["bqkv"][:h] = 0.0
    p["Wqkv"][:, 2 * h:] = np.eye(h)
    p["bqkv"][2 * h:] = 0.0
    p["Wo"] = np.eye(h)
    p["bo"][:] = 0.0
    for k in ("W1", "b1", "W2", "b2"):
        p[k][...] = 0.0
    return p


@pytest.mark.parametrize("causal", [False, True])
def test_zero_queries_give_uniform_attention(causal):
    b, s, h, heads = 2, 12, 8, 2
    p = identity_layer(b, s, h, heads, seed=1)
    x = p["x"]
    if causal:
        mean = np.cumsum(x, axis=1) / np.arange(1, s + 1)[None, :, None]
    else:
        mean = np.broadcast_to(x.mean(axis=1, keepdims=True), x.shape)
    # with W1 = b1 = W2 = b2 = 0, out = hid = x + mean(V)
    got = oracle.layer_forward(*args(p), heads=heads, causal=causal, threads=1)
    np.testing.assert_allclose(got, x + mean, rtol=0, atol=1e-13)
    got_b = oracle.layer_forward_blockwise(*args(p), heads=heads, causal=causal, q_block=4, kv_block=3, threads=1)
    np.testing.assert_allclose(got_b, x + mean, rtol=0, atol=1e-13)


def test_attention_rows_sum_to_one():
    # value weights 0 and value bias 1: V == 1, so every attention output is 1
    b, s, h, heads = 2, 10, 8, 4
    p = rand_layer(b, s, h, heads, seed=2, scale_q=5.0)
    p["Wqkv"][:, 2 * h:] = 0.0
    p["bqkv"][2 * h:] = 1.0
    Q, K, V = oracle.qkv_projection(p["x"], p["Wqkv"], p["bqkv"])
    for causal in (False, True):
        O = oracle.attention(Q, K, V, heads, causal, threads=1)
        np.testing.assert_allclose(O, 1.0, rtol=0, atol=1e-14)
        Ob = oracle.attention_blockwise(Q, K, V, heads, causal, 5, 2, threads=1)
        np.testing.assert_allclose(Ob, 1.0, rtol=0, atol=1e-14)


def test_first_causal_row_attends_only_to_itself():
    b, s, h, heads = 1, 9, 8, 2
    p = rand_layer(b, s, h, heads, seed=3, scale_q=4.0)
    Q, K, V = oracle.qkv_projection(p["x"], p["Wqkv"], p["bqkv"])
    O = oracle.attention(Q, K, V, heads, True, threads=1)
    np.testing.assert_allclose(O[:, 0], V[:, 0], rtol=0, atol=1e-15)
    # second row: two-key softmax in closed form, per head
    dh = h // heads
    for k in range(heads):
        c = slice(k * dh, (k + 1) * dh)
        a0 = Q[0, 1, c] @ K[0, 0, c] / math.sqrt(dh)
        a1 = Q[0, 1, c] @ K[0, 1, c] / math.sqrt(dh)
        w1 = 1.0 / (1.0 + math.exp(a0 - a1))
        np.testing.assert_allclose(O[0, 1, c], (1 - w1) * V[0, 0, c] + w1 * V[0, 1, c], rtol=0, atol=1e-14)


def test_zero_values_isolate_the_ffn():
    # V == 0 so O == 0: out = hid + FFN(hid) with hid = x + bo
    b, s, h, heads = 1, 6, 8, 2
    p = rand_layer(b, s, h, heads, seed=4)
    p["Wqkv"][:, 2 * h:] = 0.0
    p["bqkv"][2 * h:] = 0.0
    hid = p["x"] + p["bo"]
    ff = np.zeros_like(hid)
    for t in range(s):
        for j in range(h):
            acc = p["b2"][j]
            for m in range(4 * h):
                pre = p["b1"][m] + sum(hid[0, t, i] * p["W1"][i, m] for i in range(h))
                acc += max(pre, 0.0) * p["W2"][m, j]
            ff[0, t, j] = acc
    got = oracle.layer_forward(*args(p), heads=heads, causal=True, threads=1)
    np.testing.assert_allclose(got, hid + ff, rtol=0, atol=1e-12)


def test_single_token_sequence():
    # s == 1: attention returns V[0] exactly, causal or not
    p = rand_layer(3, 1, 8, 2, seed=6)
    Q, K, V = oracle.qkv_projection(p["x"], p["Wqkv"], p["bqkv"])
    for causal in (False, True):
        np.testing.assert_allclose(oracle.attention(Q, K, V, 2, causal, threads=1), V, rtol=0, atol=1e-15)


# ---------------------------------------------------------------------------
# structure: batch independence, permutation equivariance, row subsets
# ---------------------------------------------------------------------------

def test_batch_items_are_independent():
    p = rand_layer(3, 7, 8, 2, seed=7)
    full = oracle.layer_forward(*args(p), heads=2, causal=True, threads=1)
    for beta in range(3):
        q = dict(p)
        q["x"] = p["x"][beta:beta + 1]
        one = oracle.layer_forward(*args(q), heads=2, causal=True, threads=1)
        np.testing.assert_allclose(full[beta:beta + 1], one, rtol=0, atol=1e-13)


def test_noncausal_is_permutation_equivariant():
    p = rand_layer(1, 11, 8, 2, seed=8)
    perm = np.random.default_rng(0).permutation(11)
    y = oracle.layer_forward(*args(p), heads=2, causal=False, threads=1)
    q = dict(p)
    q["x"] = p["x"][:, perm]
    yp = oracle.layer_forward(*args(q), heads=2, causal=False, threads=1)
    np.testing.assert_allclose(yp, y[:, perm], rtol=0, atol=1e-12)


@pytest.mark.parametrize("causal", [False, True])
def test_row_subset_equals_full_layer(causal):
    p = rand_layer(2, 40, 16, 4, seed=9)
    y = oracle.layer_forward(*args(p), heads=4, causal=causal, threads=2)
    rows = np.array([0, 1, 17, 39, 40, 41, 63, 79])
    got = oracle.layer_rows(*args(p), heads=4, causal=causal, rows=rows, threads=2)
    np.testing.assert_allclose(got, y.reshape(-1, 16)[rows], rtol=0, atol=1e-12)


def test_long_sequence_row_chunking_is_exact():
    # s above the oracle's internal row chunk: result must equal the blockwise path
    p = rand_layer(1, 1100, 8, 1, seed=10)
    Q, K, V = oracle.qkv_projection(p["x"], p["Wqkv"], p["bqkv"])
    O = oracle.attention(Q, K, V, 1, True, threads=1)
    Ob = oracle.attention_blockwise(Q, K, V, 1, True, 100, 275, threads=1)
    np.testing.assert_allclose(O, Ob, rtol=0, atol=1e-12)


# ---------------------------------------------------------------------------
# library special cases (the MHSA page's validation against the official module)
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("b,s,h,heads", [(2, 9, 16, 4), (1, 33, 32, 2)])
def test_attention_matches_torch_multihead_attention(b, s, h, heads, causal):
    p = rand_layer(b, s, h, heads, seed=11, scale_q=3.0)
    mha = torch.nn.MultiheadAttention(h, heads, bias=True, batch_first=True, dtype=torch.float64)
    with torch.no_grad():
        mha.in_proj_weight.copy_(torch.from_numpy(p["Wqkv"].T.copy()))
        mha.in_proj_bias.copy_(torch.from_numpy(p["bqkv"]))
        mha.out_proj.weight.copy_(torch.from_numpy(p["Wo"].T.copy()))
        mha.out_proj.bias.copy_(torch.from_numpy(p["bo"]))
        xt = torch.from_numpy(p["x"])
        mask = torch.triu(torch.ones(s, s, dtype=torch.bool), 1) if causal else None
        ref, _ = mha(xt, xt, xt, attn_mask=mask, need_weights=False)
    Q, K, V = oracle.qkv_projection(p["x"], p["Wqkv"], p["bqkv"])
    O = oracle.attention(Q, K, V, heads, causal, threads=1)
    np.testing.assert_allclose(O @ p["Wo"] + p["bo"], ref.numpy(), rtol=0, atol=1e-13)


def test_ffn_matches_torch_linear_relu_linear():
    p = rand_layer(2, 5, 16, 2, seed=12)
    lin1 = torch.nn.Linear(16, 64, dtype=torch.float64)
    lin2 = torch.nn.Linear(64, 16, dtype=torch.float64)
    with torch.no_grad():
        lin1.weight.copy_(torch.from_numpy(p["W1"].T.copy()))
        lin1.bias.copy_(torch.from_numpy(p["b1"]))
        lin2.weight.copy_(torch.from_numpy(p["W2"].T.copy()))
        lin2.bias.copy_(torch.from_numpy(p["b2"]))
        hid_t = torch.from_numpy(p["x"])
        ref = hid_t + lin2(torch.relu(lin1(hid_t)))
    zeroO = np.zeros_like(p["x"])
    Wo0 = np.zeros_like(p["Wo"])
    got = oracle.residual_ffn(p["x"], zeroO, Wo0, np.zeros(16), p["W1"], p["b1"], p["W2"], p["b2"])
    np.testing.assert_allclose(got, ref.numpy(), rtol=0, atol=1e-13)


def test_sdpa_matches_oracle_attention_per_head():
    b, s, h, heads = 2, 17, 24, 3
    p = rand_layer(b, s, h, heads, seed=13, scale_q=2.0)
    Q, K, V = oracle.qkv_projection(p["x"], p["Wqkv"], p["bqkv"])
    dh = h // heads
    def split(M):
        return torch.from_numpy(M).view(b, s, heads, dh).transpose(1, 2)
    for causal in (False, True):
        ref = torch.nn.functional.scaled_dot_product_attention(split(Q), split(K), split(V), is_causal=causal)
        ref = ref.transpose(1, 2).reshape(b, s, h).numpy()
        np.testing.assert_allclose(oracle.attention(Q, K, V, heads, causal, threads=1), ref, rtol=0, atol=1e-13)


# ---------------------------------------------------------------------------
# the seeded workload: the oracle runs on generated bf16 inputs
# ---------------------------------------------------------------------------

def test_seeded_small_workload_is_finite_and_block_invariant():
    shp = bi.LayerShape(1, 128, 64, 2, 32, 64, True)
    inp = {k: bi.to_f64(v) for k, v in bi.make_inputs(shp, seed=0).items()}
    a = tuple(inp[k] for k in ("x", "Wqkv", "bqkv", "Wo", "bo", "W1", "b1", "W2", "b2"))
    y = oracle.layer_forward(*a, heads=2, causal=True, threads=2)
    assert np.isfinite(y).all()
    yb = oracle.layer_forward_blockwise(*a, heads=2, causal=True, q_block=32, kv_block=64, threads=2)
    np.testing.assert_allclose(y, yb, rtol=0, atol=1e-12)
