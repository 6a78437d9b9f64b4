"""Plain fp64 CPU oracle for the gradients of one BPT layer.

TEST INFRASTRUCTURE ONLY, like bpt_oracle: only the test suite may import or
call this module; the library's product path never does, and this module
imports nothing from it.

The pages train their models with the blockwise layer ("Blockwise Parallel
Transformer for Large Context Models" paper review, sections 4-5: language
modelling and reinforcement learning runs, with the blockwise FFN scanned and
rematerialised, section 3 "blockwise FFN" listing). What the backward pass
computes is fixed by the forward: the gradients of the layer's output with
respect to its input and every parameter. `layer_backward` writes that chain
rule out for the forward of bpt_oracle:

    qkv = x Wqkv + bqkv;  S = Q K^T / sqrt(dh) (masked);  P = softmax(S)
    O = P V;  hid = x + O Wo + bo;  a = hid W1 + b1;  u = max(0, a)
    y = hid + u W2 + b2

and, given dy = dL/dy,

    db2 = sum dy;  dW2 = u^T dy;  da = (dy W2^T) [a > 0]
    db1 = sum da;  dW1 = hid^T da;  dhid = dy + da W1^T
    dbo = sum dhid;  dWo = O^T dhid;  dO = dhid Wo^T
    per head: dV = P^T dO;  dP = dO V^T;  dS = P (dP - rowsum(dP P))
              dQ = dS K / sqrt(dh);  dK = dS^T Q / sqrt(dh)
    dqkv = [dQ | dK | dV];  dbqkv = sum dqkv;  dWqkv = x^T dqkv
    dx = dhid + dqkv Wqkv^T

`attention_backward_blockwise` computes the attention part block by block,
the way a blockwise layer trains without storing P: per query block and
key/value block it recomputes P from the forward's row statistics (running
max m and sum l, as Algorithm 1 records them) and accumulates dQ, dK and dV,
using D = rowsum(dO O) in place of rowsum(dP P) (the two are equal). It is
checked equal to the plain gradient for every block pair.
"""

from __future__ import annotations

import numpy as np

from . import bpt_oracle as ob


def _softmax_grad(P: np.ndarray, dP: np.ndarray) -> np.ndarray:
    """dS for dP through a row softmax P (the softmax Jacobian applied per row)."""
    return P * (dP - np.sum(dP * P, axis=-1, keepdims=True))


def _relu_grad(a: np.ndarray) -> np.ndarray:
    return (a > 0).astype(a.dtype)


def _value_grad(P: np.ndarray, dO: np.ndarray) -> np.ndarray:
    """dV = P^T dO of one head."""
    return np.swapaxes(P, -1, -2) @ dO


def _qk_grads(dS: np.ndarray, Q: np.ndarray, K: np.ndarray, scale: float):
    """dQ = dS K scale and dK = dS^T Q scale of one head."""
    return (dS @ K) * scale, (np.swapaxes(dS, -1, -2) @ Q) * scale


def _dhid(dy: np.ndarray, da: np.ndarray, W1: np.ndarray) -> np.ndarray:
    """Gradient reaching hid: through the second residual and through the FFN."""
    return dy + da @ W1.T


def _attention_probs(Q, K, dh, causal):
    """Row softmax of the scaled, masked scores of one head: P [.., s, s]."""
    s = Q.shape[-2]
    t = np.arange(s)
    allowed = ob._key_allowed(t, t, causal)
    S = (Q @ np.swapaxes(K, -1, -2)) * ob._softmax_scale(dh)
    S = np.where(allowed, S, -np.inf)
    S = S - S.max(axis=-1, keepdims=True)
    E = np.where(allowed, np.exp(S), 0.0)
    return E / E.sum(axis=-1, keepdims=True)


def attention_row_lse2(Q, K, heads: int, causal: bool) -> np.ndarray:
    """Per query row and head, the log-sum-exp of the row's scaled scores over
    its visible keys, in log2 units: log2 sum_u exp(S_tu) with S = Q K^T /
    sqrt(dh). It is the normalisation statistic of Algorithm 1 (the running max
    m and sum l of a row, taken together as m + log2 l, with m in log2 units),
    from which the backward recomputes P = exp(S - lse). Returns [b, heads, s]."""
    b, s, h = Q.shape
    dh = h // heads
    t = np.arange(s)
    allowed = ob._key_allowed(t, t, causal)
    out = np.zeros((b, heads, s))
    for k in range(heads):
        c = ob._head_cols(k, dh)
        S = np.where(allowed, (Q[..., c] @ np.swapaxes(K[..., c], -1, -2)) * ob._softmax_scale(dh), -np.inf)
        mx = S.max(axis=-1, keepdims=True)
        out[:, k, :] = (mx[..., 0] + np.log(np.exp(S - mx).sum(axis=-1))) / np.log(2.0)
    return out


def attention_backward(Q, K, V, dO, heads: int, causal: bool):
    """dQ, dK, dV [b, s, h] of O = softmax(Q K^T / sqrt(dh)) V per head, by the plain definition."""
    h = Q.shape[-1]
    dh = h // heads
    dQ, dK, dV = np.zeros_like(Q), np.zeros_like(K), np.zeros_like(V)
    for k in range(heads):
        c = ob._head_cols(k, dh)
        P = _attention_probs(Q[..., c], K[..., c], dh, causal)
        dV[..., c] = _value_grad(P, dO[..., c])
        dP = dO[..., c] @ np.swapaxes(V[..., c], -1, -2)
        dS = _softmax_grad(P, dP)
        dQ[..., c], dK[..., c] = _qk_grads(dS, Q[..., c], K[..., c], ob._softmax_scale(dh))
    return dQ, dK, dV


def attention_backward_blockwise(Q, K, V, dO, heads: int, causal: bool, q_block: int, kv_block: int):
    """dQ, dK, dV [b, s, h] block by block from the forward's row statistics.

    Forward statistics per query row (over all of its key/value blocks): the
    max m of the scaled scores and the sum l of exp(score - m); O itself. Then
    for each query block i and key/value block j: P_ij = exp(S_ij - m_i) / l_i
    (0 where masked), dV_j += P_ij^T dO_i, dP_ij = dO_i V_j^T, dS_ij = P_ij
    (dP_ij - D_i) with D_i = rowsum(dO_i O_i), dQ_i += dS_ij K_j scale,
    dK_j += dS_ij^T Q_i scale.
    """
    b, s, h = Q.shape
    if s % q_block or s % kv_block:
        raise ValueError("s must be a multiple of both block sizes")
    dh = h // heads
    scale = ob._softmax_scale(dh)
    dQ, dK, dV = np.zeros_like(Q), np.zeros_like(K), np.zeros_like(V)
    t = np.arange(s)
    for k in range(heads):
        c = ob._head_cols(k, dh)
        q, kk, v, do = Q[..., c], K[..., c], V[..., c], dO[..., c]
        # forward statistics, block by block over the keys
        m = np.full((b, s), -np.inf)
        for j0 in range(0, s, kv_block):
            tj = t[j0:j0 + kv_block]
            Sj = np.where(ob._key_allowed(t, tj, causal), (q @ np.swapaxes(kk[:, j0:j0 + kv_block], -1, -2)) * scale,
                          -np.inf)
            m = np.maximum(m, Sj.max(axis=-1))
        l = np.zeros((b, s))
        o = np.zeros_like(q)
        for j0 in range(0, s, kv_block):
            tj = t[j0:j0 + kv_block]
            allowed = ob._key_allowed(t, tj, causal)
            Sj = (q @ np.swapaxes(kk[:, j0:j0 + kv_block], -1, -2)) * scale
            Ej = np.where(allowed, np.exp(np.where(allowed, Sj, 0.0) - m[..., None]), 0.0)
            l += Ej.sum(axis=-1)
            o += Ej @ v[:, j0:j0 + kv_block]
        o /= l[..., None]
        D = np.sum(do * o, axis=-1)
        for i0 in range(0, s, q_block):
            ti = t[i0:i0 + q_block]
            qi, doi = q[:, i0:i0 + q_block], do[:, i0:i0 + q_block]
            mi, li, Di = m[:, i0:i0 + q_block], l[:, i0:i0 + q_block], D[:, i0:i0 + q_block]
            for j0 in range(0, s, kv_block):
                tj = t[j0:j0 + kv_block]
                allowed = ob._key_allowed(ti, tj, causal)
                kj, vj = kk[:, j0:j0 + kv_block], v[:, j0:j0 + kv_block]
                Sij = (qi @ np.swapaxes(kj, -1, -2)) * scale
                Pij = np.where(allowed, np.exp(np.where(allowed, Sij, 0.0) - mi[..., None]), 0.0) / li[..., None]
                dV[:, j0:j0 + kv_block, c] += np.swapaxes(Pij, -1, -2) @ doi
                dPij = doi @ np.swapaxes(vj, -1, -2)
                dSij = Pij * (dPij - Di[..., None])
                dQ[:, i0:i0 + q_block, c] += (dSij @ kj) * scale
                dK[:, j0:j0 + kv_block, c] += (np.swapaxes(dSij, -1, -2) @ qi) * scale
    return dQ, dK, dV


def attention_backward_rows(q, k, v, do, causal: bool, query_rows, key_rows, block: int = 1024):
    """Selected rows of dQ, dK and dV of one head of one sequence, by the plain
    definition, for sequences too long for the full s x s matrices.

    q, k, v, do are [s, dh]. Returns (dQ[query_rows], dK[key_rows],
    dV[key_rows]). The query rows are visited in blocks of `block` whole rows:
    for each, the scaled and masked scores S = q k^T / sqrt(dh) of all keys, the
    row softmax P (max and sum over the whole row), O = P v and D = rowsum(do O);
    then, with dP = do v^T and dS = P (dP - D) (the softmax Jacobian applied per
    row, D = rowsum(dP P) = rowsum(do O)):
        dV[u] = sum_t P[t, u] do[t],   dK[u] = sum_t dS[t, u] q[t] / sqrt(dh)
    over every query row t (the key rows u taken as columns of each block), and
    dQ[t] = sum_u dS[t, u] k[u] / sqrt(dh) for the selected query rows t of the
    block. Nothing is approximated: each row's softmax sees all of its keys.
    """
    s, dh = q.shape
    scale = ob._softmax_scale(dh)
    query_rows = np.asarray(query_rows, dtype=np.int64)
    key_rows = np.asarray(key_rows, dtype=np.int64)
    u_all = np.arange(s)
    dQ = np.zeros((query_rows.size, dh))
    dK = np.zeros((key_rows.size, dh))
    dV = np.zeros((key_rows.size, dh))
    vJ = v[key_rows]
    for r0 in range(0, s, block):
        t = np.arange(r0, min(s, r0 + block))
        allowed = ob._key_allowed(t, u_all, causal)
        S = np.where(allowed, (q[t] @ k.T) * scale, -np.inf)
        E = np.where(allowed, np.exp(S - S.max(axis=1, keepdims=True)), 0.0)
        P = E / E.sum(axis=1, keepdims=True)
        del S, E
        D = np.sum(do[t] * (P @ v), axis=1)
        # key rows: columns key_rows of P and dS over these query rows
        PJ = P[:, key_rows]
        dSJ = PJ * (do[t] @ vJ.T - D[:, None])
        dV += PJ.T @ do[t]
        dK += (dSJ.T @ q[t]) * scale
        # query rows inside this block: whole rows of dS
        sel = np.nonzero((query_rows >= t[0]) & (query_rows <= t[-1]))[0]
        if sel.size:
            li = query_rows[sel] - r0
            dSI = P[li] * (do[query_rows[sel]] @ v.T - D[li, None])
            dQ[sel] = (dSI @ k) * scale
    return dQ, dK, dV


def ffn_backward(hid, W1, b1, W2, dy) -> dict:
    """Gradients of the FFN block with its residual, y = hid + max(0, hid W1 +
    b1) W2 + b2 (the standard FFN of the BPT paper review, section 3, with the
    second residual of its blockwise FFN formula), for the upstream gradient
    dy: dhid, dW1, db1, dW2, db2. The blockwise FFN is rematerialised in the
    backward pass (paper review section 3, the scanned blockwise FFN):
    u = max(0, a) is recomputed from hid here rather than stored.

        a = hid W1 + b1;  u = max(0, a)
        db2 = sum dy;  dW2 = u^T dy;  da = (dy W2^T) [a > 0]
        db1 = sum da;  dW1 = hid^T da;  dhid = dy + da W1^T
    """
    a = hid @ W1 + b1
    u = ob._relu(a)

    def flat(z):
        return z.reshape(-1, z.shape[-1])

    g = {}
    g["db2"] = flat(dy).sum(axis=0)
    g["dW2"] = flat(u).T @ flat(dy)
    da = (dy @ W2.T) * _relu_grad(a)
    g["db1"] = flat(da).sum(axis=0)
    g["dW1"] = flat(hid).T @ flat(da)
    g["dhid"] = _dhid(dy, da, W1)
    return g


def ffn_backward_samples(hid, W1, b1, W2, dy, rows, f_cols, h_cols) -> dict:
    """Selected parts of ffn_backward's gradients, for problems whose [rows, ffn]
    intermediate is too large to form (hid, dy: [R, h]): rows `rows` of dhid,
    columns `f_cols` of dW1 and db1, the block dW2[f_cols, h_cols], and all of
    db2; plus the pre-activations a = hid W1 + b1 they used (rows `rows`, and
    columns `f_cols` over every row), so that a caller can see where a ReLU
    decision lies within rounding of zero. Same definitions as ffn_backward:
        da = (dy W2^T) [a > 0];  dhid = dy + da W1^T;  dW1 = hid^T da
        db1 = sum da;  dW2 = u^T dy with u = max(0, a);  db2 = sum dy
    taken only over the needed rows or columns of a, u and da.
    """
    rows = np.asarray(rows, dtype=np.int64)
    f_cols = np.asarray(f_cols, dtype=np.int64)
    h_cols = np.asarray(h_cols, dtype=np.int64)
    # rows of dhid need whole rows of da
    a_rows = hid[rows] @ W1 + b1
    da_rows = (dy[rows] @ W2.T) * _relu_grad(a_rows)
    # columns of dW1, db1 and dW2 need whole columns of a (over every row)
    a_cols = hid @ W1[:, f_cols] + b1[f_cols]
    da_cols = (dy @ W2[f_cols].T) * _relu_grad(a_cols)
    u_cols = ob._relu(a_cols)
    return {"dhid": _dhid(dy[rows], da_rows, W1), "dW1": hid.T @ da_cols, "db1": da_cols.sum(axis=0),
            "dW2": u_cols.T @ dy[:, h_cols], "db2": dy.sum(axis=0), "a_rows": a_rows, "a_cols": a_cols}


def layer_backward(x, Wqkv, bqkv, Wo, bo, W1, b1, W2, b2, dy, heads: int, causal: bool,
                   q_block: int | None = None, kv_block: int | None = None) -> dict:
    """Gradients of the layer output y with respect to x and every parameter,
    for the upstream gradient dy [b, s, h]; attention blockwise when both
    block sizes are given. Returns a dict keyed like the arguments: dx, dWqkv,
    dbqkv, dWo, dbo, dW1, db1, dW2, db2."""
    h = x.shape[-1]
    Q, K, V = ob.qkv_projection(x, Wqkv, bqkv)
    O = ob.attention(Q, K, V, heads, causal, threads=1)
    hid = x + O @ Wo + bo

    def flat(z):
        return z.reshape(-1, z.shape[-1])

    g = ffn_backward(hid, W1, b1, W2, dy)
    dhid = g.pop("dhid")
    g["dbo"] = flat(dhid).sum(axis=0)
    g["dWo"] = flat(O).T @ flat(dhid)
    dO = dhid @ Wo.T
    if q_block is not None and kv_block is not None:
        dQ, dK, dV = attention_backward_blockwise(Q, K, V, dO, heads, causal, q_block, kv_block)
    else:
        dQ, dK, dV = attention_backward(Q, K, V, dO, heads, causal)
    dqkv = np.concatenate([dQ, dK, dV], axis=-1)
    g["dbqkv"] = flat(dqkv).sum(axis=0)
    g["dWqkv"] = flat(x).T @ flat(dqkv)
    g["dx"] = dhid + dqkv @ Wqkv.T
    assert g["dx"].shape == x.shape and h == x.shape[-1]
    return g
