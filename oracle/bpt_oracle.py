"""Plain fp64 CPU oracle for one Blockwise Parallel Transformer (BPT) layer forward.

TEST INFRASTRUCTURE ONLY. Only the test suite, the package smoke check and the
benchmark's CPU-baseline leg may import or call this module; the library's
product path never does, and this module imports nothing from it.

What the layer computes (sources are the web pages on the method):

* "Blockwise Parallel Transformer for Large Context Models" (xllm-io paper
  review of arXiv:2305.19370), section 3 "core formulas": standard attention
  softmax(QK^T/sqrt(d))V, the position-wise FFN max(0, xW1+b1)W2+b2, the
  blockwise attention of Eq. 3 with its scaling operation, and the blockwise
  FFN with residuals, Output_i = FFN(Attn_i + x_i) + Attn_i + x_i;
  section 3 "Algorithm 1" (project, split into B_q query blocks and B_kv
  key/value blocks, double loop recording normalisation statistics, rescale,
  FFN and residual per query block); section 5 (bf16 matmul, fp32 accumulate).
* "PyTorch 2.3 multi-head self-attention from QKV to 8 heads" (tqpw.cn),
  sections 1-4: head split of the projected Q/K/V into head_dim-wide column
  groups, scaled dot product per head with masked scores excluded, heads
  concatenated and passed through the output projection.
* "Transformer QKV matrix computation and 3 parallel strategies" (mlqm.cn),
  section 1-2: Q = X W_Q, K = X W_K, V = X W_V with one fused QKV linear.

Readings where the pages are silent or garbled (each is listed in the design
notes of the repository):

* The softmax scale is 1/sqrt(dh), dh = h/heads (standard attention formula;
  Eq. 3 as printed drops it).
* The garbled scaling formula is read as: per key/value block j record the
  block max m_j, the block sum l_j = sum exp(a - m_j) and the block numerator
  n_j = sum exp(a - m_j) v; then with m = max_j m_j the output is
  sum_j exp(m_j - m) n_j / sum_j exp(m_j - m) l_j.
* "Attention(Q_i, K, V)" in the residual formula includes the output
  projection Wo, bo, and the residual adds the layer input block x_i (the
  figure caption: the input block is what gets projected to a query).
* No LayerNorm and no dropout (deterministic forward); FFN width 4h in the
  pages, taken here from the shapes of W1 [h, f] and W2 [f, h], so any f.
* Causal mask: key u is allowed for query t iff u <= t within the same
  sequence; a masked score has weight exactly 0.
* Weights are [in, out] (x @ W); Wqkv's columns are [W_Q | W_K | W_V], and
  head k of each third is the column group k*dh .. k*dh + dh - 1.

Arithmetic is fp64 throughout on the exact values the GPU library receives
(bf16 or fp32 inputs promoted to fp64). A library matmul is used as a step;
rows are independent, so long sequences are processed a chunk of query rows at
a time, which changes no sum.
"""

from __future__ import annotations

import math
import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np

try:  # keep BLAS single-threaded inside the per-head worker threads
    from threadpoolctl import threadpool_limits
except ImportError:  # pragma: no cover
    threadpool_limits = None

_ROW_CHUNK = 1024


# --------------------------------------------------------------------------
# small named steps (tests substitute wrong versions of these to check that
# the pins notice a planted mistake)
# --------------------------------------------------------------------------

def _softmax_scale(dh: int) -> float:
    """1/sqrt(d_k) of the standard attention formula, d_k = head_dim."""
    return 1.0 / math.sqrt(dh)


def _key_allowed(t: np.ndarray, u: np.ndarray, causal: bool) -> np.ndarray:
    """Boolean [len(t), len(u)]: may query position t attend to key position u?"""
    if not causal:
        return np.ones((t.size, u.size), dtype=bool)
    return u[None, :] <= t[:, None]


def _relu(z: np.ndarray) -> np.ndarray:
    """max(0, z) of the position-wise FFN."""
    return np.maximum(z, 0.0)


def _head_cols(k: int, dh: int) -> slice:
    """Columns of head k inside one of the Q, K, V thirds (or inside O)."""
    return slice(k * dh, (k + 1) * dh)


def _threads(n_items: int, threads: int | None) -> int:
    t = threads if threads is not None else (os.cpu_count() or 1)
    return max(1, min(t, n_items))


def _parallel_map(fn, items, threads):
    items = list(items)
    nt = _threads(len(items), threads)
    if nt == 1 or len(items) == 1:
        return [fn(it) for it in items]
    ctx = threadpool_limits(1) if threadpool_limits is not None else None
    try:
        if ctx is not None:
            ctx.__enter__()
        with ThreadPoolExecutor(max_workers=nt) as ex:
            return list(ex.map(fn, items))
    finally:
        if ctx is not None:
            ctx.__exit__(None, None, None)


# --------------------------------------------------------------------------
# Algorithm 1, step 1: projection
# --------------------------------------------------------------------------

def qkv_projection(x: np.ndarray, Wqkv: np.ndarray, bqkv: np.ndarray):
    """Project the input sequence to query, key and value.

    [Q | K | V] = x @ Wqkv + bqkv, x [..., h], Wqkv [h, 3h]. Returns the three
    h-wide thirds (each [..., h]). Algorithm 1 step 1 of the BPT paper review;
    Q = XW_Q, K = XW_K, V = XW_V of the QKV page, section 1.
    """
    h = x.shape[-1]
    qkv = x @ Wqkv + bqkv
    return qkv[..., :h], qkv[..., h:2 * h], qkv[..., 2 * h:]


# --------------------------------------------------------------------------
# standard attention (the plain definition)
# --------------------------------------------------------------------------

def _attention_rows(q_rows, t_idx, K, V, dh, causal):
    """softmax(q K^T / sqrt(dh)) V for query rows q_rows at positions t_idx of one head."""
    u_idx = np.arange(K.shape[0])
    a = (q_rows @ K.T) * _softmax_scale(dh)
    allowed = _key_allowed(t_idx, u_idx, causal)
    a = np.where(allowed, a, -np.inf)
    M = a.max(axis=1, keepdims=True)
    e = np.where(allowed, np.exp(a - M), 0.0)
    w = e / e.sum(axis=1, keepdims=True)
    return w @ V


def attention(Q, K, V, heads: int, causal: bool, threads: int | None = None):
    """Multi-head standard attention; returns the concatenated heads O [b, s, h].

    Per batch item and head k: O_k = softmax(Q_k K_k^T / sqrt(dh)) V_k with the
    causal mask when asked (standard attention formula of the BPT paper review,
    section 3; head split and concatenation of the MHSA page, sections 2-4).
    """
    b, s, h = Q.shape
    dh = h // heads
    O = np.empty_like(Q)

    def work(item):
        beta, k = item
        cols = _head_cols(k, dh)
        Kk, Vk = K[beta, :, cols], V[beta, :, cols]
        for r0 in range(0, s, _ROW_CHUNK):
            r1 = min(s, r0 + _ROW_CHUNK)
            O[beta, r0:r1, cols] = _attention_rows(Q[beta, r0:r1, cols], np.arange(r0, r1), Kk, Vk, dh, causal)

    _parallel_map(work, [(beta, k) for beta in range(b) for k in range(heads)], threads)
    return O


# --------------------------------------------------------------------------
# blockwise attention, Algorithm 1 steps 2-10 with Eq. 3's scaling
# --------------------------------------------------------------------------

def attention_blockwise(Q, K, V, heads: int, causal: bool, q_block: int, kv_block: int,
                        threads: int | None = None):
    """Blockwise attention in the order of Algorithm 1.

    Split the queries into B_q = s/q_block blocks and keys/values into
    B_kv = s/kv_block blocks. For each query block, visit every key/value
    block and record its normalisation statistics (block max m_j, block sum
    l_j, block numerator n_j); then rescale every block by exp(m_j - m) with m
    the max over blocks and combine (Eq. 3 and its scaling operation). A block
    whose entries are all masked for a row contributes nothing to that row.
    """
    b, s, h = Q.shape
    dh = h // heads
    if s % q_block or s % kv_block:
        raise ValueError("s must be a multiple of q_block and kv_block")
    B_q, B_kv = s // q_block, s // kv_block
    scale = _softmax_scale(dh)
    O = np.empty_like(Q)

    def work(item):
        beta, k = item
        cols = _head_cols(k, dh)
        for outer in range(B_q):
            t_idx = np.arange(outer * q_block, (outer + 1) * q_block)
            Qi = Q[beta, t_idx, cols]
            stats = []  # (m_j, l_j, n_j) per key/value block
            for inner in range(B_kv):
                u_idx = np.arange(inner * kv_block, (inner + 1) * kv_block)
                allowed = _key_allowed(t_idx, u_idx, causal)
                a = np.where(allowed, (Qi @ K[beta, u_idx, cols].T) * scale, -np.inf)
                m_j = a.max(axis=1)
                has = np.isfinite(m_j)
                e = np.where(allowed, np.exp(a - np.where(has, m_j, 0.0)[:, None]), 0.0)
                stats.append((m_j, e.sum(axis=1), e @ V[beta, u_idx, cols]))
            m = np.max(np.stack([st[0] for st in stats]), axis=0)
            num = np.zeros((q_block, dh))
            den = np.zeros(q_block)
            for m_j, l_j, n_j in stats:
                c = np.where(np.isfinite(m_j), np.exp(m_j - m), 0.0)
                num += c[:, None] * n_j
                den += c * l_j
            O[beta, t_idx, cols] = num / den[:, None]

    _parallel_map(work, [(beta, k) for beta in range(b) for k in range(heads)], threads)
    return O


# --------------------------------------------------------------------------
# output projection, residuals and the position-wise FFN
# --------------------------------------------------------------------------

def residual_ffn(x, O, Wo, bo, W1, b1, W2, b2):
    """Output_i = FFN(A_i + x_i) + A_i + x_i with A_i = O_i Wo + bo.

    hid = x + O @ Wo + bo (first residual), then
    y = hid + max(0, hid @ W1 + b1) @ W2 + b2 (FFN and second residual);
    blockwise FFN formula and standard FFN of the BPT paper review, section 3.
    """
    hid = x + (O @ Wo + bo)
    return hid + (_relu(hid @ W1 + b1) @ W2 + b2)


# --------------------------------------------------------------------------
# whole layer
# --------------------------------------------------------------------------

def layer_forward(x, Wqkv, bqkv, Wo, bo, W1, b1, W2, b2, heads: int, causal: bool,
                  threads: int | None = None):
    """The layer by its plain definition: y [b, s, h] in fp64."""
    Q, K, V = qkv_projection(x, Wqkv, bqkv)
    O = attention(Q, K, V, heads, causal, threads)
    return residual_ffn(x, O, Wo, bo, W1, b1, W2, b2)


def layer_forward_blockwise(x, Wqkv, bqkv, Wo, bo, W1, b1, W2, b2, heads: int, causal: bool,
                            q_block: int, kv_block: int, threads: int | None = None):
    """The layer in Algorithm 1's order: attention per query block, then the
    FFN and residuals applied to that block (step 11)."""
    b, s, h = x.shape
    Q, K, V = qkv_projection(x, Wqkv, bqkv)
    O = attention_blockwise(Q, K, V, heads, causal, q_block, kv_block, threads)
    y = np.empty_like(x)
    for outer in range(s // q_block):
        rows = slice(outer * q_block, (outer + 1) * q_block)
        y[:, rows] = residual_ffn(x[:, rows], O[:, rows], Wo, bo, W1, b1, W2, b2)
    return y


def layer_rows(x, Wqkv, bqkv, Wo, bo, W1, b1, W2, b2, heads: int, causal: bool,
               rows, threads: int | None = None):
    """y at selected rows only, by the plain definition.

    rows: flat indices beta*s + t. Keys and values are projected only for the
    positions those rows can attend to (all of the sequence when not causal,
    positions 0..t when causal). Returns [len(rows), h].
    """
    b, s, h = x.shape
    dh = h // heads
    rows = np.asarray(rows, dtype=np.int64)
    out = np.empty((rows.size, h))
    Wq, Wkv = Wqkv[:, :h], Wqkv[:, h:]
    bq, bkv = bqkv[:h], bqkv[h:]
    for beta in np.unique(rows // s):
        sel = np.nonzero(rows // s == beta)[0]
        t_idx = rows[sel] % s
        n_keys = s if not causal else int(t_idx.max()) + 1
        KV = x[beta, :n_keys] @ Wkv + bkv
        Kb, Vb = KV[:, :h], KV[:, h:]
        xq = x[beta, t_idx]
        Qr = xq @ Wq + bq
        O = np.empty((t_idx.size, h))

        def work(k):
            cols = _head_cols(k, dh)
            O[:, cols] = _attention_rows(Qr[:, cols], t_idx, Kb[:, cols], Vb[:, cols], dh, causal)

        _parallel_map(work, range(heads), threads)
        out[sel] = residual_ffn(xq, O, Wo, bo, W1, b1, W2, b2)
    return out
