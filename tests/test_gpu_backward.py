"""GPU parity of the FFN block's backward (bpt_ffn_backward) against the fp64
gradient oracle (oracle.bpt_oracle_backward.ffn_backward), through the C ABI.

Inputs are seeded and bf16-representable (hid and dy drawn like the layer's
x, the weights like the layer's), so the kernels' rounding of hid and dy to
bf16 operands is exact; what remains is fp32 accumulation and the bf16
rounding of the recomputed intermediate and of da. Tolerance, for each
gradient: relative L2 error <= 1e-2 and max-abs error <= 2e-2 of the largest
reference magnitude (one bf16 rounding of a summand is 2^-9 relative; sums of
many such terms stay near that; a ReLU mask decided differently for a
pre-activation within rounding of zero moves one term of one row).

The ReLU's mask is a decision taken in floating point: where a
pre-activation hid W1 + b1 lies within rounding of zero, the GPU (fp32
accumulation) and the oracle (fp64) may decide it differently, and both are
valid. A differently decided element (r, c) changes da[r, c] by at most
|(dy W2^T)[r, c]|, which moves row r of dhid by that times |W1[:, c]|, column
c of dW1 by that times |hid[r, :]| and db1[c] by that; the elementwise checks
allow exactly that much on top of the tolerance, for every pre-activation with
|hid W1 + b1| < 1e-4 (the fp32 accumulation error of these sums is about
1e-6). The relative L2 bound applies without any allowance.
"""

import numpy as np
import pytest
import torch

import blockwise_attn_ffn_bpt_b200 as bpt
import bpt_inputs as bi
from oracle import bpt_oracle_backward as obb

pytestmark = pytest.mark.gpu

REL_L2 = 1e-2
MAX_REL = 2e-2


def check(got: torch.Tensor, ref: np.ndarray, what: str, slack=0.0):
    g = got.cpu().numpy().astype(np.float64)
    assert np.isfinite(g).all(), f"{what}: non-finite"
    d = g - ref
    rl2 = float(np.linalg.norm(d) / max(np.linalg.norm(ref), 1e-300))
    excess = np.abs(d) - slack
    mx = float(excess.max() / max(np.abs(ref).max(), 1e-300))
    assert rl2 <= REL_L2 and mx <= MAX_REL, f"{what}: rel-L2 {rl2:.3e}, max-abs (beyond the mask slack)/max {mx:.3e}"


def mask_slack(hid64, W1, b1, W2, dy64):
    """Most that differently decided ReLU masks (pre-activations within 1e-4 of
    zero) can move each element of dhid, dW1 and db1."""
    ambiguous = np.abs(hid64 @ W1 + b1) < 1e-4
    da_moves = np.abs(dy64 @ W2.T) * ambiguous  # [rows, ffn]
    return {"dhid": da_moves @ np.abs(W1).T, "dW1": np.abs(hid64).T @ da_moves, "db1": da_moves.sum(axis=0)}


@pytest.mark.parametrize("rows,h,f,chunk", [(1000, 256, 1024, 384), (4096, 512, 2048, 0), (8192, 2048, 8192, 0),
                                            (300, 128, 192, 128)])
def test_ffn_backward_matches_the_gradient_oracle(rows, h, f, chunk):
    shape = bi.LayerShape(1, rows, h, h // 64, 1, 1, False, "bf16", ffn=f)
    inp = bi.make_inputs(shape, seed=rows + h)
    hid_bits = inp["x"].reshape(rows, h)  # bf16 bit patterns, N(0, 1)
    dy_bits = bi.f32_to_bf16_bits(bi.normal_f64(rows + h, 40, rows * h).astype(np.float32)).reshape(rows, h)
    hid64, dy64 = bi.to_f64(hid_bits), bi.to_f64(dy_bits)
    W1, b1, W2 = (bi.to_torch(inp[k]) for k in ("W1", "b1", "W2"))
    g = bpt.ffn_backward(torch.tensor(hid64, dtype=torch.float32, device="cuda"), W1, b1, W2,
                         torch.tensor(dy64, dtype=torch.float32, device="cuda"), chunk_rows=chunk)
    torch.cuda.synchronize()
    assert bpt.stream_status() == 0
    W1_64, b1_64, W2_64 = bi.to_f64(inp["W1"]), bi.to_f64(inp["b1"]), bi.to_f64(inp["W2"])
    ref = obb.ffn_backward(hid64, W1_64, b1_64, W2_64, dy64)
    slack = mask_slack(hid64, W1_64, b1_64, W2_64, dy64)
    for k in ("dhid", "dW1", "db1", "dW2", "db2"):
        check(g[k], ref[k], f"{k} rows={rows} h={h} f={f} chunk={chunk}", slack.get(k, 0.0))


def test_ffn_backward_does_not_depend_on_the_chunk():
    # the chunks only split the sum over rows of the weight gradients
    rows, h, f = 1536, 256, 512
    shape = bi.LayerShape(1, rows, h, 4, 1, 1, False, "bf16", ffn=f)
    inp = bi.make_inputs(shape, seed=3)
    hid = torch.tensor(bi.to_f64(inp["x"].reshape(rows, h)), dtype=torch.float32, device="cuda")
    dy = torch.randn((rows, h), generator=torch.Generator(device="cuda").manual_seed(1), device="cuda")
    W1, b1, W2 = (bi.to_torch(inp[k]) for k in ("W1", "b1", "W2"))
    a = bpt.ffn_backward(hid, W1, b1, W2, dy, chunk_rows=0)
    b = bpt.ffn_backward(hid, W1, b1, W2, dy, chunk_rows=256)
    torch.cuda.synchronize()
    assert torch.equal(a["dhid"], b["dhid"])  # row-local: identical
    for k in ("dW1", "db1", "dW2", "db2"):
        d = (a[k] - b[k]).abs().max().item()
        assert d <= 1e-3 * a[k].abs().max().item(), k


def test_ffn_backward_full_size_sampled():
    # The 7B-class layer's FFN block (rows 32768, h 4096, ffn 16384: two 16384-row
    # chunks, every product on SM pairs): rows of dhid, columns of dW1 and db1, a
    # block of dW2 and all of db2 against the sampled oracle, which forms the
    # pre-activations it needs in fp64 over every row; the first and last rows and
    # columns, the chunk boundary and a few inside.
    rows, h, f = 32768, 4096, 16384
    shape = bi.LayerShape(1, rows, h, h // 128, 1, 1, False, "bf16", ffn=f)
    inp = bi.make_inputs(shape, seed=2024)
    hid64 = bi.to_f64(inp["x"].reshape(rows, h))
    dy64 = bi.to_f64(bi.f32_to_bf16_bits(bi.normal_f64(2024, 40, rows * h).astype(np.float32)).reshape(rows, h))
    W1, b1, W2 = (bi.to_torch(inp[k]) for k in ("W1", "b1", "W2"))
    g = bpt.ffn_backward(torch.tensor(hid64, dtype=torch.float32, device="cuda"), W1, b1, W2,
                         torch.tensor(dy64, dtype=torch.float32, device="cuda"))
    torch.cuda.synchronize()
    assert bpt.stream_status() == 0
    W1_64, b1_64, W2_64 = bi.to_f64(inp["W1"]), bi.to_f64(inp["b1"]), bi.to_f64(inp["W2"])
    rs = np.random.default_rng(5)
    r_s = np.unique(np.concatenate([[0, 1, 16383, 16384, 32767], rs.integers(0, rows, 5)]))
    f_s = np.unique(np.concatenate([[0, 255, 256, 16383], rs.integers(0, f, 3)]))
    h_s = np.unique(np.concatenate([[0, 4095], rs.integers(0, h, 2)]))
    ref = obb.ffn_backward_samples(hid64, W1_64, b1_64, W2_64, dy64, r_s, f_s, h_s)
    # mask slack as in mask_slack(), over the sampled rows and columns
    amb_rows = np.abs(ref["a_rows"]) < 1e-4
    da_rows = np.abs(dy64[r_s] @ W2_64.T) * amb_rows
    amb_cols = np.abs(ref["a_cols"]) < 1e-4
    da_cols = np.abs(dy64 @ W2_64[f_s].T) * amb_cols
    slack = {"dhid": da_rows @ np.abs(W1_64).T, "dW1": np.abs(hid64).T @ da_cols, "db1": da_cols.sum(axis=0)}
    got = {"dhid": g["dhid"][r_s], "dW1": g["dW1"][:, f_s], "db1": g["db1"][f_s],
           "dW2": g["dW2"][f_s][:, h_s], "db2": g["db2"]}
    for k in ("dhid", "dW1", "db1", "dW2", "db2"):
        check(got[k], ref[k], f"{k} (rows 32768, h 4096, ffn 16384, sampled)", slack.get(k, 0.0))
