"""The seeded input generator: counter-based draws, distributions, rounding."""

import math

import numpy as np
import pytest
import torch

import bpt_inputs as bi


def test_splitmix64_known_first_outputs():
    # splitmix64 seeded with state 0 has a published first output,
    # 0xE220A8397B1DCDAF (the reference C implementation by Vigna).
    assert bi.mix64_int(0 + bi.GAMMA) == 0xE220A8397B1DCDAF
    assert bi.mix64_int(2 * bi.GAMMA) == 0x6E789E6AA1B965F4


@pytest.mark.parametrize("tensor_id", [0, 1, 8])
def test_vector_draws_match_scalar_definition(tensor_id):
    n = 5000
    v = bi.normal_f64(7, tensor_id, n)
    for j in [0, 1, 2, 17, 999, 4999]:
        assert v[j] == bi.normal_scalar(7, tensor_id, j)


def test_chunked_threaded_draws_are_position_stable():
    n = (1 << 22) + 12345  # spans two chunks
    v = bi.normal_f64(3, 2, n, threads=4)
    w = bi.normal_f64(3, 2, 100)
    assert np.array_equal(v[:100], w)
    for j in [(1 << 22) - 1, 1 << 22, n - 1]:
        assert v[j] == bi.normal_scalar(3, 2, j)


def test_moments_are_standard_normal():
    v = bi.normal_f64(0, 5, 1 << 20)
    assert abs(v.mean()) < 5e-3
    assert abs(v.std() - 1.0) < 5e-3
    # fraction within one sigma of a standard normal
    assert abs(np.mean(np.abs(v) < 1.0) - math.erf(1 / math.sqrt(2))) < 3e-3


def test_streams_differ_by_tensor_and_seed():
    a = bi.normal_f64(0, 0, 64)
    assert not np.array_equal(a, bi.normal_f64(0, 1, 64))
    assert not np.array_equal(a, bi.normal_f64(1, 0, 64))


def test_bf16_rounding_matches_torch_round_to_nearest_even():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.standard_normal(100000).astype(np.float32),
                        np.array([1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -1.0 - 2 ** -8, 0.0, -0.0], np.float32)])
    mine = bi.f32_to_bf16_bits(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(mine, ref)
    back = bi.bf16_bits_to_f64(mine)
    assert np.array_equal(back, torch.from_numpy(x).to(torch.bfloat16).double().numpy())


def test_make_inputs_shapes_and_scales():
    shp = bi.LayerShape(1, 64, 128, 2, 64, 64, True)
    inp = bi.make_inputs(shp, seed=0)
    assert inp["x"].shape == (1, 64, 128) and inp["x"].dtype == np.uint16
    assert inp["Wqkv"].shape == (128, 384)
    assert inp["W2"].shape == (512, 128)
    w1 = bi.to_f64(inp["W1"])
    assert abs(w1.std() - 1 / math.sqrt(128)) < 0.01 / math.sqrt(128) * 10
    w2 = bi.to_f64(inp["W2"])
    assert abs(w2.std() - 1 / math.sqrt(512)) < 0.1 / math.sqrt(512)
    assert abs(bi.to_f64(inp["b1"]).std() - 0.02) < 0.004
    f32 = bi.make_inputs(bi.LayerShape(1, 8, 64, 1, 8, 8, False, "f32"))
    assert f32["x"].dtype == np.float32


def test_ffn_width_sets_the_ffn_shapes_and_keeps_the_streams():
    base = bi.LayerShape(1, 8, 64, 1, 8, 8, True)
    wide = bi.LayerShape(1, 8, 64, 1, 8, 8, True, ffn=192)
    assert base.f == 256 and wide.f == 192
    shp = bi.tensor_shapes(wide)
    assert shp["W1"] == (64, 192) and shp["b1"] == (192,) and shp["W2"] == (192, 64)
    assert bi.tensor_std("W2", wide) == 1.0 / math.sqrt(192)
    assert bi.tensor_std("W1", wide) == 1.0 / math.sqrt(64)
    a, b = bi.make_inputs(base, seed=3), bi.make_inputs(wide, seed=3)
    # same counter streams: tensors of equal shape are identical, W1 is a prefix
    for k in ("x", "Wqkv", "bqkv", "Wo", "bo", "b2"):
        assert np.array_equal(a[k], b[k])
    assert np.array_equal(a["W1"].reshape(-1)[: 64 * 192], b["W1"].reshape(-1))
