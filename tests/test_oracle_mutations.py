"""Plant plausible mistakes in the oracle (on the CPU) and check that the pins catch each.

Every mutation replaces one named step of the oracle with a wrong version for
the duration of one test; at least one pin of test_oracle_pins.py must then
fail. This shows that the pins constrain every step: scale, mask, activation,
head split, projection layout and both residuals.
"""

import math

import numpy as np
import pytest

import oracle
from oracle import bpt_oracle as ob
from tests import test_oracle_pins as pins

_orig_qkv = ob.qkv_projection
_orig_ffn = ob.residual_ffn


def _qkv_kv_swapped(x, Wqkv, bqkv):
    q, k, v = _orig_qkv(x, Wqkv, bqkv)
    return q, v, k


def _ffn_without_first_residual(x, O, Wo, bo, W1, b1, W2, b2):
    hid = O @ Wo + bo
    return hid + (np.maximum(hid @ W1 + b1, 0) @ W2 + b2)


def _ffn_without_second_residual(x, O, Wo, bo, W1, b1, W2, b2):
    hid = x + (O @ Wo + bo)
    return np.maximum(hid @ W1 + b1, 0) @ W2 + b2


def _ffn_without_bias2(x, O, Wo, bo, W1, b1, W2, b2):
    hid = x + (O @ Wo + bo)
    return hid + np.maximum(hid @ W1 + b1, 0) @ W2


MUTATIONS = {
    "scale_dropped": [("_softmax_scale", lambda dh: 1.0)],
    "scale_1_over_d": [("_softmax_scale", lambda dh: 1.0 / dh)],
    "causal_strict": [("_key_allowed", lambda t, u, c: (u[None, :] < t[:, None]) if c else np.ones((t.size, u.size), bool))],
    "causal_one_late": [("_key_allowed", lambda t, u, c: (u[None, :] <= t[:, None] + 1) if c else np.ones((t.size, u.size), bool))],
    "causal_reversed": [("_key_allowed", lambda t, u, c: (u[None, :] >= t[:, None]) if c else np.ones((t.size, u.size), bool))],
    "relu_missing": [("_relu", lambda z: z)],
    "relu_wrong_side": [("_relu", lambda z: np.minimum(z, 0.0))],
    "heads_merged": [("_head_cols", lambda k, dh: slice(0, None))],
    "kv_swapped": [("qkv_projection", _qkv_kv_swapped)],
    "first_residual_missing": [("residual_ffn", _ffn_without_first_residual)],
    "second_residual_missing": [("residual_ffn", _ffn_without_second_residual)],
    "ffn_bias2_missing": [("residual_ffn", _ffn_without_bias2)],
}

PINS = [
    lambda: pins.test_layer_equals_brute_force(1, 3, 4, 2, True),
    lambda: pins.test_layer_equals_brute_force(2, 5, 4, 2, False),
    lambda: pins.test_zero_queries_give_uniform_attention(True),
    lambda: pins.test_first_causal_row_attends_only_to_itself(),
    lambda: pins.test_zero_values_isolate_the_ffn(),
    lambda: pins.test_attention_matches_torch_multihead_attention(2, 9, 16, 4, True),
    lambda: pins.test_ffn_matches_torch_linear_relu_linear(),
]


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_planted_mistake_is_caught(name, monkeypatch):
    for attr, fn in MUTATIONS[name]:
        monkeypatch.setattr(ob, attr, fn)
        if hasattr(oracle, attr):
            monkeypatch.setattr(oracle, attr, fn)
    caught = []
    for i, pin in enumerate(PINS):
        try:
            with np.errstate(all="ignore"):
                pin()
        except (AssertionError, ValueError, IndexError, FloatingPointError):
            caught.append(i)
    assert caught, f"no pin caught the planted mistake {name!r}"


def test_pins_pass_without_mutation():
    for pin in PINS:
        pin()
    assert math.isfinite(1.0)
