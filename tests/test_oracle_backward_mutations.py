"""Plant plausible mistakes in the backward oracle (on the CPU) and check that
the pins of test_oracle_backward_pins.py catch each: the softmax Jacobian, the
ReLU gradient, the value, query and key gradients, the attention scale and
both paths into hid."""

import numpy as np
import pytest

from oracle import bpt_oracle_backward as obb
from tests import test_oracle_backward_pins as pins


def _qk_swapped(dS, Q, K, scale):
    return (np.swapaxes(dS, -1, -2) @ Q) * scale, (dS @ K) * scale


def _dq_unscaled(dS, Q, K, scale):
    return dS @ K, (np.swapaxes(dS, -1, -2) @ Q) * scale


MUTATIONS = {
    "softmax_jacobian_term_dropped": ("_softmax_grad", lambda P, dP: P * dP),
    "softmax_jacobian_sign": ("_softmax_grad", lambda P, dP: P * (dP + np.sum(dP * P, axis=-1, keepdims=True))),
    "relu_grad_ignored": ("_relu_grad", lambda a: np.ones_like(a)),
    "relu_grad_wrong_side": ("_relu_grad", lambda a: (a < 0).astype(a.dtype)),
    "value_grad_untransposed": ("_value_grad", lambda P, dO: P @ dO),
    "query_key_grads_swapped": ("_qk_grads", _qk_swapped),
    "query_grad_unscaled": ("_qk_grads", _dq_unscaled),
    "second_residual_grad_missing": ("_dhid", lambda dy, da, W1: da @ W1.T),
    "ffn_grad_into_hid_missing": ("_dhid", lambda dy, da, W1: dy),
}

PINS = [
    lambda: pins.test_gradients_match_central_differences(1, 3, 4, 2, 8, 3, False),
    lambda: pins.test_gradients_match_central_differences(1, 3, 4, 2, 8, 3, True),
    lambda: pins.test_gradients_match_torch_autograd(2, 7, 16, 4, 24, True),
]


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_planted_mistake_is_caught(name, monkeypatch):
    attr, fn = MUTATIONS[name]
    monkeypatch.setattr(obb, attr, fn)
    caught = []
    for i, pin in enumerate(PINS):
        try:
            with np.errstate(all="ignore"):
                pin()
        except (AssertionError, ValueError, IndexError):
            caught.append(i)
    assert caught, f"no pin caught the planted mistake {name!r}"


def test_unmutated_oracle_passes_every_pin():
    for pin in PINS:
        pin()
