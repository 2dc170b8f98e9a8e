"""Pins of oracle/layer.py (CPU): the gate prologue, the L2 normalisation and the
second (NumPy) implementation of the recurrence.

* softplus against closed forms: softplus(0) = ln 2, softplus(x) - softplus(-x) = x,
  e^{-softplus(x)} = 1 / (1 + e^x), and the asymptotes at |x| = 40..700;
* L2 normalisation against a hand example (3, 4) -> (0.6, 0.8), unit norms,
  scale invariance, direction, zero rows;
* the NumPy recurrence against the C oracle (two independent implementations)
  to 1e-12, with and without an initial state;
* planted mistakes in copies of these functions fail the pins.
"""
import math

import numpy as np
import pytest
import torch

import kda_inputs as I
import oracle
from oracle import layer


def test_softplus_closed_forms():
    assert layer.softplus(0.0) == pytest.approx(math.log(2.0), abs=1e-16)
    x = np.linspace(-30, 30, 601)
    np.testing.assert_allclose(layer.softplus(x) - layer.softplus(-x), x, atol=1e-13)
    # alpha = e^{-softplus(x)} = 1 / (1 + e^x)
    np.testing.assert_allclose(np.exp(layer.gate_log_alpha(x)), 1.0 / (1.0 + np.exp(x)), rtol=1e-13)
    # asymptotes: softplus(x) = x + e^{-x} + O(e^{-2x}) for large x, e^{x} for very negative x
    for big in (40.0, 200.0, 700.0):
        assert layer.softplus(big) == pytest.approx(big + math.exp(-big), rel=1e-15)
        assert layer.softplus(-big) == pytest.approx(math.exp(-big), rel=1e-12)
    assert np.all(layer.gate_log_alpha(x) < 0)


def test_l2_normalize_pins():
    np.testing.assert_allclose(layer.l2_normalize(np.array([3.0, 4.0])), [0.6, 0.8], atol=1e-16)
    rng = np.random.default_rng(0)
    x = rng.standard_normal((5, 7, 128))
    y = layer.l2_normalize(x)
    np.testing.assert_allclose(np.linalg.norm(y, axis=-1), 1.0, atol=1e-14)
    np.testing.assert_allclose(layer.l2_normalize(37.5 * x), y, atol=1e-15)       # scale invariance
    np.testing.assert_allclose(np.sum(x * y, axis=-1), np.linalg.norm(x, axis=-1), rtol=1e-13)
    z = np.zeros((2, 4))
    assert np.all(layer.l2_normalize(z) == 0)


@pytest.mark.parametrize("with_state", [False, True])
def test_numpy_recurrence_matches_c_oracle(with_state):
    inp = I.prefill_inputs("fp32_small", B=2, T=37, H=3, dk=16, dv=12,
                           s0_std=0.3 if with_state else 0.0)
    ref_o, ref_s = oracle.forward(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"],
                                  inp["S0"])
    o, s = layer.recurrence(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"], inp["S0"])
    np.testing.assert_allclose(o, ref_o, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(s, ref_s, rtol=1e-12, atol=1e-13)


def test_numpy_recurrence_bf16_inputs_match_c_oracle():
    inp = I.prefill_inputs("prefill_4k", B=1, T=40, H=2, gate="strong")
    ref_o, ref_s = oracle.forward(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"])
    o, s = layer.recurrence(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"])
    np.testing.assert_allclose(o, ref_o, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(s, ref_s, rtol=1e-11, atol=1e-12)


def test_fused_forward_composes_the_prologue():
    """fused_forward(q, k, v, x, beta) is the recurrence on (q/|q|, k/|k|, v, -softplus(x), beta)."""
    g = torch.Generator().manual_seed(3)
    q, k = torch.randn(1, 20, 2, 16, generator=g) * 3, torch.randn(1, 20, 2, 16, generator=g) * 0.2
    v, x = torch.randn(1, 20, 2, 16, generator=g), torch.randn(1, 20, 2, 16, generator=g)
    beta = torch.sigmoid(torch.randn(1, 20, 2, generator=g))
    o, s = layer.fused_forward(q, k, v, x, beta)
    qn = (q.double() / q.double().norm(dim=-1, keepdim=True)).numpy()
    kn = (k.double() / k.double().norm(dim=-1, keepdim=True)).numpy()
    la = -np.log1p(np.exp(x.double().numpy()))
    o2, s2 = layer.recurrence(qn, kn, v, la, beta)
    np.testing.assert_allclose(o, o2, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(s, s2, rtol=1e-12, atol=1e-13)


MUTANTS = {
    "softplus_sign": ("softplus", lambda x: np.maximum(x, 0.0) - np.log1p(np.exp(-np.abs(x)))),
    "softplus_no_max": ("softplus", lambda x: np.log1p(np.exp(-np.abs(np.asarray(x, float))))),
    "norm_squared": ("l2_normalize", lambda x: np.asarray(x) / np.sum(np.asarray(x) ** 2, -1, keepdims=True)),
    "norm_wrong_axis": ("l2_normalize", lambda x: np.asarray(x) / np.linalg.norm(np.asarray(x), axis=0, keepdims=True)),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_planted_mistakes(name, monkeypatch):
    fn, bad = MUTANTS[name]
    monkeypatch.setattr(layer, fn, bad)
    caught = False
    for pin in (test_softplus_closed_forms, test_l2_normalize_pins):
        try:
            pin()
        except AssertionError:
            caught = True
    assert caught, f"no pin caught mutant {name}"
