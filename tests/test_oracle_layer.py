"""Pins of oracle/layer.py (CPU): the gate prologue, the L2 normalisation and the
second (NumPy) implementation of the recurrence.

* softplus against closed forms: softplus(0) = ln 2, softplus(x) - softplus(-x) = x,
  e^{-softplus(x)} = 1 / (1 + e^x), and the asymptotes at |x| = 40..700;
* L2 normalisation against a hand example (3, 4) -> (0.6, 0.8), unit norms,
  scale invariance, direction, zero rows;
* the NumPy recurrence against the C oracle (two independent implementations)
  to 1e-12, with and without an initial state;
* sigmoid and Swish against closed forms (sigma(0) = 1/2, sigma(ln 3) = 3/4,
  sigma(x) + sigma(-x) = 1, swish(x) - swish(-x) = x);
* ShortConv against numpy.convolve per channel (an independent library
  routine), a delta filter (identity), a shifted delta (delay by one token), a
  constant input (prefix sums of the taps) and packed sequences (no leakage
  across a boundary);
* the RMSNorm + output gate against a hand example, unit RMS, scale invariance
  and the gate's limits;
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


def test_sigmoid_swish_closed_forms():
    assert layer.sigmoid(0.0) == 0.5
    assert layer.sigmoid(math.log(3.0)) == pytest.approx(0.75, abs=1e-15)
    x = np.linspace(-40, 40, 801)
    np.testing.assert_allclose(layer.sigmoid(x) + layer.sigmoid(-x), 1.0, atol=1e-15)
    np.testing.assert_allclose(layer.swish(x) - layer.swish(-x), x, atol=1e-12)
    assert layer.swish(0.0) == 0.0
    assert layer.swish(math.log(3.0)) == pytest.approx(0.75 * math.log(3.0), rel=1e-15)
    assert layer.sigmoid(-800.0) == 0.0 and layer.sigmoid(800.0) == 1.0


def test_short_conv_pins():
    rng = np.random.default_rng(1)
    B, T, H, d, W = 2, 11, 3, 5, 4
    x = rng.standard_normal((B, T, H, d))
    w = rng.standard_normal((H, d, W))
    y = layer.short_conv(x, w)
    for b in range(B):
        for h in range(H):
            for c in range(d):   # causal convolution = the first T terms of the full one
                np.testing.assert_allclose(y[b, :, h, c], np.convolve(x[b, :, h, c], w[h, c])[:T], atol=1e-13)
    delta = np.zeros((H, d, W)); delta[..., 0] = 1.0
    np.testing.assert_array_equal(layer.short_conv(x, delta), x)
    shift = np.zeros((H, d, W)); shift[..., 1] = 1.0
    ys = layer.short_conv(x, shift)
    np.testing.assert_array_equal(ys[:, 1:], x[:, :-1])
    assert np.all(ys[:, 0] == 0)
    ones = np.ones((1, T, H, d))
    np.testing.assert_allclose(layer.short_conv(ones, w)[0, :, 0, 0],
                               [w[0, 0, : min(t + 1, W)].sum() for t in range(T)], atol=1e-14)
    # packed sequences: each piece is convolved on its own
    cu = np.array([0, 3, 3, 11])
    flat = x[0]
    yp = layer.short_conv(flat, w, cu)
    np.testing.assert_allclose(yp[:3], layer.short_conv(flat[None, :3], w)[0], atol=1e-15)
    np.testing.assert_allclose(yp[3:], layer.short_conv(flat[None, 3:], w)[0], atol=1e-15)
    np.testing.assert_allclose(layer.short_conv_swish(x, w), layer.swish(y), atol=0)


def test_rms_norm_gate_pins():
    # hand example: o = (3, 4), mean(o^2) = 12.5, sigmoid(0) = 1/2
    y = layer.rms_norm_gate(np.array([3.0, 4.0]), np.zeros(2), np.ones(2), eps=0.0)
    np.testing.assert_allclose(y, [0.5 * 3 / math.sqrt(12.5), 0.5 * 4 / math.sqrt(12.5)], rtol=1e-15)
    rng = np.random.default_rng(2)
    o = rng.standard_normal((4, 7, 16))
    big = np.full_like(o, 60.0)   # sigmoid -> 1
    y = layer.rms_norm_gate(o, big, np.ones(16), eps=0.0)
    np.testing.assert_allclose(np.mean(y * y, axis=-1), 1.0, atol=1e-12)
    np.testing.assert_allclose(layer.rms_norm_gate(7.5 * o, big, np.ones(16), eps=0.0), y, atol=1e-13)
    gw = rng.standard_normal(16)
    np.testing.assert_allclose(layer.rms_norm_gate(o, big, gw, eps=0.0), y * gw, atol=1e-13)
    assert np.all(layer.rms_norm_gate(o, -big * 20, gw) == 0.0)
    # eps inside the root: o = 0 stays 0, a tiny o is damped
    assert np.all(layer.rms_norm_gate(np.zeros(16), big[0, 0], gw) == 0.0)
    small = layer.rms_norm_gate(np.full(16, 1e-4), big[0, 0], np.ones(16), eps=1e-6)
    np.testing.assert_allclose(small, 1e-4 / math.sqrt(1e-8 + 1e-6), rtol=1e-12)


MUTANTS = {
    "softplus_sign": ("softplus", lambda x: np.maximum(x, 0.0) - np.log1p(np.exp(-np.abs(x)))),
    "softplus_no_max": ("softplus", lambda x: np.log1p(np.exp(-np.abs(np.asarray(x, float))))),
    "norm_squared": ("l2_normalize", lambda x: np.asarray(x) / np.sum(np.asarray(x) ** 2, -1, keepdims=True)),
    "norm_wrong_axis": ("l2_normalize", lambda x: np.asarray(x) / np.linalg.norm(np.asarray(x), axis=0, keepdims=True)),
    "sigmoid_sign": ("sigmoid", lambda x: 1.0 / (1.0 + np.exp(np.asarray(x, float)))),
    "swish_sign": ("swish", lambda x: np.asarray(x, float) / (1.0 + np.exp(np.asarray(x, float)))),
    "conv_anticausal": ("short_conv", lambda x, w, cu=None: _conv_shifted(x, w, -1)),
    "conv_off_by_one": ("short_conv", lambda x, w, cu=None: _conv_shifted(x, w, 1)),
    "rms_sum_not_mean": ("rms_norm_gate", lambda o, z, g, eps=1e-6: np.asarray(o) / np.sqrt(np.sum(np.asarray(o) ** 2, -1, keepdims=True) + eps) * g * layer.sigmoid(z)),
    "rms_eps_outside": ("rms_norm_gate", lambda o, z, g, eps=1e-6: np.asarray(o) / (np.sqrt(np.mean(np.asarray(o) ** 2, -1, keepdims=True)) + eps) * g * layer.sigmoid(z)),
    "rms_no_gate": ("rms_norm_gate", lambda o, z, g, eps=1e-6: np.asarray(o) / np.sqrt(np.mean(np.asarray(o) ** 2, -1, keepdims=True) + eps) * g),
}


def _conv_shifted(x, w, shift):
    """A wrong convolution: taps applied with an extra shift (shift -1: looks ahead)."""
    x, w = np.asarray(x, float), np.asarray(w, float)
    T, W = x.shape[1], w.shape[-1]
    y = np.zeros_like(x)
    for j in range(W):
        s = j + shift
        if 0 <= s < T:
            y[:, s:] += w[None, None, :, :, j] * x[:, : T - s]
        elif s < 0 and -s < T:
            y[:, : T + s] += w[None, None, :, :, j] * x[:, -s:]
    return y


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_planted_mistakes(name, monkeypatch):
    fn, bad = MUTANTS[name]
    monkeypatch.setattr(layer, fn, bad)
    caught = False
    for pin in (test_softplus_closed_forms, test_l2_normalize_pins, test_sigmoid_swish_closed_forms,
                test_short_conv_pins, test_rms_norm_gate_pins):
        try:
            pin()
        except AssertionError:
            caught = True
    assert caught, f"no pin caught mutant {name}"
