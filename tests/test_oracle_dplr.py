"""Pins of oracle/dplr.py, the fp64 general-DPLR recurrence (CPU).

* KDA is the case a = -beta k, b = alpha * k with write vector beta k: the DPLR
  oracle then equals the C KDA oracle (itself pinned in test_oracle.py) to 1e-12;
* a = 0 is gated linear attention: the output equals the closed form
  o_t = sum_{j<=t} (sum_c q_tc e^{g_tc - g_jc} k_jc) v_j + (q_t e^{g_t})^T S0,
  written out with loops on a tiny case;
* brute force: the product of the explicit d_k x d_k transition matrices
  Diag(alpha_t) + a_t b_t^T on T <= 6;
* linearity in (v, S0);
* planted mistakes in a copy of the recurrence fail one of these.
"""
import math

import numpy as np
import pytest
import torch

import kda_inputs as I
import oracle
from oracle import dplr


def small(seed=0, B=1, T=5, H=2, dk=3, dv=2):
    rng = np.random.default_rng(seed)
    q, k, a, b = (rng.standard_normal((B, T, H, dk)) for _ in range(4))
    v = rng.standard_normal((B, T, H, dv))
    la = -np.log1p(np.exp(rng.standard_normal((B, T, H, dk))))
    S0 = rng.standard_normal((B, H, dk, dv))
    return q, k, v, 0.4 * a, 0.4 * b, la, S0


def test_kda_is_a_special_case():
    inp = I.prefill_inputs("fp32_small", B=2, T=23, H=2, dk=8, dv=6, s0_std=0.3)
    a, b, wk = dplr.kda_as_dplr(inp["k"], inp["log_alpha"], inp["beta"])
    o, s = dplr.forward(inp["q"], wk, inp["v"], a, b, inp["log_alpha"], inp["S0"])
    ro, rs = oracle.forward(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"], inp["S0"])
    np.testing.assert_allclose(o, ro, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(s, rs, rtol=1e-12, atol=1e-12)


def test_gla_closed_form():
    q, k, v, a, b, la, S0 = small(1)
    o, _ = dplr.forward(q, k, v, np.zeros_like(a), b, la, S0)
    B, T, H, dk = q.shape
    g = np.cumsum(la, axis=1)
    ref = np.zeros_like(o)
    for bb in range(B):
        for h in range(H):
            for t in range(T):
                acc = np.zeros(v.shape[-1])
                for j in range(t + 1):
                    w = sum(q[bb, t, h, c] * math.exp(g[bb, t, h, c] - g[bb, j, h, c]) * k[bb, j, h, c]
                            for c in range(dk))
                    acc += w * v[bb, j, h]
                for c in range(dk):
                    acc += q[bb, t, h, c] * math.exp(g[bb, t, h, c]) * S0[bb, h, c]
                ref[bb, t, h] = acc
    np.testing.assert_allclose(o, ref, rtol=1e-12, atol=1e-12)


def test_brute_force_transition_products():
    q, k, v, a, b, la, S0 = small(2, T=6)
    o, s = dplr.forward(q, k, v, a, b, la, S0)
    B, T, H, dk = q.shape
    for bb in range(B):
        for h in range(H):
            S = S0[bb, h].copy()
            for t in range(T):
                M = np.diag(np.exp(la[bb, t, h])) + np.outer(a[bb, t, h], b[bb, t, h])
                S = M @ S + np.outer(k[bb, t, h], v[bb, t, h])
                np.testing.assert_allclose(o[bb, t, h], S.T @ q[bb, t, h], rtol=1e-12, atol=1e-12)
            np.testing.assert_allclose(s[bb, h], S, rtol=1e-12, atol=1e-12)


def test_linearity():
    q, k, v, a, b, la, S0 = small(3)
    _, _, v2, _, _, _, S02 = small(4)
    o1, s1 = dplr.forward(q, k, v, a, b, la, S0)
    o2, s2 = dplr.forward(q, k, v2, a, b, la, S02)
    o3, s3 = dplr.forward(q, k, v + 2.0 * v2, a, b, la, S0 + 2.0 * S02)
    np.testing.assert_allclose(o3, o1 + 2.0 * o2, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(s3, s1 + 2.0 * s2, rtol=1e-11, atol=1e-12)


def test_inputs_stay_bounded():
    """The synthetic a, b keep the state bounded over a long sequence."""
    inp = I.dplr_inputs("prefill_4k", B=1, T=600, H=1, dk=16, dv=4)
    o, s = dplr.forward(inp["q"], inp["k"], inp["v"], inp["a"], inp["b"], inp["log_alpha"])
    assert np.isfinite(o).all() and np.abs(s).max() < 50


def _wrong(kind):
    def fwd(q, k, v, a, b, log_alpha, S0=None):
        q, k, v, a, b, la = (dplr._np64(t) for t in (q, k, v, a, b, log_alpha))
        B, T, H, dk = q.shape
        S = np.zeros((B, H, dk, v.shape[-1])) if S0 is None else dplr._np64(S0).copy()
        out = np.zeros((B, T, H, v.shape[-1]))
        for t in range(T):
            Sd = np.exp(la[:, t])[..., None] * S
            probe = np.einsum("bhi,bhij->bhj", b[:, t], Sd if kind == "probe_after_decay" else S)
            sign = -1.0 if kind == "sign" else 1.0
            S = Sd + sign * a[:, t][..., None] * probe[..., None, :]
            if kind != "no_write":
                S = S + k[:, t][..., None] * v[:, t][..., None, :]
            out[:, t] = np.einsum("bhi,bhij->bhj", q[:, t], S if kind != "output_before_write" else Sd)
        return out, S
    return fwd


@pytest.mark.parametrize("kind", ["probe_after_decay", "sign", "no_write", "output_before_write"])
def test_pins_catch_planted_mistakes(kind, monkeypatch):
    monkeypatch.setattr(dplr, "forward", _wrong(kind))
    caught = False
    for pin in (test_kda_is_a_special_case, test_gla_closed_form, test_brute_force_transition_products):
        try:
            pin()
        except AssertionError:
            caught = True
    assert caught, f"no pin caught {kind}"
