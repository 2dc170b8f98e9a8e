"""Pins of the fp64 backward oracle (``oracle/grad.py``), all on CPU.

The backward pass is the derivative of the recurrence, so it is pinned by
what fixes a derivative independently of how it was derived: central finite
differences of the forward (per element on a tiny problem, along random
directions on a larger one), the textbook gradients of unnormalised linear
attention (the special case alpha = 1, erase 0, write 1), and torch autograd
through a separately written recurrence. ``forward64`` itself is pinned to the
C oracle, whose own pins are in test_oracle.py.
"""
import numpy as np
import pytest
import torch

import oracle
from oracle import grad

NAMES = ["q", "k", "v", "log_alpha", "beta", "S0"]


def problem(B=1, T=6, H=2, dk=4, dv=3, seed=0, s0=True):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((B, T, H, dk))
    k = rng.standard_normal((B, T, H, dk))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((B, T, H, dv))
    la = -np.log1p(np.exp(rng.standard_normal((B, T, H, dk))))
    beta = 1.0 / (1.0 + np.exp(-rng.standard_normal((B, T, H))))
    S0 = 0.3 * rng.standard_normal((B, H, dk, dv)) if s0 else None
    dout = rng.standard_normal((B, T, H, dv))
    dST = rng.standard_normal((B, H, dk, dv))
    return dict(q=q, k=k, v=v, log_alpha=la, beta=beta, S0=S0), dout, dST


def loss(x, dout, dST, **kw):
    out, ST = grad.forward64(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], x["S0"], **kw)
    return float(np.sum(out * dout) + np.sum(ST * dST))


def grads(x, dout, dST, **kw):
    g = grad.backward(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], dout, S0=x["S0"],
                      dS_T=dST, **kw)
    g = {n[1:]: a for n, a in g.items()}
    return g


def test_forward64_matches_the_c_oracle():
    x, _, _ = problem(B=2, T=37, H=3, dk=8, dv=5, seed=3)
    f32 = {n: (a.astype(np.float32) if a is not None else None) for n, a in x.items()}
    out, ST = grad.forward64(**f32)
    t = {n: (torch.from_numpy(a) if a is not None else None) for n, a in f32.items()}
    ref_out, ref_ST = oracle.forward(t["q"], t["k"], t["v"], t["log_alpha"], t["beta"], t["S0"])
    np.testing.assert_allclose(out, ref_out, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(ST, ref_ST, rtol=1e-11, atol=1e-12)


def test_every_element_against_central_differences():
    x, dout, dST = problem(B=1, T=4, H=1, dk=3, dv=2, seed=1)
    g = grads(x, dout, dST)
    h = 1e-6
    for n in NAMES:
        a = x[n]
        num = np.zeros_like(a)
        for idx in np.ndindex(a.shape):
            saved = a[idx]
            a[idx] = saved + h
            lp = loss(x, dout, dST)
            a[idx] = saved - h
            lm = loss(x, dout, dST)
            a[idx] = saved
            num[idx] = (lp - lm) / (2 * h)
        np.testing.assert_allclose(g[n], num, rtol=1e-6, atol=1e-8, err_msg=n)


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_random_directions_against_central_differences(seed):
    x, dout, dST = problem(B=2, T=19, H=2, dk=6, dv=5, seed=seed)
    g = grads(x, dout, dST)
    rng = np.random.default_rng(100 + seed)
    for _ in range(3):
        d = {n: rng.standard_normal(x[n].shape) for n in NAMES}
        analytic = sum(float(np.sum(g[n] * d[n])) for n in NAMES)
        h = 1e-6
        xp = {n: x[n] + h * d[n] for n in NAMES}
        xm = {n: x[n] - h * d[n] for n in NAMES}
        numeric = (loss(xp, dout, dST) - loss(xm, dout, dST)) / (2 * h)
        assert abs(analytic - numeric) <= 1e-6 * max(1.0, abs(numeric))


def test_linear_attention_closed_form():
    """alpha = 1, erase 0, write 1: S_t = S0 + sum_{s<=t} k_s v_s^T and o_t = S_t^T q_t,
    whose gradients are the textbook ones (cumulative sums, no recurrence)."""
    x, dout, dST = problem(B=1, T=9, H=1, dk=4, dv=3, seed=5)
    T = 9
    x["log_alpha"] = np.zeros_like(x["log_alpha"])
    erase = np.zeros_like(x["beta"])
    write = np.ones_like(x["beta"])
    g = grad.backward(x["q"], x["k"], x["v"], x["log_alpha"], erase, dout, S0=x["S0"], dS_T=dST,
                      beta_write=write)
    q, k, v, S0 = x["q"][0, :, 0], x["k"][0, :, 0], x["v"][0, :, 0], x["S0"][0, 0]
    dO, dS = dout[0, :, 0], dST[0, 0]
    kv = np.einsum("ti,tj->tij", k, v)
    S = S0 + np.cumsum(kv, axis=0)                          # S_t, t = 1..T
    S_prev = np.concatenate([S0[None], S[:-1]])             # S_{t-1}
    qdo = np.einsum("ti,tj->tij", q, dO)
    G = dS + np.cumsum(qdo[::-1], axis=0)[::-1]             # dL/dS_t = dS_T + sum_{s>=t} q_s dO_s^T
    np.testing.assert_allclose(g["dq"][0, :, 0], np.einsum("tij,tj->ti", S, dO), rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(g["dv"][0, :, 0], np.einsum("tij,ti->tj", G, k), rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(g["dk"][0, :, 0], np.einsum("tij,tj->ti", G, v), rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(g["dS0"][0, 0], G[0], rtol=1e-12, atol=1e-12)
    gk = np.einsum("tij,ti->tj", G, k)
    np.testing.assert_allclose(g["dbeta_write"][0, :, 0], np.sum(v * gk, axis=1), rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(g["dbeta"][0, :, 0], -np.einsum("tij,ti,tj->t", S_prev, k, gk),
                               rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(g["dlog_alpha"][0, :, 0], np.sum(G * S_prev, axis=2), rtol=1e-12, atol=1e-12)
    assert T == g["dq"].shape[1]


def test_autograd_of_an_independent_torch_recurrence():
    x, dout, dST = problem(B=1, T=12, H=2, dk=5, dv=4, seed=7)
    tx = {n: torch.tensor(x[n], dtype=torch.float64, requires_grad=True) for n in NAMES}
    B, T, H = 1, 12, 2
    total = torch.zeros((), dtype=torch.float64)
    for h in range(H):
        S = tx["S0"][0, h]
        for t in range(T):
            kt = tx["k"][0, t, h]
            a = torch.exp(tx["log_alpha"][0, t, h])
            b = tx["beta"][0, t, h]
            M = torch.eye(5, dtype=torch.float64) - b * torch.outer(kt, kt)
            S = M @ (a[:, None] * S) + b * torch.outer(kt, tx["v"][0, t, h])
            total = total + (S.T @ tx["q"][0, t, h]) @ torch.from_numpy(dout[0, t, h])
        total = total + torch.sum(S * torch.from_numpy(dST[0, h]))
    total.backward()
    g = grads(x, dout, dST)
    for n in NAMES:
        np.testing.assert_allclose(g[n], tx[n].grad.numpy(), rtol=1e-10, atol=1e-12, err_msg=n)


def test_zero_cotangents_give_zero_gradients():
    x, dout, dST = problem(seed=9)
    g = grads(x, np.zeros_like(dout), np.zeros_like(dST))
    for n in NAMES:
        assert np.all(g[n] == 0.0), n


MUTANTS = [
    ("dbe[b, t, h] = -(r @ g)", "dbe[b, t, h] = (r @ g)"),                        # sign of the erase term
    ("G = alpha[:, None] * dSp", "G = dSp"),                                        # decay dropped going back
    ("dk_[b, t, h] = G @ w - be[b, t, h] * (Sp @ g)", "dk_[b, t, h] = G @ w"),      # erase path of dk dropped
    ("dSp = G - be[b, t, h] * np.outer(kt, g)", "dSp = G"),                        # erase path of dS' dropped
    ("G = G + np.outer(qt, do)", "G = G + np.outer(qt, do) * 0.5"),                 # output cotangent halved
    ("dq[b, t, h] = S_t @ do", "dq[b, t, h] = S_prev @ do"),                        # off-by-one state
    ("dla[b, t, h] = alpha * np.sum(dSp * S_prev, axis=1)",
     "dla[b, t, h] = np.sum(dSp * S_prev, axis=1)"),                                 # d alpha vs d log alpha
]


@pytest.mark.parametrize("old,new", MUTANTS)
def test_planted_mistakes_fail_the_difference_pin(old, new):
    import inspect
    import types
    src = inspect.getsource(grad)
    assert src.count(old) == 1, old
    mod = types.ModuleType("grad_mutant")
    exec(compile(src.replace(old, new), "grad_mutant", "exec"), mod.__dict__)
    x, dout, dST = problem(B=1, T=7, H=1, dk=4, dv=3, seed=11)
    g = mod.backward(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], dout, S0=x["S0"], dS_T=dST)
    g = {n[1:]: a for n, a in g.items()}
    rng = np.random.default_rng(5)
    d = {n: rng.standard_normal(x[n].shape) for n in NAMES}
    analytic = sum(float(np.sum(g[n] * d[n])) for n in NAMES)
    h = 1e-6
    numeric = (loss({n: x[n] + h * d[n] for n in NAMES}, dout, dST)
               - loss({n: x[n] - h * d[n] for n in NAMES}, dout, dST)) / (2 * h)
    assert abs(analytic - numeric) > 1e-4 * max(1.0, abs(numeric))
