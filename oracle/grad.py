"""fp64 reverse-mode derivative of the KDA recurrence -- test infrastructure only.

The pages define the forward recurrence (Kimi Linear summary,
es.news.hada.io/topic?id=31936, sections "De la atencion lineal a Gated
DeltaNet" and "Control fino de memoria en Kimi Delta Attention") and say the
chunked algorithm is built for training throughput (section "Algoritmo paralelo
por chunks"); they print no backward pass. This module is the plain definition
of one: the derivative of a scalar loss through the token-by-token recurrence,
taken step by step in reverse order, in fp64 numpy, one (batch, head) at a
time. Like the rest of ``oracle/``, only tests may call it.

Per token t (alpha_t = exp(log_alpha_t); erase strength b_t and write strength
c_t, both beta_t in KDA):

    S'_t = Diag(alpha_t) S_{t-1}
    w_t  = c_t v_t - b_t S'_t^T k_t
    S_t  = S'_t + k_t w_t^T                   (= (I - b_t k_t k_t^T) S'_t + c_t k_t v_t^T)
    o_t  = S_t^T q_t

Given dO = dL/do and dS_T = dL/dS_T, with G = dL/dS_t accumulated backwards
and g_t = G^T k_t:

    G      += q_t dO_t^T
    dq_t    = S_t dO_t
    dv_t    = c_t g_t
    dc_t    = v_t . g_t
    db_t    = -(S'_t^T k_t) . g_t
    dk_t    = G w_t - b_t S'_t g_t
    dS'_t   = G - b_t k_t g_t^T
    dlog_alpha_t = alpha_t * rowsum(dS'_t * S_{t-1})
    G       = Diag(alpha_t) dS'_t               (dL/dS_{t-1})

and dS0 is the final G. For KDA (b = c = beta) dbeta = db + dc.

Parity pins (tests/test_oracle_grad.py): central finite differences of
``forward64`` along random directions and per element on tiny problems, the
closed form of unnormalised linear attention (alpha = 1, erase strength 0,
write strength 1), autograd of an independent torch recurrence, and
``forward64`` against the C oracle's forward.
"""
from __future__ import annotations

import numpy as np
import torch


def _np64(x):
    if x is None:
        return None
    if isinstance(x, torch.Tensor):
        return x.detach().cpu().to(torch.float64).numpy()
    return np.asarray(x, dtype=np.float64)


def forward64(q, k, v, log_alpha, beta, S0=None, beta_write=None, keep_states=False):
    """The recurrence in fp64 with fp64 inputs (the C oracle takes fp32/bf16
    inputs; finite differences need inputs that can move by 1e-7).

    Shapes as the C oracle: q, k, log_alpha ``[B,T,H,dk]``, v ``[B,T,H,dv]``,
    beta ``[B,T,H]`` (erase strength), beta_write ``[B,T,H]`` (default: beta),
    S0 ``[B,H,dk,dv]`` or None. Returns ``(out, S_T)``, plus the states
    ``[B,H,T+1,dk,dv]`` (S_0 .. S_T) when ``keep_states``.
    """
    q, k, v, la, be = (_np64(x) for x in (q, k, v, log_alpha, beta))
    bw = be if beta_write is None else _np64(beta_write)
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    s0 = np.zeros((B, H, dk, dv)) if S0 is None else _np64(S0)
    out = np.zeros((B, T, H, dv))
    ST = np.zeros((B, H, dk, dv))
    states = np.zeros((B, H, T + 1, dk, dv)) if keep_states else None
    for b in range(B):
        for h in range(H):
            S = s0[b, h].copy()
            if keep_states:
                states[b, h, 0] = S
            for t in range(T):
                kt = k[b, t, h]
                Sp = np.exp(la[b, t, h])[:, None] * S
                w = bw[b, t, h] * v[b, t, h] - be[b, t, h] * (Sp.T @ kt)
                S = Sp + np.outer(kt, w)
                out[b, t, h] = S.T @ q[b, t, h]
                if keep_states:
                    states[b, h, t + 1] = S
            ST[b, h] = S
    return (out, ST, states) if keep_states else (out, ST)


def backward(q, k, v, log_alpha, beta, dout, S0=None, dS_T=None, beta_write=None):
    """Gradients of L = sum(dout * out) + sum(dS_T * S_T) with respect to every
    input of the recurrence, in fp64.

    Returns a dict with ``dq``, ``dk``, ``dv``, ``dlog_alpha`` (shapes of the
    inputs), ``dbeta`` ``[B,T,H]`` and ``dS0`` ``[B,H,dk,dv]``. With a separate
    ``beta_write``, ``dbeta`` is the erase strength's gradient and
    ``dbeta_write`` the write strength's; without one, ``dbeta`` is their sum.
    """
    k64, v64, la, be, dO = (_np64(x) for x in (k, v, log_alpha, beta, dout))
    q64 = _np64(q)
    bw = be if beta_write is None else _np64(beta_write)
    B, T, H, dk = q64.shape
    dv = v64.shape[-1]
    _, _, states = forward64(q64, k64, v64, la, be, S0, beta_write=bw, keep_states=True)
    g_T = np.zeros((B, H, dk, dv)) if dS_T is None else _np64(dS_T)
    dq = np.zeros_like(q64)
    dk_ = np.zeros_like(k64)
    dv_ = np.zeros_like(v64)
    dla = np.zeros_like(la)
    dbe = np.zeros_like(be)
    dbw = np.zeros_like(be)
    dS0 = np.zeros((B, H, dk, dv))
    for b in range(B):
        for h in range(H):
            G = g_T[b, h].copy()
            for t in range(T - 1, -1, -1):
                kt, qt, do = k64[b, t, h], q64[b, t, h], dO[b, t, h]
                alpha = np.exp(la[b, t, h])
                S_prev, S_t = states[b, h, t], states[b, h, t + 1]
                Sp = alpha[:, None] * S_prev
                r = Sp.T @ kt
                w = bw[b, t, h] * v64[b, t, h] - be[b, t, h] * r
                G = G + np.outer(qt, do)
                dq[b, t, h] = S_t @ do
                g = G.T @ kt
                dv_[b, t, h] = bw[b, t, h] * g
                dbw[b, t, h] = v64[b, t, h] @ g
                dbe[b, t, h] = -(r @ g)
                dk_[b, t, h] = G @ w - be[b, t, h] * (Sp @ g)
                dSp = G - be[b, t, h] * np.outer(kt, g)
                dla[b, t, h] = alpha * np.sum(dSp * S_prev, axis=1)
                G = alpha[:, None] * dSp
            dS0[b, h] = G
    res = {"dq": dq, "dk": dk_, "dv": dv_, "dlog_alpha": dla, "dS0": dS0}
    if beta_write is None:
        res["dbeta"] = dbe + dbw
    else:
        res["dbeta"] = dbe
        res["dbeta_write"] = dbw
    return res
