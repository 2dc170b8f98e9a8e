"""fp64 oracle of the general diagonal-plus-low-rank (DPLR) delta recurrence, the
comparator of KDA's operator efficiency -- test infrastructure only (loaded by
tests/ and by bench.py's CPU baseline, never by the product path).

The Kimi Linear summary (es.news.hada.io/topic?id=31936), section "Menor cantidad
de operaciones que DPLR general", compares KDA with the general DPLR transition:
both admit fine-grained decay, but KDA ties both low-rank vectors of the
transition to the key, which halves the secondary-chunk products (4 -> 2) and
removes 3 matrix products, for about twice the operator efficiency measured per
input length.

Reading (the page gives the claim, not the formula): the general DPLR recurrence
is, per head with a d_k x d_v state S,
    S_t = (Diag(alpha_t) + a_t b_t^T) S_{t-1} + k_t v_t^T,   o_t = S_t^T q_t,
with alpha_t = e^{log_alpha_t} per channel and a_t, b_t, k_t free d_k-vectors.
KDA is the case a_t = -beta_t k_t, b_t = alpha_t * k_t, and the write vector
beta_t k_t: (I - beta k k^T) Diag(alpha) = Diag(alpha) - beta k (alpha * k)^T.
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


def forward(q, k, v, a, b, log_alpha, S0=None):
    """The general DPLR recurrence token by token in fp64.

    q, k, a, b, log_alpha [B,T,H,dk]; v [B,T,H,dv]; S0 [B,H,dk,dv] or None.
    Returns (out [B,T,H,dv], S_T [B,H,dk,dv]) as float64 arrays."""
    q, k, v, a, b, la = (_np64(t) for t in (q, k, v, a, b, log_alpha))
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    S = np.zeros((B, H, dk, dv)) if S0 is None else _np64(S0).copy()
    out = np.zeros((B, T, H, dv))
    for t in range(T):
        probe = np.einsum("bhi,bhij->bhj", b[:, t], S)              # b_t^T S_{t-1}
        S = np.exp(la[:, t])[..., None] * S                          # Diag(alpha_t) S_{t-1}
        S = S + a[:, t][..., None] * probe[..., None, :]             # + a_t (b_t^T S_{t-1})
        S = S + k[:, t][..., None] * v[:, t][..., None, :]           # + k_t v_t^T
        out[:, t] = np.einsum("bhi,bhij->bhj", q[:, t], S)           # S_t^T q_t
    return out, S


def kda_as_dplr(k, log_alpha, beta):
    """The (a, b, write vector) of the general form that reproduce KDA's transition:
    a = -beta k, b = e^{log_alpha} * k, write vector beta k."""
    k, la, be = _np64(k), _np64(log_alpha), _np64(beta)
    bk = be[..., None] * k
    return -bk, np.exp(la) * k, bk
