"""fp64 oracle of the steps around the KDA recurrence in a Kimi Linear layer --
test infrastructure only (loaded by tests/, never by the product path).

The Kimi Linear summary (es.news.hada.io/topic?id=31936), section
"Configuracion del modelo Kimi Linear", lists what surrounds the recurrence in
a KDA layer:
  * q and k are L2-normalised (for the stability of the eigenvalues of the
    transition, whose Householder factor needs a unit key);
  * the per-channel decay comes from a low-rank, data-dependent gate, "similar
    to GDN and Mamba": the gate's pre-activation x (one value per channel)
    becomes log alpha = -softplus(x), so alpha = 1 / (1 + e^x) in (0, 1);
  * the value path and q/k pass through a short causal convolution with a
    Swish activation before the recurrence; the output goes through a
    per-head RMSNorm and a low-rank, data-dependent output gate.

Readings (the pages give no formulas for these steps):
  * L2 normalisation over the head dimension, x / ||x||_2; a zero vector stays
    zero.
  * The gate maps x to log alpha = -softplus(x) = -log(1 + e^x), the recipe of
    the workloads' gates; no per-head scale or bias.
  * The functions here take already-projected per-channel tensors: the
    low-rank projections themselves are plain matrix products outside the
    recurrence's hot path.

``recurrence`` is a second, independent fp64 implementation of the
token-by-token KDA recurrence (plain NumPy, vectorised over batch and heads);
its tests pin it to the C oracle, so each checks the other.
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


def softplus(x):
    """log(1 + e^x) in fp64, written so that it neither overflows nor loses
    precision: max(x, 0) + log1p(e^{-|x|})."""
    x = _np64(x)
    return np.maximum(x, 0.0) + np.log1p(np.exp(-np.abs(x)))


def gate_log_alpha(x):
    """log alpha = -softplus(x) for the gate pre-activation x (per channel)."""
    return -softplus(x)


def l2_normalize(x):
    """x / ||x||_2 over the last dimension (fp64); zero rows stay zero."""
    x = _np64(x)
    n = np.sqrt(np.sum(x * x, axis=-1, keepdims=True))
    return np.divide(x, n, out=np.zeros_like(x), where=n > 0)


def recurrence(q, k, v, log_alpha, beta, S0=None):
    """The KDA recurrence, token by token, in fp64:
        S_t = (I - beta_t k_t k_t^T) Diag(e^{log_alpha_t}) S_{t-1} + beta_t k_t v_t^T,
        o_t = S_t^T q_t.
    q, k, log_alpha [B,T,H,dk]; v [B,T,H,dv]; beta [B,T,H]; S0 [B,H,dk,dv] or None.
    Returns (out [B,T,H,dv], S_T [B,H,dk,dv]) as float64 arrays."""
    q, k, v, la, be = (_np64(t) for t in (q, k, v, log_alpha, beta))
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    S = np.zeros((B, H, dk, dv)) if S0 is None else _np64(S0).copy()
    out = np.zeros((B, T, H, dv))
    for t in range(T):
        S = np.exp(la[:, t])[..., None] * S                        # Diag(alpha_t) S
        kt, qt, vt, bt = k[:, t], q[:, t], v[:, t], be[:, t]
        r = np.einsum("bhi,bhij->bhj", kt, S)                      # S'^T k_t
        u = bt[..., None] * (vt - r)                               # beta (v - S'^T k)
        S = S + kt[..., None] * u[..., None, :]                    # + k u^T
        out[:, t] = np.einsum("bhi,bhij->bhj", qt, S)              # S_t^T q_t
    return out, S


def fused_forward(q_raw, k_raw, v, gate_x, beta, S0=None):
    """The recurrence fed through the layer's prologue: q and k L2-normalised,
    log alpha = -softplus(gate_x). All in fp64."""
    return recurrence(l2_normalize(q_raw), l2_normalize(k_raw), v, gate_log_alpha(gate_x), beta, S0)
