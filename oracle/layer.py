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
  * ShortConv is a causal depthwise convolution along the tokens of each
    sequence, one filter of width W = 4 per (head, channel), without bias:
    y_t = sum_{j=0}^{W-1} w[j] x_{t-j}, with x_{t-j} = 0 before the sequence's
    first token (no state crosses a sequence boundary). Swish is
    swish(y) = y * sigmoid(y). The order is ShortConv, Swish, then (q, k only)
    the L2 normalisation.
  * The per-head RMSNorm normalises each token-head's d_v output channels,
    o / sqrt(mean(o^2) + eps) * g_w, with a learned weight g_w per channel
    (shared by the heads) and eps = 1e-6. The data-dependent output gate
    multiplies channel-wise by sigmoid(z), z the gate's pre-activation per
    (token, head, channel): final = RMSNorm(o) * sigmoid(z).
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


def sigmoid(x):
    """1 / (1 + e^{-x}) in fp64, without overflow for large |x|."""
    x = _np64(x)
    e = np.exp(-np.abs(x))
    return np.where(x >= 0, 1.0 / (1.0 + e), e / (1.0 + e))


def swish(x):
    """x * sigmoid(x) (the SiLU)."""
    x = _np64(x)
    return x * sigmoid(x)


def short_conv(x, w, cu_seqlens=None):
    """Causal depthwise convolution along tokens: y_t = sum_j w[h, c, j] x_{t-j}.

    x [B,T,H,d] (or [total_T,H,d] packed, with cu_seqlens [N+1]); w [H,d,W].
    Tokens before a sequence's start count as zero. Plain loops over the taps."""
    x, w = _np64(x), _np64(w)
    W = w.shape[-1]
    if cu_seqlens is None:
        y = np.zeros_like(x)
        T = x.shape[1]
        for j in range(W):
            if j < T:
                y[:, j:] += w[None, None, :, :, j] * x[:, : T - j]
        return y
    cu = [int(c) for c in np.asarray(cu_seqlens)]
    y = np.zeros_like(x)
    for n in range(len(cu) - 1):
        y[cu[n]:cu[n + 1]] = short_conv(x[None, cu[n]:cu[n + 1]], w)[0]
    return y


def short_conv_swish(x, w, cu_seqlens=None):
    """swish(short_conv(x, w)), the layer's q/k/v prologue before the L2 norm."""
    return swish(short_conv(x, w, cu_seqlens))


def rms_norm_gate(o, z, g_w, eps=1e-6):
    """Per-head RMSNorm over the last (d_v) dimension, times the output gate:
    o / sqrt(mean(o^2) + eps) * g_w * sigmoid(z). o, z [..., d_v]; g_w [d_v]."""
    o, z, g_w = _np64(o), _np64(z), _np64(g_w)
    r = 1.0 / np.sqrt(np.mean(o * o, axis=-1, keepdims=True) + eps)
    return o * r * g_w * sigmoid(z)


def layer_core(q_raw, k_raw, v, gate_x, beta, out_gate, g_w, S0=None, eps=1e-6):
    """The KDA layer between its projections, in fp64: the recurrence on L2-normalised
    q, k and log alpha = -softplus(gate_x), then the per-head RMSNorm and the output
    gate on its output. Returns (final output, S_T)."""
    o, s = fused_forward(q_raw, k_raw, v, gate_x, beta, S0)
    return rms_norm_gate(o, out_gate, g_w, eps), s
