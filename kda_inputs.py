"""Seeded synthetic inputs for Kimi Delta Attention (KDA) workloads.

This module is shared by the fp64 oracle (``oracle/``) and the CUDA path
(``gated_delta_rule_116_b200``). It holds no KDA arithmetic: it only draws
random tensors with the shapes and value distributions of the workloads and
returns them. Both sides receive the same tensors.

Workloads (one dict per entry of ``WORKLOADS``):

* ``fp32_small``   B=1,  H=2,  T=64,     d=16,  chunk=16, fp32 q/k/v, S0 = 0
* ``prefill_4k``   B=8,  H=32, T=4096,   d=128, chunk=64, bf16 q/k/v, S0 = 0
* ``prefill_32k``  B=1,  H=32, T=32768,  d=128, chunk=64, bf16 q/k/v,
                   slow forgetting (log a = -softplus(N(-2,1))), S0 ~ N(0, 0.01)
* ``decode_256``   256 sequences x H=32, d=128, one token per step, fp32 state
                   cache ~ N(0, 0.05), bf16 q/k/v
* ``prefill_128k`` B=1,  H=16, T=131072, d=128, chunk=64, bf16 q/k/v, half the
                   channels with log a = -1e-3, the other half -softplus(N(0,1))

Edge-case gate recipe ``strong`` (parity tests only): channel c gets, for every
token, log a = -4 if c % 8 == 0 (a chunk of 64 tokens decays by e^-256),
0 if c % 8 == 1 (no forgetting), -12 if c % 8 == 2 (a ~ 6e-6: the channel keeps
almost nothing from one token to the next), -1e-3 if c % 8 == 3, and
-softplus(N(0,1)) otherwise. It stresses the range of the gate factors of the
chunked form (the fine-grained decay that the Kimi Linear summary names as the
precision problem inside a chunk).

Recipe (all workloads): q, k ~ N(0,1), L2-normalised over the head dimension
per (batch, token, head) in fp32 and then cast to the workload's dtype; v ~
N(0,1); beta = sigmoid(N(0,1)); log a = -softplus(N(0,1)) per channel unless
stated. ``N(m, s)`` means mean m and standard deviation s. One generator,
seeded with the workload's seed, draws in the order q, k, v, beta logits,
gate logits, S0. Layouts are token-major with heads interleaved:
q, k, log_alpha ``[B,T,H,dk]``; v ``[B,T,H,dv]``; beta ``[B,T,H]``;
S0 ``[B,H,dk,dv]``.
"""
from __future__ import annotations

import dataclasses

import torch


@dataclasses.dataclass(frozen=True)
class Prefill:
    name: str
    B: int
    T: int
    H: int
    dk: int
    dv: int
    chunk: int
    dtype: torch.dtype          # dtype of q, k, v and out
    gate: str = "softplus01"    # softplus01 | slow | mixed | strong
    s0_std: float = 0.0         # 0 -> no initial state (S0 = None)
    seed: int = 0

    @property
    def tokens(self) -> int:
        return self.B * self.T


@dataclasses.dataclass(frozen=True)
class Decode:
    name: str
    N: int                      # sequences (state slots), one new token each per step
    H: int
    dk: int
    dv: int
    steps: int
    dtype: torch.dtype
    state_std: float = 0.05
    seed: int = 3


WORKLOADS = {
    "fp32_small": Prefill("fp32_small", 1, 64, 2, 16, 16, 16, torch.float32, seed=0),
    "prefill_4k": Prefill("prefill_4k", 8, 4096, 32, 128, 128, 64, torch.bfloat16, seed=1),
    "prefill_32k": Prefill("prefill_32k", 1, 32768, 32, 128, 128, 64, torch.bfloat16,
                           gate="slow", s0_std=0.01, seed=2),
    "decode_256": Decode("decode_256", 256, 32, 128, 128, 1000, torch.bfloat16, seed=3),
    "prefill_128k": Prefill("prefill_128k", 1, 131072, 16, 128, 128, 64, torch.bfloat16,
                            gate="mixed", seed=4),
}


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def _unit_rows(x: torch.Tensor) -> torch.Tensor:
    """Scale each row (last dim) to unit Euclidean length, in fp32."""
    x = x.float()
    return x / x.norm(dim=-1, keepdim=True).clamp_min(1e-12)


def _gates(logits: torch.Tensor, mode: str) -> torch.Tensor:
    """log a from N(0,1) gate logits, following the workload's gate recipe."""
    if mode == "softplus01":
        return -torch.nn.functional.softplus(logits)
    if mode == "slow":                                   # -softplus(N(-2, 1))
        return -torch.nn.functional.softplus(logits - 2.0)
    if mode == "mixed":                                  # half -1e-3, half -softplus(N(0,1))
        out = -torch.nn.functional.softplus(logits)
        out[..., : out.shape[-1] // 2] = -1e-3
        return out
    if mode == "strong":                                 # per channel c % 8: -4, 0, -12, -1e-3
        out = -torch.nn.functional.softplus(logits)
        out[..., 0::8] = -4.0
        out[..., 1::8] = 0.0
        out[..., 2::8] = -12.0
        out[..., 3::8] = -1e-3
        return out
    raise ValueError(f"unknown gate recipe {mode!r}")


def prefill_inputs(w: Prefill | str, device="cpu", **override) -> dict:
    """Draw the inputs of a prefill workload.

    ``override`` replaces fields of the workload (e.g. ``T=256, B=1``) to get a
    smaller case with the same distributions. Returns a dict with q, k, v,
    log_alpha, beta, S0 (None when the workload has no initial state) and the
    workload itself under ``"w"``.
    """
    if isinstance(w, str):
        w = WORKLOADS[w]
    if override:
        w = dataclasses.replace(w, **override)
    g = _gen(w.seed, device)
    B, T, H, dk, dv = w.B, w.T, w.H, w.dk, w.dv
    f32 = dict(device=device, dtype=torch.float32, generator=g)
    q = _unit_rows(torch.randn(B, T, H, dk, **f32)).to(w.dtype)
    k = _unit_rows(torch.randn(B, T, H, dk, **f32)).to(w.dtype)
    v = torch.randn(B, T, H, dv, **f32).to(w.dtype)
    beta = torch.sigmoid(torch.randn(B, T, H, **f32))
    log_alpha = _gates(torch.randn(B, T, H, dk, **f32), w.gate)
    S0 = None
    if w.s0_std > 0:
        S0 = torch.randn(B, H, dk, dv, **f32) * w.s0_std
    return dict(q=q.contiguous(), k=k.contiguous(), v=v.contiguous(),
                log_alpha=log_alpha.contiguous(), beta=beta.contiguous(), S0=S0, w=w)


# Gate pre-activations x with -softplus(x) equal to the fixed log a values of the gate
# recipes (log(e^{-log a} - 1)); "no forgetting" (log a = 0) has no finite x and takes
# x = -30 (log a = -9e-14).
_X_FOR_LOG_A = {-1e-3: -6.907255, -4.0: 3.9814331, -12.0: 11.999994, 0.0: -30.0}


def prefill_layer_inputs(w: Prefill | str, device="cpu", **override) -> dict:
    """Inputs of the fused layer prologue: raw (un-normalised) q and k, v, the gate's
    pre-activation x, beta and S0, all in the workload's dtype except beta and S0 (fp32).

    The same draws as ``prefill_inputs`` (same generator and order), with q and k
    left un-normalised and the gate logits turned into the x for which -softplus(x)
    is the workload's log a: x = logits (softplus01), logits - 2 (slow), or the
    fixed values above for the recipe's fixed channels.
    """
    if isinstance(w, str):
        w = WORKLOADS[w]
    if override:
        w = dataclasses.replace(w, **override)
    g = _gen(w.seed, device)
    B, T, H, dk, dv = w.B, w.T, w.H, w.dk, w.dv
    f32 = dict(device=device, dtype=torch.float32, generator=g)
    q = torch.randn(B, T, H, dk, **f32).to(w.dtype)
    k = torch.randn(B, T, H, dk, **f32).to(w.dtype)
    v = torch.randn(B, T, H, dv, **f32).to(w.dtype)
    beta = torch.sigmoid(torch.randn(B, T, H, **f32))
    x = torch.randn(B, T, H, dk, **f32)
    if w.gate == "slow":
        x = x - 2.0
    elif w.gate == "mixed":
        x[..., : dk // 2] = _X_FOR_LOG_A[-1e-3]
    elif w.gate == "strong":
        x[..., 0::8] = _X_FOR_LOG_A[-4.0]
        x[..., 1::8] = _X_FOR_LOG_A[0.0]
        x[..., 2::8] = _X_FOR_LOG_A[-12.0]
        x[..., 3::8] = _X_FOR_LOG_A[-1e-3]
    elif w.gate != "softplus01":
        raise ValueError(f"unknown gate recipe {w.gate!r}")
    S0 = None
    if w.s0_std > 0:
        S0 = torch.randn(B, H, dk, dv, **f32) * w.s0_std
    return dict(q=q.contiguous(), k=k.contiguous(), v=v.contiguous(), gate=x.to(w.dtype).contiguous(),
                beta=beta.contiguous(), S0=S0, w=w)


def layer_extras(w: Prefill | str, device="cpu", conv_width: int = 4, **override) -> dict:
    """Seeded synthetic weights and data of the layer steps around the recurrence (the
    pages give no trained weights): the output gate's pre-activation z ~ N(0,1)
    ``[B,T,H,dv]`` (workload dtype), the RMSNorm weight 1 + 0.1 N(0,1) ``[dv]`` fp32,
    ShortConv filters for q, k and v ~ N(0, 0.5^2) ``[H,d,conv_width]`` fp32, and
    pre-convolution inputs x_q, x_k, x_v ~ N(0,1) ``[B,T,H,d]`` (workload dtype).
    Drawn from the workload's seed + 1000, in that order."""
    if isinstance(w, str):
        w = WORKLOADS[w]
    if override:
        w = dataclasses.replace(w, **override)
    g = _gen(w.seed + 1000, device)
    B, T, H, dk, dv = w.B, w.T, w.H, w.dk, w.dv
    f32 = dict(device=device, dtype=torch.float32, generator=g)
    z = torch.randn(B, T, H, dv, **f32).to(w.dtype).contiguous()
    norm_w = (1.0 + 0.1 * torch.randn(dv, **f32)).contiguous()
    conv = {n: (0.5 * torch.randn(H, d, conv_width, **f32)).contiguous()
            for n, d in (("q", dk), ("k", dk), ("v", dv))}
    pre = {n: torch.randn(B, T, H, d, **f32).to(w.dtype).contiguous()
           for n, d in (("q", dk), ("k", dk), ("v", dv))}
    return dict(out_gate=z, norm_weight=norm_w, conv_q=conv["q"], conv_k=conv["k"], conv_v=conv["v"],
                x_q=pre["q"], x_k=pre["k"], x_v=pre["v"], w=w)


def dplr_inputs(w: Prefill | str, device="cpu", **override) -> dict:
    """Inputs of the general DPLR recurrence S_t = (Diag(alpha_t) + a_t b_t^T) S_{t-1} + k_t v_t^T
    (the comparator of KDA's operator efficiency): q, k, v, log alpha and S0 as
    ``prefill_inputs`` (same draws), and two low-rank vectors drawn from the workload's
    seed + 2000: a = -gamma * unit(r1) with gamma = sigmoid(N(0,1)) per token, and
    b = e^{log alpha} * unit(r1 + 0.5 r2) (r1, r2 ~ N(0,1) per channel), so that a and b
    differ but the transition stays contracting, as KDA's does. a and b in the
    workload's dtype."""
    base = prefill_inputs(w, device=device, **override)
    w = base["w"]
    g = _gen(w.seed + 2000, device)
    f32 = dict(device=device, dtype=torch.float32, generator=g)
    B, T, H, dk = w.B, w.T, w.H, w.dk
    r1 = torch.randn(B, T, H, dk, **f32)
    r2 = torch.randn(B, T, H, dk, **f32)
    gamma = torch.sigmoid(torch.randn(B, T, H, **f32))
    a = -gamma[..., None] * _unit_rows(r1)
    b = torch.exp(base["log_alpha"]) * _unit_rows(r1 + 0.5 * r2)
    base["a"] = a.to(w.dtype).contiguous()
    base["b"] = b.to(w.dtype).contiguous()
    return base


def packed_lengths(n: int, lo: int, hi: int, seed: int = 5) -> list[int]:
    """Lengths of n packed sequences for the variable-length prefill: uniform integers
    in [lo, hi] from a generator seeded with `seed` (a mix of short and long prompts)."""
    g = torch.Generator().manual_seed(int(seed))
    return [int(x) for x in torch.randint(lo, hi + 1, (n,), generator=g)]


def decode_state(w: Decode | str = "decode_256", device="cpu", **override) -> torch.Tensor:
    """The initial fp32 state cache ``[N, H, dk, dv]`` ~ N(0, state_std)."""
    if isinstance(w, str):
        w = WORKLOADS[w]
    if override:
        w = dataclasses.replace(w, **override)
    g = _gen(w.seed, device)
    return torch.randn(w.N, w.H, w.dk, w.dv, device=device, dtype=torch.float32,
                       generator=g) * w.state_std


def decode_step_inputs(w: Decode | str, step: int, device="cpu", **override) -> dict:
    """Inputs of decode step ``step``: q, k, v ``[N,H,d]``, log_alpha ``[N,H,dk]``, beta ``[N,H]``.

    Each step has its own generator (seeded from the workload seed and the step
    index), so any step can be redrawn on its own.
    """
    if isinstance(w, str):
        w = WORKLOADS[w]
    if override:
        w = dataclasses.replace(w, **override)
    g = _gen(w.seed * 1_000_003 + 1 + step, device)
    N, H, dk, dv = w.N, w.H, w.dk, w.dv
    f32 = dict(device=device, dtype=torch.float32, generator=g)
    q = _unit_rows(torch.randn(N, H, dk, **f32)).to(w.dtype)
    k = _unit_rows(torch.randn(N, H, dk, **f32)).to(w.dtype)
    v = torch.randn(N, H, dv, **f32).to(w.dtype)
    beta = torch.sigmoid(torch.randn(N, H, **f32))
    log_alpha = -torch.nn.functional.softplus(torch.randn(N, H, dk, **f32))
    return dict(q=q.contiguous(), k=k.contiguous(), v=v.contiguous(),
                log_alpha=log_alpha.contiguous(), beta=beta.contiguous())
