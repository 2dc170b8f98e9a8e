"""fp64 CPU oracle for Kimi Delta Attention (KDA) -- test infrastructure only.

This package is the checker that the CUDA library is compared against. It is
loaded only by ``tests/``, by the smoke check in ``__graft_entry__`` and by the
CPU-baseline leg of ``bench.py``; the product path never imports it. It shares
no code with the CUDA path: the only common module is ``kda_inputs`` (seeded
random inputs, no KDA arithmetic).

``forward`` runs the token-by-token recurrence of ``kda_oracle.c`` in fp64:
    S_t = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T,
    o_t = S_t^T q_t,
as the Kimi Linear summary (es.news.hada.io/topic?id=31936) describes it in its
sections "De la atencion lineal a Gated DeltaNet" (delta rule, scalar-gated
GDN) and "Control fino de memoria en Kimi Delta Attention" (per-channel
diagonal gate). ``decode_step`` is one step of the same recurrence applied to a
slot-indexed state cache. ``oracle.grad`` holds the backward pass of the same
recurrence (fp64 numpy).
"""
from __future__ import annotations

import contextlib
import ctypes
import os
import subprocess

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "kda_oracle.c")
_LIB = os.path.join(_HERE, "libkda_oracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile the C oracle into ``oracle/libkda_oracle.so`` (gcc, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c99",
               "-o", _LIB + ".tmp", _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(_LIB + ".tmp", _LIB)
    return _LIB


def _bind(path):
    lib = ctypes.CDLL(path)
    p = ctypes.c_void_p
    L = ctypes.c_long
    lib.kda_oracle_fwd.argtypes = [p, p, p, ctypes.c_int, p, p, p, p, p, p,
                                   L, L, L, L, L, p, L, ctypes.c_int]
    lib.kda_oracle_fwd.restype = ctypes.c_int
    lib.kda_oracle_max_threads.restype = ctypes.c_int
    return lib


def _load():
    global _lib
    if _lib is None:
        _lib = _bind(build())
    return _lib


@contextlib.contextmanager
def swapped_library(path):
    """Temporarily run ``forward`` on another build of the oracle source (used by
    the mutation test, which plants mistakes in copies of ``kda_oracle.c``)."""
    global _lib
    saved = _load()
    _lib = _bind(path)
    try:
        yield
    finally:
        _lib = saved


def max_threads() -> int:
    return int(_load().kda_oracle_max_threads())


def _as_input(x):
    """(numpy array, dtype code) for q/k/v: fp32 -> 0, bf16 -> 1 (raw bits)."""
    if isinstance(x, torch.Tensor):
        x = x.detach().cpu().contiguous()
        if x.dtype == torch.bfloat16:
            return x.view(torch.int16).numpy().view(np.uint16), 1
        return x.to(torch.float32).numpy(), 0
    return np.ascontiguousarray(x, dtype=np.float32), 0


def _f32(x):
    if x is None:
        return None
    if isinstance(x, torch.Tensor):
        return x.detach().cpu().to(torch.float32).contiguous().numpy()
    return np.ascontiguousarray(x, dtype=np.float32)


def _f64(x):
    if x is None:
        return None
    if isinstance(x, torch.Tensor):
        return x.detach().cpu().to(torch.float64).contiguous().numpy()
    return np.ascontiguousarray(x, dtype=np.float64)


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def forward(q, k, v, log_alpha, beta, S0=None, beta_write=None, heads=None, nthreads=0):
    """Run the fp64 recurrence.

    q, k ``[B,T,H,dk]`` and v ``[B,T,H,dv]`` (fp32 or bf16), log_alpha
    ``[B,T,H,dk]`` and beta ``[B,T,H]`` (fp32), optional S0 ``[B,H,dk,dv]``.
    ``beta`` is the erase strength; ``beta_write`` (default: ``beta``) is the
    write strength -- equal for KDA. ``heads`` optionally lists flat head
    indices ``b*H + h`` to compute; other heads are left as NaN.

    Returns ``(out [B,T,H,dv], S_T [B,H,dk,dv])`` as float64 numpy arrays.
    """
    qa, dt_q = _as_input(q)
    ka, dt_k = _as_input(k)
    va, dt_v = _as_input(v)
    if not (dt_q == dt_k == dt_v):
        raise TypeError("q, k and v must share one dtype")
    B, T, H, dk = qa.shape
    dv = va.shape[-1]
    if ka.shape != (B, T, H, dk) or va.shape != (B, T, H, dv):
        raise ValueError("q/k/v shapes disagree")
    la = _f32(log_alpha)
    be = _f32(beta)
    bw = _f32(beta_write)
    s0 = _f64(S0)
    if la.shape != (B, T, H, dk) or be.shape != (B, T, H):
        raise ValueError("gate shapes disagree with q")
    if bw is not None and bw.shape != (B, T, H):
        raise ValueError("beta_write shape")
    if s0 is not None and s0.shape != (B, H, dk, dv):
        raise ValueError("S0 shape")
    out = np.full((B, T, H, dv), np.nan, dtype=np.float64)
    st = np.full((B, H, dk, dv), np.nan, dtype=np.float64)
    hs = None
    if heads is not None:
        hs = np.ascontiguousarray(np.asarray(heads, dtype=np.int64).reshape(-1))
    rc = _load().kda_oracle_fwd(
        _ptr(qa), _ptr(ka), _ptr(va), dt_q, _ptr(la), _ptr(be), _ptr(bw), _ptr(s0),
        _ptr(out), _ptr(st), B, T, H, dk, dv, _ptr(hs), 0 if hs is None else len(hs),
        int(nthreads))
    if rc != 0:
        raise RuntimeError("kda_oracle_fwd failed (bad arguments or out of memory)")
    return out, st


def decode_step(q, k, v, log_alpha, beta, state, slot=None, rows=None, nthreads=0):
    """One decode step against a slot-indexed state cache, in fp64.

    q, k ``[N,H,dk]``, v ``[N,H,dv]``, log_alpha ``[N,H,dk]``, beta ``[N,H]``,
    state ``[slots,H,dk,dv]`` (not modified), slot ``[N]`` int (default: n).
    ``rows`` optionally restricts the step to some sequences n.

    Returns ``(out [n,H,dv], new_state [n,H,dk,dv])`` for the selected rows,
    where new_state[i] is the updated state of slot ``slot[rows[i]]``.
    """
    N = q.shape[0]
    rows = np.arange(N) if rows is None else np.asarray(rows, dtype=np.int64)
    slot = np.arange(N) if slot is None else np.asarray(
        slot.cpu() if isinstance(slot, torch.Tensor) else slot, dtype=np.int64)
    sel = torch.as_tensor(rows, dtype=torch.long)
    s0 = _f64(state)[slot[rows]]
    out, st = forward(q[sel].unsqueeze(1), k[sel].unsqueeze(1), v[sel].unsqueeze(1),
                      log_alpha[sel].unsqueeze(1), beta[sel].unsqueeze(1), S0=s0,
                      nthreads=nthreads)
    return out[:, 0], st
