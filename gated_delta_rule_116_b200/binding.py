"""ctypes binding of libkda (``include/kda.h``) for torch tensors.

Argument marshalling only: every step of the computation runs in the CUDA
kernels of ``libkda.so``. There is no CPU or PyTorch fallback -- if the library
is missing, or the tensors are not on a CUDA device, the calls raise.
"""
from __future__ import annotations

import ctypes
import os

import torch

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libkda.so")

KDA_BF16, KDA_F32 = 0, 1
ENGINES = {"auto": 0, "generic": 1, "tc_cluster": 3}
_DTYPES = {torch.bfloat16: KDA_BF16, torch.float32: KDA_F32}

_lib = None


class KdaError(RuntimeError):
    def __init__(self, code: int, name: str, detail: str):
        super().__init__(f"{name} ({code}): {detail}")
        self.code = code
        self.name = name
        self.detail = detail


def load():
    """Load libkda.so (once). Raises if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"libkda.so is not built ({LIB_PATH}); run "
                           "`python -m gated_delta_rule_116_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    p, i, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
    lib.kda_workspace_bytes.argtypes = [i, i, i, i, i, i, i]
    lib.kda_workspace_bytes.restype = sz
    chunk_args = [p, p, p, p, p, p, p, p, i, i, i, i, i, i, i, p, sz, p]
    lib.kda_chunk_fwd.argtypes = chunk_args
    lib.kda_chunk_fwd.restype = i
    lib.kda_chunk_fwd_engine.argtypes = [i] + chunk_args
    lib.kda_chunk_fwd_fused.argtypes = chunk_args
    lib.kda_chunk_fwd_fused.restype = i
    lib.kda_chunk_fwd_engine.restype = i
    lib.kda_engine_supported.argtypes = [i, i, i, i, i]
    lib.kda_engine_supported.restype = i
    lib.kda_chunk_fwd_varlen.argtypes = [p] * 10 + [i, i, i, i, i, i, p]
    lib.kda_chunk_fwd_varlen.restype = i
    lib.kda_chunk_fwd_varlen_engine.argtypes = [i] + [p] * 10 + [i, i, i, i, i, i, p, sz, p]
    lib.kda_chunk_fwd_varlen_engine.restype = i
    lib.kda_layer_fwd.argtypes = [p, p, p, p, p, p, p, ctypes.c_float, p, p, p, i, i, i, i, i, i, i, p, sz, p]
    lib.kda_layer_fwd.restype = i
    lib.kda_dplr_chunk_fwd.argtypes = [p] * 9 + [i] * 7 + [p]
    lib.kda_dplr_chunk_fwd.restype = i
    lib.kda_short_conv_swish.argtypes = [p, p, p, p, i, i, i, i, i, i, p]
    lib.kda_short_conv_swish.restype = i
    lib.kda_varlen_workspace_bytes.argtypes = [i, i, i, i, i]
    lib.kda_varlen_workspace_bytes.restype = sz
    lib.kda_chunk_bwd.argtypes = [p] * 14 + [i, i, i, i, i, i, p, sz, p]
    lib.kda_chunk_bwd.restype = i
    lib.kda_bwd_workspace_bytes.argtypes = [i, i, i, i, i, i]
    lib.kda_bwd_workspace_bytes.restype = sz
    lib.kda_recurrent_step.argtypes = [p, p, p, p, p, p, p, p, i, i, i, i, i, p]
    lib.kda_recurrent_step.restype = i
    lib.kda_strerror.argtypes = [i]
    lib.kda_strerror.restype = ctypes.c_char_p
    lib.kda_last_error_detail.argtypes = []
    lib.kda_last_error_detail.restype = ctypes.c_char_p
    lib.kda_device_status.argtypes = [p]
    lib.kda_test_inject_wait_timeout.argtypes = [i]
    lib.kda_test_inject_wait_timeout.restype = i
    lib.kda_device_status.restype = i
    lib.kda_version.restype = i
    _lib = lib
    return lib


def _check(rc: int):
    if rc != 0:
        lib = load()
        raise KdaError(rc, lib.kda_strerror(rc).decode(), lib.kda_last_error_detail().decode())


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(device, stream):
    if stream is None:
        stream = torch.cuda.current_stream(device)
    return ctypes.c_void_p(stream.cuda_stream)


def _require(t, name, device, dtype=None, shape=None):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.device.type != "cuda":
        raise ValueError(f"{name} must be on a CUDA device (got {t.device})")
    if t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype} (got {t.dtype})")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)} (got {tuple(t.shape)})")


def engine_supported(engine: str, dk: int, dv: int, chunk: int, dtype=torch.bfloat16) -> bool:
    return bool(load().kda_engine_supported(ENGINES[engine], dk, dv, chunk, _DTYPES[dtype]))


def workspace_bytes(B, T, H, dk, dv, chunk=64, dtype=torch.bfloat16) -> int:
    return int(load().kda_workspace_bytes(B, T, H, dk, dv, chunk, _DTYPES[dtype]))


def bwd_workspace_bytes(B, T, H, dk, dv, dtype=torch.bfloat16) -> int:
    """Device scratch that ``chunk_bwd`` needs (``kda_bwd_workspace_bytes``)."""
    return int(load().kda_bwd_workspace_bytes(B, T, H, dk, dv, _DTYPES[dtype]))


def chunk_fwd(q, k, v, log_alpha, beta, S0=None, chunk: int = 64, *, out=None, S_T=None,
              output_final_state: bool = True, engine: str = "auto", workspace=None, stream=None):
    """Chunked KDA prefill (``kda_chunk_fwd``).

    q, k ``[B,T,H,dk]``, v ``[B,T,H,dv]`` (bf16 or fp32, same dtype);
    log_alpha ``[B,T,H,dk]`` and beta ``[B,T,H]`` fp32; S0 ``[B,H,dk,dv]`` fp32 or
    None. Returns ``(out, S_T)``; ``S_T`` is None when ``output_final_state`` is
    False and no ``S_T`` buffer is given. ``S_T`` may be ``S0`` (in place).
    """
    lib = load()
    device = q.device
    _require(q, "q", device)
    if q.dtype not in _DTYPES:
        raise TypeError(f"q must be bf16 or fp32 (got {q.dtype})")
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    _require(k, "k", device, q.dtype, (B, T, H, dk))
    _require(v, "v", device, q.dtype, (B, T, H, dv))
    _require(log_alpha, "log_alpha", device, torch.float32, (B, T, H, dk))
    _require(beta, "beta", device, torch.float32, (B, T, H))
    if S0 is not None:
        _require(S0, "S0", device, torch.float32, (B, H, dk, dv))
    if out is None:
        out = torch.empty(B, T, H, dv, device=device, dtype=q.dtype)
    _require(out, "out", device, q.dtype, (B, T, H, dv))
    if S_T is None and output_final_state:
        S_T = torch.empty(B, H, dk, dv, device=device, dtype=torch.float32)
    if S_T is not None:
        _require(S_T, "S_T", device, torch.float32, (B, H, dk, dv))
    need = int(lib.kda_workspace_bytes(B, T, H, dk, dv, chunk, _DTYPES[q.dtype]))
    if workspace is None and need > 0:
        workspace = torch.empty(need, device=device, dtype=torch.uint8)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    if engine not in ENGINES:
        raise ValueError(f"engine must be one of {sorted(ENGINES)}")
    with torch.cuda.device(device):
        rc = lib.kda_chunk_fwd_engine(
            ENGINES[engine], _ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta), _ptr(S0),
            _ptr(out), _ptr(S_T), B, T, H, dk, dv, chunk, _DTYPES[q.dtype], _ptr(workspace),
            ws_bytes, _stream(device, stream))
    _check(rc)
    return out, S_T


def chunk_fwd_fused(q, k, v, gate, beta, S0=None, chunk: int = 64, *, out=None, S_T=None,
                    output_final_state: bool = True, workspace=None, stream=None):
    """Chunked prefill with the layer prologue fused in (``kda_chunk_fwd_fused``):
    q and k are L2-normalised and log_alpha = -softplus(gate) inside the kernel.

    q, k ``[B,T,H,128]`` (un-normalised), v ``[B,T,H,128]`` and gate ``[B,T,H,128]``
    (the gate's pre-activation), all bf16; beta ``[B,T,H]`` fp32; S0 as ``chunk_fwd``.
    Returns ``(out, S_T)`` like ``chunk_fwd``.
    """
    lib = load()
    device = q.device
    _require(q, "q", device, torch.bfloat16)
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    _require(k, "k", device, torch.bfloat16, (B, T, H, dk))
    _require(v, "v", device, torch.bfloat16, (B, T, H, dv))
    _require(gate, "gate", device, torch.bfloat16, (B, T, H, dk))
    _require(beta, "beta", device, torch.float32, (B, T, H))
    if S0 is not None:
        _require(S0, "S0", device, torch.float32, (B, H, dk, dv))
    if out is None:
        out = torch.empty(B, T, H, dv, device=device, dtype=torch.bfloat16)
    _require(out, "out", device, torch.bfloat16, (B, T, H, dv))
    if S_T is None and output_final_state:
        S_T = torch.empty(B, H, dk, dv, device=device, dtype=torch.float32)
    if S_T is not None:
        _require(S_T, "S_T", device, torch.float32, (B, H, dk, dv))
    need = int(lib.kda_workspace_bytes(B, T, H, dk, dv, chunk, KDA_BF16))
    if workspace is None and need > 0:
        workspace = torch.empty(need, device=device, dtype=torch.uint8)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    with torch.cuda.device(device):
        rc = lib.kda_chunk_fwd_fused(
            _ptr(q), _ptr(k), _ptr(v), _ptr(gate), _ptr(beta), _ptr(S0), _ptr(out), _ptr(S_T),
            B, T, H, dk, dv, chunk, KDA_BF16, _ptr(workspace), ws_bytes, _stream(device, stream))
    _check(rc)
    return out, S_T


def layer_fwd(q, k, v, gate, beta, out_gate, norm_weight, S0=None, eps: float = 1e-6, chunk: int = 64, *,
              out=None, S_T=None, output_final_state: bool = True, workspace=None, stream=None):
    """The KDA layer between its projections (``kda_layer_fwd``): ``chunk_fwd_fused`` followed
    by the per-head RMSNorm and the sigmoid output gate on every output row, in one kernel.

    q, k, v, gate as ``chunk_fwd_fused``; out_gate ``[B,T,H,128]`` bf16 (the output gate's
    pre-activation); norm_weight ``[128]`` fp32. Returns ``(out, S_T)``.
    """
    lib = load()
    device = q.device
    _require(q, "q", device, torch.bfloat16)
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    _require(k, "k", device, torch.bfloat16, (B, T, H, dk))
    _require(v, "v", device, torch.bfloat16, (B, T, H, dv))
    _require(gate, "gate", device, torch.bfloat16, (B, T, H, dk))
    _require(beta, "beta", device, torch.float32, (B, T, H))
    _require(out_gate, "out_gate", device, torch.bfloat16, (B, T, H, dv))
    _require(norm_weight, "norm_weight", device, torch.float32, (dv,))
    if S0 is not None:
        _require(S0, "S0", device, torch.float32, (B, H, dk, dv))
    if out is None:
        out = torch.empty(B, T, H, dv, device=device, dtype=torch.bfloat16)
    _require(out, "out", device, torch.bfloat16, (B, T, H, dv))
    if S_T is None and output_final_state:
        S_T = torch.empty(B, H, dk, dv, device=device, dtype=torch.float32)
    if S_T is not None:
        _require(S_T, "S_T", device, torch.float32, (B, H, dk, dv))
    need = int(lib.kda_workspace_bytes(B, T, H, dk, dv, chunk, KDA_BF16))
    if workspace is None and need > 0:
        workspace = torch.empty(need, device=device, dtype=torch.uint8)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    with torch.cuda.device(device):
        rc = lib.kda_layer_fwd(
            _ptr(q), _ptr(k), _ptr(v), _ptr(gate), _ptr(beta), _ptr(out_gate), _ptr(norm_weight),
            float(eps), _ptr(S0), _ptr(out), _ptr(S_T), B, T, H, dk, dv, chunk, KDA_BF16,
            _ptr(workspace), ws_bytes, _stream(device, stream))
    _check(rc)
    return out, S_T


def varlen_workspace_bytes(N, H, dk, dv, dtype=torch.bfloat16) -> int:
    """Device scratch of the tensor-core engine of ``chunk_fwd_varlen`` (``kda_varlen_workspace_bytes``)."""
    return int(load().kda_varlen_workspace_bytes(N, H, dk, dv, _DTYPES[dtype]))


def chunk_fwd_varlen(q, k, v, log_alpha, beta, cu_seqlens, S0=None, *, slot=None, out=None,
                     S_T=None, output_final_state: bool = True, engine: str = "auto",
                     workspace=None, stream=None):
    """Chunked prefill of packed variable-length sequences (``kda_chunk_fwd_varlen_engine``).

    q, k ``[total_T,H,dk]``, v ``[total_T,H,dv]`` (bf16 or fp32), log_alpha
    ``[total_T,H,dk]`` and beta ``[total_T,H]`` fp32, cu_seqlens ``[N+1]`` int32
    token offsets on the device. Without ``slot``, S0 and S_T are ``[N,H,dk,dv]``.
    With ``slot`` (``[N]`` int32), they are a state cache ``[slots,H,dk,dv]``
    (the decode step's) and sequence n uses row ``slot[n]``; S_T then defaults
    to S0, updated in place. ``engine`` is "auto" (the tensor-core engine where it
    supports the shape: bf16, dk = dv = 128), "tc_cluster" or "generic" (fp32 CUDA
    cores); the tensor-core engine's ``workspace`` is allocated when not given.
    Returns ``(out, S_T)``.
    """
    lib = load()
    device = q.device
    _require(q, "q", device)
    if q.dtype not in _DTYPES:
        raise TypeError(f"q must be bf16 or fp32 (got {q.dtype})")
    TT, H, dk = q.shape
    dv = v.shape[-1]
    _require(k, "k", device, q.dtype, (TT, H, dk))
    _require(v, "v", device, q.dtype, (TT, H, dv))
    _require(log_alpha, "log_alpha", device, torch.float32, (TT, H, dk))
    _require(beta, "beta", device, torch.float32, (TT, H))
    _require(cu_seqlens, "cu_seqlens", device, torch.int32)
    if cu_seqlens.dim() != 1 or cu_seqlens.numel() < 1:
        raise ValueError("cu_seqlens must be a 1-D tensor of N+1 offsets")
    N = cu_seqlens.numel() - 1
    if slot is not None:
        _require(slot, "slot", device, torch.int32, (N,))
        if S_T is None and output_final_state:
            if S0 is None:
                raise ValueError("with a slot map, give the state cache as S0 or S_T")
            S_T = S0
        for t, name in ((S0, "S0"), (S_T, "S_T")):
            if t is not None:
                _require(t, name, device, torch.float32)
                if t.dim() != 4 or tuple(t.shape[1:]) != (H, dk, dv):
                    raise ValueError(f"{name} must be [slots,{H},{dk},{dv}] (got {tuple(t.shape)})")
    else:
        if S0 is not None:
            _require(S0, "S0", device, torch.float32, (N, H, dk, dv))
        if S_T is None and output_final_state:
            S_T = torch.empty(N, H, dk, dv, device=device, dtype=torch.float32)
        if S_T is not None:
            _require(S_T, "S_T", device, torch.float32, (N, H, dk, dv))
    if out is None:
        out = torch.empty(TT, H, dv, device=device, dtype=q.dtype)
    _require(out, "out", device, q.dtype, (TT, H, dv))
    if engine not in ENGINES:
        raise ValueError(f"unknown engine {engine!r}")
    ws_bytes = 0
    if engine != "generic" and TT > 0:
        need = int(lib.kda_varlen_workspace_bytes(N, H, dk, dv, _DTYPES[q.dtype]))
        if need > 0 and workspace is None:
            workspace = torch.empty(need, device=device, dtype=torch.uint8)
    if workspace is not None:
        _require(workspace, "workspace", device, torch.uint8)
        ws_bytes = workspace.numel()
    with torch.cuda.device(device):
        rc = lib.kda_chunk_fwd_varlen_engine(
            ENGINES[engine], _ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta), _ptr(cu_seqlens),
            _ptr(slot), _ptr(S0), _ptr(out), _ptr(S_T), N, TT, H, dk, dv, _DTYPES[q.dtype],
            _ptr(workspace), ws_bytes, _stream(device, stream))
    _check(rc)
    return out, S_T


def dplr_chunk_fwd(q, k, v, a, b, log_alpha, S0=None, chunk: int = 32, *, out=None, S_T=None,
                   output_final_state: bool = True, stream=None):
    """The general DPLR comparator (``kda_dplr_chunk_fwd``): S_t = (Diag(alpha_t) + a_t b_t^T)
    S_{t-1} + k_t v_t^T, o_t = S_t^T q_t, fp32 CUDA cores. q, k, a, b ``[B,T,H,dk]`` and v in
    one dtype (bf16 or fp32), log_alpha fp32. Returns ``(out, S_T)``."""
    lib = load()
    device = q.device
    _require(q, "q", device)
    if q.dtype not in _DTYPES:
        raise TypeError(f"q must be bf16 or fp32 (got {q.dtype})")
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    for t, name in ((k, "k"), (a, "a"), (b, "b")):
        _require(t, name, device, q.dtype, (B, T, H, dk))
    _require(v, "v", device, q.dtype, (B, T, H, dv))
    _require(log_alpha, "log_alpha", device, torch.float32, (B, T, H, dk))
    if S0 is not None:
        _require(S0, "S0", device, torch.float32, (B, H, dk, dv))
    if out is None:
        out = torch.empty(B, T, H, dv, device=device, dtype=q.dtype)
    if S_T is None and output_final_state:
        S_T = torch.empty(B, H, dk, dv, device=device, dtype=torch.float32)
    with torch.cuda.device(device):
        rc = lib.kda_dplr_chunk_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(a), _ptr(b), _ptr(log_alpha), _ptr(S0),
                                    _ptr(out), _ptr(S_T), B, T, H, dk, dv, chunk, _DTYPES[q.dtype],
                                    _stream(device, stream))
    _check(rc)
    return out, S_T


def short_conv_swish(x, weight, cu_seqlens=None, *, out=None, stream=None):
    """ShortConv + Swish (``kda_short_conv_swish``): y_t = swish(sum_j weight[h,c,j] x_{t-j}),
    causal per sequence. x ``[B,T,H,d]`` (or packed ``[T,H,d]`` with ``cu_seqlens``
    ``[N+1]`` int32), bf16 or fp32; weight ``[H,d,W]`` fp32 with W <= 4. Returns y."""
    lib = load()
    device = x.device
    _require(x, "x", device)
    if x.dtype not in _DTYPES:
        raise TypeError(f"x must be bf16 or fp32 (got {x.dtype})")
    if cu_seqlens is None:
        B, T, H, d = x.shape
    else:
        T, H, d = x.shape
        _require(cu_seqlens, "cu_seqlens", device, torch.int32)
        B = cu_seqlens.numel() - 1
    if weight.dim() != 3 or tuple(weight.shape[:2]) != (H, d):
        raise ValueError(f"weight must be [{H},{d},W] (got {tuple(weight.shape)})")
    _require(weight, "weight", device, torch.float32)
    if out is None:
        out = torch.empty_like(x)
    _require(out, "out", device, x.dtype, tuple(x.shape))
    with torch.cuda.device(device):
        rc = lib.kda_short_conv_swish(_ptr(x), _ptr(weight), _ptr(cu_seqlens), _ptr(out), B, T, H, d,
                                      weight.shape[2], _DTYPES[x.dtype], _stream(device, stream))
    _check(rc)
    return out


def chunk_bwd(q, k, v, log_alpha, beta, grad_out, S0=None, grad_S_T=None, *, workspace=None,
              stream=None):
    """Backward pass of ``chunk_fwd`` (``kda_chunk_bwd``).

    Inputs as ``chunk_fwd``; ``grad_out`` ``[B,T,H,dv]`` in the input dtype and
    ``grad_S_T`` ``[B,H,dk,dv]`` fp32 (or None) are dL/d(out) and dL/d(S_T).
    Returns a dict with ``q``, ``k``, ``v`` (input dtype), ``log_alpha``,
    ``beta`` and ``S0`` (fp32) gradients.
    """
    lib = load()
    device = q.device
    _require(q, "q", device)
    if q.dtype not in _DTYPES:
        raise TypeError(f"q must be bf16 or fp32 (got {q.dtype})")
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    _require(k, "k", device, q.dtype, (B, T, H, dk))
    _require(v, "v", device, q.dtype, (B, T, H, dv))
    _require(log_alpha, "log_alpha", device, torch.float32, (B, T, H, dk))
    _require(beta, "beta", device, torch.float32, (B, T, H))
    _require(grad_out, "grad_out", device, q.dtype, (B, T, H, dv))
    if S0 is not None:
        _require(S0, "S0", device, torch.float32, (B, H, dk, dv))
    if grad_S_T is not None:
        _require(grad_S_T, "grad_S_T", device, torch.float32, (B, H, dk, dv))
    g = dict(q=torch.empty_like(q), k=torch.empty_like(k), v=torch.empty_like(v),
             log_alpha=torch.empty_like(log_alpha), beta=torch.empty_like(beta),
             S0=torch.empty(B, H, dk, dv, device=device, dtype=torch.float32))
    need = int(lib.kda_bwd_workspace_bytes(B, T, H, dk, dv, _DTYPES[q.dtype]))
    if workspace is None and need > 0:
        workspace = torch.empty(need, device=device, dtype=torch.uint8)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    with torch.cuda.device(device):
        rc = lib.kda_chunk_bwd(
            _ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta), _ptr(S0), _ptr(grad_out),
            _ptr(grad_S_T), _ptr(g["q"]), _ptr(g["k"]), _ptr(g["v"]), _ptr(g["log_alpha"]),
            _ptr(g["beta"]), _ptr(g["S0"]), B, T, H, dk, dv, _DTYPES[q.dtype], _ptr(workspace),
            ws_bytes, _stream(device, stream))
    _check(rc)
    return g


def recurrent_step(q, k, v, log_alpha, beta, state, slot=None, *, out=None, stream=None):
    """One decode step (``kda_recurrent_step``); updates ``state`` in place.

    q, k ``[N,H,dk]``, v ``[N,H,dv]`` (bf16 or fp32), log_alpha ``[N,H,dk]`` and
    beta ``[N,H]`` fp32, state ``[slots,H,dk,dv]`` fp32, slot ``[N]`` int32 or
    None. Returns ``out [N,H,dv]``.
    """
    lib = load()
    device = q.device
    _require(q, "q", device)
    if q.dtype not in _DTYPES:
        raise TypeError(f"q must be bf16 or fp32 (got {q.dtype})")
    N, H, dk = q.shape
    dv = v.shape[-1]
    _require(k, "k", device, q.dtype, (N, H, dk))
    _require(v, "v", device, q.dtype, (N, H, dv))
    _require(log_alpha, "log_alpha", device, torch.float32, (N, H, dk))
    _require(beta, "beta", device, torch.float32, (N, H))
    _require(state, "state", device, torch.float32)
    if state.dim() != 4 or tuple(state.shape[1:]) != (H, dk, dv):
        raise ValueError(f"state must be [slots,{H},{dk},{dv}] (got {tuple(state.shape)})")
    if slot is not None:
        _require(slot, "slot", device, torch.int32, (N,))
    elif state.shape[0] < N:
        raise ValueError("state has fewer slots than sequences and no slot map was given")
    if out is None:
        out = torch.empty(N, H, dv, device=device, dtype=q.dtype)
    _require(out, "out", device, q.dtype, (N, H, dv))
    with torch.cuda.device(device):
        rc = lib.kda_recurrent_step(_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta),
                                    _ptr(state), _ptr(slot), _ptr(out), N, H, dk, dv,
                                    _DTYPES[q.dtype], _stream(device, stream))
    _check(rc)
    return out


def test_inject_wait_timeout(on: bool) -> bool:
    """Test hook of the prefill engine's give-up path (``kda_test_inject_wait_timeout``):
    while on, cluster-engine launches run out a bounded device wait on purpose (no
    fault, no trap) and ``device_status`` reports it. Returns the previous setting."""
    return bool(load().kda_test_inject_wait_timeout(1 if on else 0))


def device_status(stream=None, device=None):
    """Synchronise and raise KdaError if a bounded device wait gave up."""
    lib = load()
    device = torch.device("cuda", torch.cuda.current_device()) if device is None else device
    _check(lib.kda_device_status(_stream(device, stream)))
