"""B200 (sm_100a) Kimi Delta Attention: chunked prefill, its backward pass and
recurrent decode.

The compute runs in ``libkda.so`` (hand-written CUDA, C ABI in
``include/kda.h``); this package is its thin Python binding.

    out, S_T = chunk_fwd(q, k, v, log_alpha, beta, S0, chunk=64)
    out, S_T = chunk_fwd_varlen(q, k, v, log_alpha, beta, cu_seqlens, S0)   # packed sequences
    grads = chunk_bwd(q, k, v, log_alpha, beta, grad_out, S0, grad_S_T)
    out, S_T = kda_prefill(q, k, v, log_alpha, beta, S0)   # torch.autograd wiring of the two
    out = recurrent_step(q, k, v, log_alpha, beta, state, slot)
"""
from .binding import (ENGINES, KDA_BF16, KDA_F32, LIB_PATH, KdaError, bwd_workspace_bytes, chunk_bwd,
                      chunk_fwd, chunk_fwd_fused, chunk_fwd_varlen, device_status, dplr_chunk_fwd, engine_supported,
                      layer_fwd,
                      load, recurrent_step, short_conv_swish, varlen_workspace_bytes,
                      workspace_bytes)
from .autograd import kda_prefill

__all__ = ["chunk_fwd", "chunk_fwd_fused", "chunk_fwd_varlen", "chunk_bwd", "kda_prefill", "recurrent_step", "workspace_bytes", "bwd_workspace_bytes", "varlen_workspace_bytes", "short_conv_swish", "layer_fwd", "dplr_chunk_fwd", "device_status",
           "engine_supported", "load", "KdaError", "ENGINES", "KDA_BF16", "KDA_F32", "LIB_PATH"]
