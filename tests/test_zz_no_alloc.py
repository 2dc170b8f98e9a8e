"""kda_chunk_fwd_static: prefill without any device allocation by the library.

Some callers cannot let a library allocate device memory when they call it: a
serving process whose pool allocator has already claimed the free memory, or a
plug-in inside a framework that owns every allocation. For them the library
keeps the prefill engine's scratch in a fixed device array (a pool of 40
operand rings, claimed per cluster) and kda_chunk_fwd_static takes only inputs
and outputs.

The GPU test calls it twice in a row through the C ABI, on different problems
queued back to back on one stream: the first has more heads (66) than the pool
has rings, so clusters wait for and reuse rings; the second reuses the array
the first left behind. Both calls run the same deterministic kernel as kda_chunk_fwd
with a workspace, so their results must be bit-for-bit equal to that call's;
the second problem is also compared with the fp64 oracle within the bf16
tolerance of the parity tests, and no bounded device wait may have given up.
The file is named to be collected last, so a run that stops at its first
failure has run every other test before it.
"""
import ctypes

import pytest
import torch

import kda_inputs as I
import oracle
from kda_check import BF16_ATOL, BF16_RTOL, BF16_STATE_MAX_ABS, assert_close
from gated_delta_rule_116_b200 import binding

KDA_BF16 = 0
POOL_RINGS = 40


def lib():
    from gated_delta_rule_116_b200 import build as kbuild
    kbuild.build()
    lib = ctypes.CDLL(binding.LIB_PATH)
    p, i, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
    lib.kda_chunk_fwd_static.argtypes = [p, p, p, p, p, p, p, p, i, i, i, i, i, i, i, p]
    lib.kda_chunk_fwd_static.restype = i
    lib.kda_chunk_fwd.argtypes = [p, p, p, p, p, p, p, p, i, i, i, i, i, i, i, p, sz, p]
    lib.kda_chunk_fwd.restype = i
    lib.kda_workspace_bytes.argtypes = [i, i, i, i, i, i, i]
    lib.kda_workspace_bytes.restype = sz
    lib.kda_last_error_detail.restype = ctypes.c_char_p
    lib.kda_device_status.argtypes = [p]
    lib.kda_device_status.restype = i
    return lib


def ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def problem(seed, B, T, H, with_state):
    inp = I.prefill_inputs("prefill_4k", "cuda", B=B, T=T, H=H, seed=seed,
                           s0_std=0.05 if with_state else 0.0, gate="mixed")
    q, k, v, S0 = inp["q"], inp["k"], inp["v"], inp["S0"]
    assert (S0 is not None) == with_state
    out = torch.full((B, T, H, 128), float("nan"), device="cuda", dtype=torch.bfloat16)
    S_T = torch.full((B, H, 128, 128), float("nan"), device="cuda")
    return dict(q=q, k=k, v=v, la=inp["log_alpha"], beta=inp["beta"], S0=S0, out=out, S_T=S_T,
                B=B, T=T, H=H)


def call_static(L, pb, stream):
    return L.kda_chunk_fwd_static(ptr(pb["q"]), ptr(pb["k"]), ptr(pb["v"]), ptr(pb["la"]),
                                  ptr(pb["beta"]), ptr(pb["S0"]), ptr(pb["out"]), ptr(pb["S_T"]),
                                  pb["B"], pb["T"], pb["H"], 128, 128, 64, KDA_BF16,
                                  ctypes.c_void_p(stream.cuda_stream))


def call_with_workspace(L, pb, stream):
    B, T, H = pb["B"], pb["T"], pb["H"]
    out = torch.empty_like(pb["out"])
    S_T = torch.empty_like(pb["S_T"])
    need = int(L.kda_workspace_bytes(B, T, H, 128, 128, 64, KDA_BF16))
    ws = torch.empty(max(need, 1), device="cuda", dtype=torch.uint8)
    rc = L.kda_chunk_fwd(ptr(pb["q"]), ptr(pb["k"]), ptr(pb["v"]), ptr(pb["la"]), ptr(pb["beta"]),
                         ptr(pb["S0"]), ptr(out), ptr(S_T), B, T, H, 128, 128, 64, KDA_BF16,
                         ptr(ws), need, ctypes.c_void_p(stream.cuda_stream))
    assert rc == 0, L.kda_last_error_detail().decode()
    return out, S_T


def test_static_rejects_unsupported_shapes():
    """Host-side checks, no device call."""
    L = lib()
    fake = ctypes.c_void_p(0x10000)
    rc = L.kda_chunk_fwd_static(fake, fake, fake, fake, fake, None, fake, None,
                                 1, 64, 2, 64, 128, 64, KDA_BF16, None)
    assert rc == -2  # KDA_ERR_UNSUPPORTED: dk = 64
    # more tokens than 32-bit token rows address (B*T = 2^31 + 2), within the head limit
    rc = L.kda_chunk_fwd_static(fake, fake, fake, fake, fake, None, fake, None,
                                 2, 2**30 + 1, 2, 128, 128, 64, KDA_BF16, None)
    assert rc == -2
    assert "2^31" in L.kda_last_error_detail().decode()


@pytest.mark.gpu
def test_static_matches_workspace_entry_point_on_two_calls_in_a_row():
    L = lib()
    stream = torch.cuda.current_stream()
    # first: more heads than the pool has rings, a ragged last chunk, an initial state
    first = problem(seed=11, B=3, T=700, H=22, with_state=True)
    # second: fewer heads, a shorter sequence, no initial state
    second = problem(seed=12, B=1, T=130, H=5, with_state=False)
    assert first["B"] * first["H"] > POOL_RINGS
    for pb in (first, second):
        rc = call_static(L, pb, stream)
        assert rc == 0, L.kda_last_error_detail().decode()
    torch.cuda.synchronize()
    assert L.kda_device_status(ctypes.c_void_p(stream.cuda_stream)) == 0, "a device wait gave up"
    for name, pb in (("first", first), ("second", second)):
        ref_out, ref_st = call_with_workspace(L, pb, stream)
        torch.cuda.synchronize()
        assert torch.equal(pb["out"], ref_out), f"{name} out differs from kda_chunk_fwd"
        assert torch.equal(pb["S_T"], ref_st), f"{name} S_T differs from kda_chunk_fwd"
    # the second problem (it ran on the array the first one left behind) against the oracle
    cpu = {k: (v.cpu() if isinstance(v, torch.Tensor) else v) for k, v in second.items()}
    o_ref, s_ref = oracle.forward(cpu["q"], cpu["k"], cpu["v"], cpu["la"], cpu["beta"], None)
    assert_close(second["out"], o_ref, BF16_ATOL, BF16_RTOL, "second out vs oracle")
    assert_close(second["S_T"], s_ref, BF16_ATOL, BF16_RTOL, "second S_T vs oracle", max_abs=BF16_STATE_MAX_ABS)
