"""Parity of the variable-length prefill (kda_chunk_fwd_varlen) with the oracle (GPU).

Packed sequences of different lengths (empty and one-token ones included),
each compared element by element with the oracle run on that sequence alone
from its own initial state, within the forward's tolerances (kda_check).
(This file sorts after every other GPU test.)
"""
import numpy as np
import pytest
import torch

import kda_inputs as I
import oracle
from kda_check import assert_close, state_max_abs, tol_for

kda = pytest.importorskip("gated_delta_rule_116_b200")

pytestmark = pytest.mark.gpu
DEV = "cuda"


def packed(name, lens, H, seed, **kw):
    """One synthetic sequence of sum(lens) tokens (the workload's recipe), cut into pieces."""
    x = I.prefill_inputs(name, B=1, T=int(sum(lens)), H=H, **kw)
    flat = {n: x[n][0] for n in ("q", "k", "v", "log_alpha", "beta")}
    g = torch.Generator().manual_seed(seed)
    S0 = 0.1 * torch.randn(len(lens), H, x["q"].shape[-1], x["v"].shape[-1], generator=g)
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lens)]), dtype=torch.int32)
    return flat, S0, cu


def check(flat, S0, cu, with_state=True, engine="auto"):
    dev = {n: t.to(DEV) for n, t in flat.items()}
    out, ST = kda.chunk_fwd_varlen(dev["q"], dev["k"], dev["v"], dev["log_alpha"], dev["beta"],
                                   cu.to(DEV), None if S0 is None else S0.to(DEV),
                                   output_final_state=with_state, engine=engine)
    torch.cuda.synchronize()
    out = out.cpu()
    atol, rtol = tol_for(flat["q"].dtype)
    for n in range(cu.numel() - 1):
        a, b = int(cu[n]), int(cu[n + 1])
        s0 = None if S0 is None else S0[n][None]
        ref_o, ref_s = oracle.forward(flat["q"][None, a:b], flat["k"][None, a:b], flat["v"][None, a:b],
                                      flat["log_alpha"][None, a:b], flat["beta"][None, a:b], s0)
        assert_close(out[a:b], ref_o[0], atol, rtol, f"out of sequence {n}")
        if with_state:
            assert_close(ST[n].cpu(), ref_s[0], atol, rtol, f"S_T of sequence {n}",
                         max_abs=state_max_abs(flat["q"].dtype))


def test_fp32_mixed_lengths():
    flat, S0, cu = packed("fp32_small", [0, 1, 17, 64, 5, 33], H=2, seed=1)
    check(flat, S0, cu)


def test_fp32_other_sizes_no_state():
    flat, _, cu = packed("fp32_small", [40, 23], H=3, seed=2, dk=24, dv=40)
    check(flat, None, cu, with_state=False)


BF16_ENGINES = ["generic", "tc_cluster"]


@pytest.mark.parametrize("engine", BF16_ENGINES)
def test_bf16_head_size_128(engine):
    flat, S0, cu = packed("prefill_4k", [50, 0, 70], H=2, seed=3)
    check(flat, S0, cu, engine=engine)


@pytest.mark.parametrize("lens", [[0, 1, 63, 64, 65, 200, 129], [300], [5, 0, 0, 190, 64 * 5 + 7]])
def test_bf16_tensor_core_engine_lengths(lens):
    """The tensor-core engine over packed sequences: empty and one-token sequences,
    lengths at and around the 64-token chunk, several chunks and a ragged tail."""
    flat, S0, cu = packed("prefill_4k", lens, H=3, seed=4)
    check(flat, S0, cu, engine="tc_cluster")
    check(flat, None, cu, with_state=False, engine="tc_cluster")


def test_paged_prefill_then_decode():
    """Prefill packed sequences into rows of a state cache (slot map, in place), then
    one decode step from the same rows: the serving handoff. Each sequence's
    outputs, its decode output and its cache row equal the oracle run on that
    sequence plus its next token; rows outside the map are untouched."""
    lens, slots, H = [20, 0, 37], [3, 0, 4], 2
    flat, _, cu = packed("fp32_small", lens, H=H, seed=6)
    g = torch.Generator().manual_seed(7)
    cache0 = 0.1 * torch.randn(5, H, 16, 16, generator=g)
    nxt = I.prefill_inputs("fp32_small", B=1, T=len(lens), H=H, seed=9)   # one new token per sequence
    step = {n: nxt[n][0].contiguous() for n in ("q", "k", "v", "log_alpha", "beta")}
    cache = cache0.to(DEV)
    slot = torch.tensor(slots, dtype=torch.int32, device=DEV)
    dev = {n: t.to(DEV) for n, t in flat.items()}
    out, ST = kda.chunk_fwd_varlen(dev["q"], dev["k"], dev["v"], dev["log_alpha"], dev["beta"],
                                   cu.to(DEV), cache, slot=slot)
    assert ST.data_ptr() == cache.data_ptr()
    o1 = kda.recurrent_step(*(step[n].to(DEV) for n in ("q", "k", "v", "log_alpha", "beta")), cache, slot)
    torch.cuda.synchronize()
    out, o1, cache = out.cpu(), o1.cpu(), cache.cpu()
    atol, rtol = tol_for(torch.float32)
    for n, r in enumerate(slots):
        a, b = int(cu[n]), int(cu[n + 1])
        cat = lambda name: torch.cat([flat[name][a:b], step[name][n:n + 1]])[None]
        ref_o, ref_s = oracle.forward(cat("q"), cat("k"), cat("v"), cat("log_alpha"), cat("beta"), cache0[r][None])
        assert_close(out[a:b], ref_o[0, :-1], atol, rtol, f"prefill out of sequence {n}")
        assert_close(o1[n], ref_o[0, -1], atol, rtol, f"decode out of sequence {n}")
        assert_close(cache[r], ref_s[0], atol, rtol, f"cache row {r}", max_abs=state_max_abs(flat["q"].dtype))
    for r in (1, 2):
        assert torch.equal(cache[r], cache0[r])


@pytest.mark.parametrize("engine", BF16_ENGINES)
def test_bf16_strong_decay_mixed_lengths(engine):
    flat, S0, cu = packed("prefill_4k", [70, 1, 33, 130], H=2, seed=9, gate="strong")
    check(flat, S0, cu, engine=engine)


def test_bf16_tensor_core_paged_prefill_then_decode():
    """The serving handoff on the tensor-core engine: bf16 prompts prefilled into rows
    of a state cache through a slot map (in place), then one decode step from the same
    rows; rows outside the map are untouched."""
    lens, slots, H = [130, 0, 64, 7], [5, 1, 0, 3], 2
    flat, _, cu = packed("prefill_4k", lens, H=H, seed=10)
    g = torch.Generator().manual_seed(11)
    cache0 = 0.05 * torch.randn(7, H, 128, 128, generator=g)
    nxt = I.prefill_inputs("prefill_4k", B=1, T=len(lens), H=H, seed=12)
    step = {n: nxt[n][0].contiguous() for n in ("q", "k", "v", "log_alpha", "beta")}
    cache = cache0.to(DEV)
    slot = torch.tensor(slots, dtype=torch.int32, device=DEV)
    dev = {n: t.to(DEV) for n, t in flat.items()}
    out, ST = kda.chunk_fwd_varlen(dev["q"], dev["k"], dev["v"], dev["log_alpha"], dev["beta"],
                                   cu.to(DEV), cache, slot=slot, engine="tc_cluster")
    assert ST.data_ptr() == cache.data_ptr()
    kda.device_status()
    o1 = kda.recurrent_step(*(step[n].to(DEV) for n in ("q", "k", "v", "log_alpha", "beta")), cache, slot)
    torch.cuda.synchronize()
    out, o1, cache = out.cpu(), o1.cpu(), cache.cpu()
    atol, rtol = tol_for(torch.bfloat16)
    for n, r in enumerate(slots):
        a, b = int(cu[n]), int(cu[n + 1])
        cat = lambda name: torch.cat([flat[name][a:b], step[name][n:n + 1]])[None]
        ref_o, ref_s = oracle.forward(cat("q"), cat("k"), cat("v"), cat("log_alpha"), cat("beta"), cache0[r][None])
        assert_close(out[a:b], ref_o[0, :-1], atol, rtol, f"prefill out of sequence {n}")
        assert_close(o1[n], ref_o[0, -1], atol, rtol, f"decode out of sequence {n}")
        assert_close(cache[r], ref_s[0], atol, rtol, f"cache row {r}", max_abs=state_max_abs(flat["q"].dtype))
    for r in (2, 4, 6):
        assert torch.equal(cache[r], cache0[r])


def test_engine_choice_errors():
    flat, S0, cu = packed("fp32_small", [10, 20], H=2, seed=13)
    dev = {n: t.to(DEV) for n, t in flat.items()}
    with pytest.raises(kda.KdaError):   # fp32, d = 16: not the tensor-core engine's shape
        kda.chunk_fwd_varlen(dev["q"], dev["k"], dev["v"], dev["log_alpha"], dev["beta"], cu.to(DEV),
                             S0.to(DEV), engine="tc_cluster")
