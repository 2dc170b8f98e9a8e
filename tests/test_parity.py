"""Parity of the CUDA library with the fp64 oracle (GPU).

Every test runs the CUDA path through the C ABI (via the thin binding) and
compares ``out`` and ``S_T`` element by element with the oracle on the same
seeded inputs, within the tolerances of ``kda_check``. Small cases compare
every element; full-size workloads compare every element of a sample of
heads (heads are independent, so the oracle computes just those).
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


def engines(dtype, dk, dv, chunk):
    return [e for e in ("generic", "tc_cluster") if kda.engine_supported(e, dk, dv, chunk, dtype)]


def run_gpu(inp, chunk, engine="auto", with_state=True):
    g = {k: (v.to(DEV) if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    out, st = kda.chunk_fwd(g["q"], g["k"], g["v"], g["log_alpha"], g["beta"], g["S0"],
                            chunk=chunk, engine=engine, output_final_state=with_state)
    torch.cuda.synchronize()
    return out, st


def run_oracle(inp, heads=None):
    return oracle.forward(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"], inp["S0"],
                          heads=heads)


def compare(inp, out, st, ref_out, ref_st, heads=None):
    atol, rtol = tol_for(inp["q"].dtype)
    ma = state_max_abs(inp["q"].dtype)
    H = inp["q"].shape[2]
    if heads is None:
        assert_close(out, ref_out, atol, rtol, "out")
        if st is not None:
            assert_close(st, ref_st, atol, rtol, "S_T", max_abs=ma)
        return
    out_c = out.float().cpu()
    st_c = None if st is None else st.cpu()
    for bh in heads:
        b, h = divmod(int(bh), H)
        assert_close(out_c[b, :, h], ref_out[b, :, h], atol, rtol, f"out[b={b},h={h}]")
        if st_c is not None:
            assert_close(st_c[b, h], ref_st[b, h], atol, rtol, f"S_T[b={b},h={h}]", max_abs=ma)


# --- fp32 ----------------------------------------------------------------------

@pytest.mark.parametrize("chunk", [16, 32, 64])
def test_fp32_small_workload(chunk):
    inp = I.prefill_inputs("fp32_small")
    ref = run_oracle(inp)
    for eng in engines(torch.float32, 16, 16, chunk):
        out, st = run_gpu(inp, chunk, eng)
        compare(inp, out, st, *ref)


@pytest.mark.parametrize("dk,dv,T", [(64, 32, 100), (128, 128, 70), (8, 4, 33), (3, 12, 5)])
def test_fp32_other_head_sizes(dk, dv, T):
    inp = I.prefill_inputs("fp32_small", dk=dk, dv=dv, T=T, B=2, s0_std=0.5)
    ref = run_oracle(inp)
    out, st = run_gpu(inp, 16)
    compare(inp, out, st, *ref)


def test_fp32_initial_state_in_place():
    inp = I.prefill_inputs("fp32_small", s0_std=1.0, T=50)
    ref = run_oracle(inp)
    g = {k: (v.to(DEV) if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    state = g["S0"].clone()
    out, st = kda.chunk_fwd(g["q"], g["k"], g["v"], g["log_alpha"], g["beta"], state, chunk=16,
                            S_T=state)
    torch.cuda.synchronize()
    assert st.data_ptr() == state.data_ptr()
    compare(inp, out, st, *ref)


# --- bf16, reduced sizes with full comparison -------------------------------------

SHRUNK = [
    ("prefill_4k", dict(B=2, T=300)),
    ("prefill_32k", dict(T=1000, H=4)),
    ("prefill_128k", dict(T=700, H=3)),
]


@pytest.mark.parametrize("name,kw", SHRUNK)
def test_bf16_reduced_workloads(name, kw):
    inp = I.prefill_inputs(name, **kw)
    ref = run_oracle(inp)
    for eng in engines(torch.bfloat16, 128, 128, 64):
        out, st = run_gpu(inp, 64, eng)
        compare(inp, out, st, *ref)


@pytest.mark.parametrize("T", [1, 17, 63, 64, 65, 129])
def test_bf16_ragged_lengths(T):
    inp = I.prefill_inputs("prefill_32k", T=T, H=2, B=2)
    ref = run_oracle(inp)
    for eng in engines(torch.bfloat16, 128, 128, 64):
        out, st = run_gpu(inp, 64, eng)
        compare(inp, out, st, *ref)


@pytest.mark.parametrize("chunk", [16, 32, 64])
def test_bf16_chunk_size_invariance(chunk):
    inp = I.prefill_inputs("prefill_4k", B=1, H=2, T=200)
    ref = run_oracle(inp)
    for eng in engines(torch.bfloat16, 128, 128, chunk):
        out, st = run_gpu(inp, chunk, eng)
        compare(inp, out, st, *ref)


def test_bf16_initial_state_in_place():
    """S_T may alias S0: each engine reads a head's initial state before writing its final one."""
    inp = I.prefill_inputs("prefill_32k", T=150, H=3, B=2)
    ref_out, ref_st = run_oracle(inp)
    for eng in engines(torch.bfloat16, 128, 128, 64):
        g = {k: (v.to(DEV) if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
        state = g["S0"].clone()
        out, st = kda.chunk_fwd(g["q"], g["k"], g["v"], g["log_alpha"], g["beta"], state,
                                chunk=64, engine=eng, S_T=state)
        torch.cuda.synchronize()
        assert st.data_ptr() == state.data_ptr()
        compare(inp, out, st, ref_out, ref_st)


# --- strong decay (the fine-grained decay inside a chunk that the pages single out) --------

@pytest.mark.parametrize("B,T,H", [(2, 300, 3), (1, 64, 2), (1, 1000, 4)])
def test_bf16_strong_decay_all_engines(B, T, H):
    """Channels with log a = -4 (a chunk decays by e^-256), 0, -12 and -1e-3 next to
    softplus gates, with an initial state: beyond any chunk-wide anchor's range."""
    inp = I.prefill_inputs("prefill_4k", B=B, T=T, H=H, gate="strong", s0_std=0.05)
    ref = run_oracle(inp)
    for eng in engines(torch.bfloat16, 128, 128, 64):
        out, st = run_gpu(inp, 64, eng)
        compare(inp, out, st, *ref)


@pytest.mark.parametrize("chunk", [16, 32, 64])
def test_bf16_strong_decay_chunk_sizes(chunk):
    inp = I.prefill_inputs("prefill_4k", B=1, T=200, H=2, gate="strong", s0_std=0.05)
    ref = run_oracle(inp)
    for eng in engines(torch.bfloat16, 128, 128, chunk):
        out, st = run_gpu(inp, chunk, eng)
        compare(inp, out, st, *ref)


@pytest.mark.parametrize("chunk", [16, 32, 64])
def test_fp32_strong_decay(chunk):
    inp = I.prefill_inputs("fp32_small", gate="strong", s0_std=0.5, T=100)
    ref = run_oracle(inp)
    out, st = run_gpu(inp, chunk)
    compare(inp, out, st, *ref)


@pytest.mark.parametrize("T", [64 * 7 + 5, 64 * 12])
def test_bf16_decay_changes_from_chunk_to_chunk(T):
    """The gate's range changes from one 64-token chunk to the next, so that an engine
    that picks its factorisation per chunk switches inside one head: softplus gates;
    log a = -2.49 on every channel (a 16-token sub-chunk decays by e^-39.8 and the chunk by
    e^-159); the strong recipe; log a = -2.6 on every other channel (sub-chunks just past
    e^-40); uniform -30."""
    inp = I.prefill_inputs("prefill_4k", B=2, T=T, H=3, s0_std=0.05)
    strong = I.prefill_inputs("prefill_4k", B=2, T=T, H=3, gate="strong")["log_alpha"]
    la = inp["log_alpha"]
    for c in range((T + 63) // 64):
        sl = slice(64 * c, 64 * (c + 1))
        kind = c % 5
        if kind == 1:
            la[:, sl] = -2.49
        elif kind == 2:
            la[:, sl] = strong[:, sl]
        elif kind == 3:
            la[:, sl, :, 0::2] = -2.6
        elif kind == 4:
            la[:, sl] = -30.0
    ref = run_oracle(inp)
    for eng in engines(torch.bfloat16, 128, 128, 64):
        out, st = run_gpu(inp, 64, eng)
        compare(inp, out, st, *ref)


def test_bf16_uniform_extreme_decay():
    """Every channel at log a = -30 (a ~ 1e-13): the state keeps only the last token."""
    inp = I.prefill_inputs("prefill_4k", B=1, T=150, H=2, s0_std=0.05)
    inp["log_alpha"] = torch.full_like(inp["log_alpha"], -30.0)
    ref = run_oracle(inp)
    for eng in engines(torch.bfloat16, 128, 128, 64):
        out, st = run_gpu(inp, 64, eng)
        compare(inp, out, st, *ref)


def test_zero_length_copies_state():
    inp = I.prefill_inputs("fp32_small", T=0, s0_std=1.0)
    out, st = run_gpu(inp, 16)
    assert out.shape[1] == 0
    torch.testing.assert_close(st.cpu(), inp["S0"], rtol=0, atol=0)
    inp = I.prefill_inputs("fp32_small", T=0)
    out, st = run_gpu(inp, 16)
    assert (st == 0).all()


def test_no_final_state_requested():
    inp = I.prefill_inputs("prefill_4k", B=1, H=2, T=80)
    ref_out, _ = run_oracle(inp)
    out, st = run_gpu(inp, 64, with_state=False)
    assert st is None
    assert_close(out, ref_out, *tol_for(torch.bfloat16), "out")


def test_split_run_on_gpu():
    """Two calls chained through S_T -> S0 equal one call (chunk-boundary resume)."""
    inp = I.prefill_inputs("prefill_32k", T=300, H=2)
    ref_out, ref_st = run_oracle(inp)
    a = {k: (v[:, :128] if k in ("q", "k", "v", "log_alpha", "beta") else v) for k, v in inp.items()}
    b = {k: (v[:, 128:].contiguous() if k in ("q", "k", "v", "log_alpha", "beta") else v)
         for k, v in inp.items()}
    o1, s1 = run_gpu(a, 64)
    b["S0"] = s1.cpu()
    o2, s2 = run_gpu(b, 64)
    compare(inp, torch.cat([o1, o2], dim=1), s2, ref_out, ref_st)


def test_misaligned_pointer_is_rejected():
    inp = I.prefill_inputs("prefill_4k", B=1, H=1, T=8)
    g = {k: (v.to(DEV) if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    flat = torch.empty(g["q"].numel() + 1, device=DEV, dtype=torch.bfloat16)
    q_bad = flat[1:].view_as(g["q"])
    with pytest.raises(kda.KdaError, match="KDA_ERR_ALIGNMENT"):
        kda.chunk_fwd(q_bad, g["k"], g["v"], g["log_alpha"], g["beta"], chunk=64)


def test_unsupported_engine_shape_is_rejected():
    inp = I.prefill_inputs("fp32_small", T=8)
    g = {k: (v.to(DEV) if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    with pytest.raises(kda.KdaError, match="UNSUPPORTED"):
        kda.chunk_fwd(g["q"], g["k"], g["v"], g["log_alpha"], g["beta"], chunk=16, engine="tc_cluster")


# --- full-size workloads, sampled heads -----------------------------------------

FULL = [
    ("prefill_4k", [0, 37, 130, 255], {}),
    ("prefill_32k", [0, 7, 19, 31], {}),
    ("prefill_128k", [0, 15], {}),
    ("prefill_32k", [3, 30], {"gate": "strong"}),
]


@pytest.mark.parametrize("name,heads,kw", FULL)
def test_full_workload_sampled_heads(name, heads, kw):
    inp = I.prefill_inputs(name, device=DEV, **kw)
    out, st = kda.chunk_fwd(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"],
                            inp["S0"], chunk=inp["w"].chunk)
    torch.cuda.synchronize()
    assert torch.isfinite(out).all() and torch.isfinite(st).all()
    cpu = {k: (v.cpu() if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    ref_out, ref_st = run_oracle(cpu, heads=heads)
    compare(cpu, out, st, ref_out, ref_st, heads=heads)


# --- decode --------------------------------------------------------------------

def test_fp32_decode_token_by_token_matches_oracle():
    """The fp32 small workload fed one token at a time through the decode step."""
    inp = I.prefill_inputs("fp32_small", s0_std=0.3)
    B, T, H, dk = inp["q"].shape
    dv = inp["v"].shape[-1]
    ref_out, ref_st = run_oracle(inp)
    state = inp["S0"].to(DEV).clone()
    outs = []
    for t in range(T):
        sl = {k: inp[k][:, t].contiguous().to(DEV) for k in ("q", "k", "v", "log_alpha", "beta")}
        outs.append(kda.recurrent_step(sl["q"], sl["k"], sl["v"], sl["log_alpha"], sl["beta"],
                                       state).cpu())
    torch.cuda.synchronize()
    assert_close(torch.stack(outs, dim=1), ref_out, 1e-4, 0, "decode out")
    assert_close(state, ref_st, 1e-4, 0, "decode state")


def test_decode_equals_prefill_on_gpu():
    inp = I.prefill_inputs("prefill_32k", T=40, H=2, B=3)
    out_p, st_p = run_gpu(inp, 64)
    state = inp["S0"].to(DEV).clone()
    outs = []
    for t in range(inp["q"].shape[1]):
        sl = {k: inp[k][:, t].contiguous().to(DEV) for k in ("q", "k", "v", "log_alpha", "beta")}
        outs.append(kda.recurrent_step(sl["q"], sl["k"], sl["v"], sl["log_alpha"], sl["beta"], state))
    out_d = torch.stack(outs, dim=1)
    torch.cuda.synchronize()
    atol, rtol = tol_for(torch.bfloat16)
    assert_close(out_d, out_p.float(), 2 * atol, 2 * rtol, "decode vs prefill out")
    assert_close(state, st_p, 2 * atol, 2 * rtol, "decode vs prefill state")


def test_decode_slot_map_and_other_sizes():
    w = I.WORKLOADS["decode_256"]
    for dk, dv in [(128, 128), (64, 32), (16, 16)]:
        state = I.decode_state(w, N=9, H=3, dk=dk, dv=dv)
        inp = I.decode_step_inputs(w, 0, N=6, H=3, dk=dk, dv=dv)
        slot = torch.tensor([8, 0, 3, 5, 1, 7], dtype=torch.int32)
        ref_out, ref_new = oracle.decode_step(inp["q"], inp["k"], inp["v"], inp["log_alpha"],
                                              inp["beta"], state, slot=slot)
        st = state.to(DEV)
        g = {k: v.to(DEV) for k, v in inp.items()}
        out = kda.recurrent_step(g["q"], g["k"], g["v"], g["log_alpha"], g["beta"], st,
                                 slot.to(DEV))
        torch.cuda.synchronize()
        atol, rtol = tol_for(torch.bfloat16)
        assert_close(out, ref_out, atol, rtol, "decode out")
        assert_close(st.cpu()[slot.long()], ref_new, atol, rtol, "decode state")
        untouched = [i for i in range(9) if i not in set(slot.tolist())]
        torch.testing.assert_close(st.cpu()[untouched], state[untouched], rtol=0, atol=0)


def test_decode_workload_first_steps_all_heads():
    """Full 256 x 32 state cache: the first 4 steps, every head compared."""
    w = I.WORKLOADS["decode_256"]
    state0 = I.decode_state(w, device=DEV)
    ref_state = state0.cpu()
    st = state0.clone()
    atol, rtol = tol_for(torch.bfloat16)
    for step in range(4):
        inp = I.decode_step_inputs(w, step, device=DEV)
        out = kda.recurrent_step(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"], st)
        cpu = {k: v.cpu() for k, v in inp.items()}
        ref_out, ref_new = oracle.decode_step(cpu["q"], cpu["k"], cpu["v"], cpu["log_alpha"],
                                              cpu["beta"], ref_state)
        assert_close(out, ref_out, atol, rtol, f"step {step} out")
        ref_state = torch.from_numpy(ref_new).float()
        assert_close(st, ref_new, atol, rtol, f"step {step} state")


def test_decode_workload_1000_steps_sampled_sequences():
    """All 1000 steps of the decode workload; sequences 0-7 (all heads) compared at every step."""
    w = I.WORKLOADS["decode_256"]
    rows = np.arange(8)
    st = I.decode_state(w, device=DEV)
    ref_state = st[: len(rows)].cpu().double().numpy()
    atol, rtol = tol_for(torch.bfloat16)
    for step in range(w.steps):
        inp = I.decode_step_inputs(w, step, device=DEV)
        out = kda.recurrent_step(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"], st)
        sub = {k: v[: len(rows)].cpu() for k, v in inp.items()}
        ref_out, ref_state = oracle.decode_step(sub["q"], sub["k"], sub["v"], sub["log_alpha"],
                                                sub["beta"], ref_state)
        assert_close(out[: len(rows)], ref_out, atol, rtol, f"step {step} out")
    assert_close(st[: len(rows)], ref_state, atol, rtol, "final state")
