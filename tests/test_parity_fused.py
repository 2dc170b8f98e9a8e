"""Parity of the fused layer prologue (kda_chunk_fwd_fused) with the fp64 layer oracle (GPU).

The kernel reads raw q, k and the gate's pre-activation x and computes
q/||q||, k/||k|| and log alpha = -softplus(x) itself; ``oracle.layer.fused_forward``
does the same in fp64 and runs the recurrence (its pins are in
tests/test_oracle_layer.py). Every element of ``out`` and ``S_T`` within the bf16
bound of the parity tests. Also: the fused call equals the plain call on the
inputs the oracle's prologue produces, to within that bound.
"""
import numpy as np
import pytest
import torch

import kda_inputs as I
from kda_check import BF16_STATE_MAX_ABS, assert_close, tol_for
from oracle import layer

kda = pytest.importorskip("gated_delta_rule_116_b200")
pytestmark = pytest.mark.gpu


def run_fused(inp):
    g = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    out, st = kda.chunk_fwd_fused(g["q"], g["k"], g["v"], g["gate"], g["beta"], g["S0"])
    torch.cuda.synchronize()
    return out, st


def check(inp, heads=None):
    out, st = run_fused(inp)
    atol, rtol = tol_for(torch.bfloat16)
    ref_o, ref_s = layer.fused_forward(inp["q"], inp["k"], inp["v"], inp["gate"], inp["beta"], inp["S0"])
    assert_close(out, ref_o, atol, rtol, "fused out")
    assert_close(st, ref_s, atol, rtol, "fused S_T", max_abs=BF16_STATE_MAX_ABS)


@pytest.mark.parametrize("name,kw", [
    ("prefill_4k", dict(B=2, T=300, H=3)),
    ("prefill_32k", dict(T=700, H=2)),
    ("prefill_128k", dict(T=500, H=2)),
    ("prefill_4k", dict(B=1, T=260, H=2, gate="strong", s0_std=0.05)),
])
def test_fused_prologue_matches_layer_oracle(name, kw):
    check(I.prefill_layer_inputs(name, **kw))


@pytest.mark.parametrize("T", [1, 63, 65, 130])
def test_fused_ragged_lengths(T):
    check(I.prefill_layer_inputs("prefill_32k", T=T, H=2, B=2))


def test_fused_zero_rows_stay_zero():
    """A q or k row of zeros normalises to zeros (no NaN)."""
    inp = I.prefill_layer_inputs("prefill_4k", B=1, T=80, H=2)
    inp["q"][0, 5] = 0
    inp["k"][0, 9] = 0
    check(inp)


def test_fused_rejects_unsupported_shapes():
    inp = I.prefill_layer_inputs("fp32_small", T=8, dtype=torch.bfloat16)
    g = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    with pytest.raises(kda.KdaError, match="UNSUPPORTED"):
        kda.chunk_fwd_fused(g["q"], g["k"], g["v"], g["gate"], g["beta"], chunk=16)
