"""Parity of the general-DPLR comparator kernel (kda_dplr_chunk_fwd) with the fp64
DPLR oracle (GPU), with the forward tolerances of the KDA tests (kda_check): fp32
inputs within 1e-4, bf16 inputs within 2e-3 + 1e-2 |ref|. Also the KDA special case
(a = -beta k, b = alpha * k, write vector beta k) against the KDA oracle."""
import numpy as np
import pytest
import torch

import kda_inputs as I
import oracle
from kda_check import assert_close, state_max_abs, tol_for
from oracle import dplr

kda = pytest.importorskip("gated_delta_rule_116_b200")
pytestmark = pytest.mark.gpu
DEV = "cuda"


def run(inp, chunk, a=None, b=None, k=None):
    g = {n: (t.to(DEV) if isinstance(t, torch.Tensor) else t) for n, t in inp.items()}
    a = g["a"] if a is None else a.to(DEV)
    b = g["b"] if b is None else b.to(DEV)
    k = g["k"] if k is None else k.to(DEV)
    out, st = kda.dplr_chunk_fwd(g["q"], k, g["v"], a, b, g["log_alpha"], g["S0"], chunk)
    torch.cuda.synchronize()
    return out, st


@pytest.mark.parametrize("chunk", [16, 32])
@pytest.mark.parametrize("name,kw", [
    ("fp32_small", dict(T=77, s0_std=0.3)),
    ("prefill_4k", dict(B=2, T=150, H=2, s0_std=0.05)),
    ("prefill_4k", dict(B=1, T=70, H=2, gate="strong")),
])
def test_dplr_matches_oracle(name, kw, chunk):
    inp = I.dplr_inputs(name, **kw)
    out, st = run(inp, chunk)
    ref_o, ref_s = dplr.forward(inp["q"], inp["k"], inp["v"], inp["a"], inp["b"], inp["log_alpha"], inp["S0"])
    atol, rtol = tol_for(inp["q"].dtype)
    assert_close(out, ref_o, atol, rtol, f"dplr out {name} C={chunk}")
    assert_close(st, ref_s, atol, rtol, f"dplr S_T {name} C={chunk}", max_abs=state_max_abs(inp["q"].dtype))


def test_dplr_kernel_reproduces_kda():
    inp = I.prefill_inputs("fp32_small", B=1, T=90, H=2, s0_std=0.2)
    a, b, wk = (torch.from_numpy(x).float() for x in dplr.kda_as_dplr(inp["k"], inp["log_alpha"], inp["beta"]))
    out, st = run(dict(inp, a=a, b=b), 32, k=wk)
    ref_o, ref_s = oracle.forward(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"], inp["S0"])
    assert_close(out, ref_o, 1e-4, 0.0, "dplr as kda out")
    assert_close(st, ref_s, 1e-4, 0.0, "dplr as kda S_T")


def test_dplr_rejects_chunk_64_at_d128():
    inp = I.dplr_inputs("prefill_4k", B=1, T=64, H=1)
    with pytest.raises(kda.KdaError):
        run(inp, 64)
