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
from kda_check import assert_close, tol_for

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


def check(flat, S0, cu, with_state=True):
    dev = {n: t.to(DEV) for n, t in flat.items()}
    out, ST = kda.chunk_fwd_varlen(dev["q"], dev["k"], dev["v"], dev["log_alpha"], dev["beta"],
                                   cu.to(DEV), None if S0 is None else S0.to(DEV),
                                   output_final_state=with_state)
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
            assert_close(ST[n].cpu(), ref_s[0], atol, rtol, f"S_T of sequence {n}")


def test_fp32_mixed_lengths():
    flat, S0, cu = packed("fp32_small", [0, 1, 17, 64, 5, 33], H=2, seed=1)
    check(flat, S0, cu)


def test_fp32_other_sizes_no_state():
    flat, _, cu = packed("fp32_small", [40, 23], H=3, seed=2, dk=24, dv=40)
    check(flat, None, cu, with_state=False)


def test_bf16_head_size_128():
    flat, S0, cu = packed("prefill_4k", [50, 0, 70], H=2, seed=3)
    check(flat, S0, cu)
