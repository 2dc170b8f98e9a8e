"""Parity of the CUDA backward pass (kda_chunk_bwd) with the fp64 backward oracle (GPU).

Every gradient (q, k, v, log alpha, beta, S0) is compared element by element
with ``oracle.grad.backward`` on the same seeded inputs and output cotangents.
Tolerances: bf16 inputs use the forward's bf16 bound, |x - ref| <= 2e-3 +
1e-2 |ref| (grad_q, grad_k and grad_v are rounded to bf16 like ``out``); fp32
inputs use the forward's fp32 bound scaled by the gradient's magnitude,
|x - ref| <= 1e-4 * max(1, max |ref|), because gradients are sums over the
whole sequence and grow with it where outputs do not. (This file sorts last so
that the forward's parity tests run first.)
"""
import numpy as np
import pytest
import torch

import kda_inputs as I
from kda_check import assert_close
from oracle import grad

kda = pytest.importorskip("gated_delta_rule_116_b200")

pytestmark = pytest.mark.gpu
DEV = "cuda"
NAMES = ["q", "k", "v", "log_alpha", "beta", "S0"]


def cotangents(B, T, H, dk, dv, dtype, seed, with_dst=True):
    g = torch.Generator().manual_seed(seed)
    dO = torch.randn(B, T, H, dv, generator=g).to(dtype)
    dST = torch.randn(B, H, dk, dv, generator=g) if with_dst else None
    return dO, dST


def check(inp, dO, dST):
    dev = {k: (v.to(DEV) if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    got = kda.chunk_bwd(dev["q"], dev["k"], dev["v"], dev["log_alpha"], dev["beta"], dO.to(DEV),
                        dev["S0"], None if dST is None else dST.to(DEV))
    torch.cuda.synchronize()
    ref = grad.backward(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"], dO,
                        S0=inp["S0"], dS_T=dST)
    for n in NAMES:
        r = ref["d" + n]
        if inp["q"].dtype == torch.float32:
            atol = 1e-4 * max(1.0, float(np.abs(r).max()))
            assert_close(got[n], r, atol, 0.0, f"grad {n}")
        else:
            assert_close(got[n], r, 2e-3, 1e-2, f"grad {n}")


@pytest.mark.parametrize("T", [1, 16, 40, 64])
def test_fp32_small(T):
    inp = I.prefill_inputs("fp32_small", T=T)
    B, _, H, dk = inp["q"].shape
    inp["S0"] = 0.1 * torch.randn(B, H, dk, inp["v"].shape[-1], generator=torch.Generator().manual_seed(5))
    dO, dST = cotangents(B, T, H, dk, inp["v"].shape[-1], torch.float32, seed=T)
    check(inp, dO, dST)


@pytest.mark.parametrize("dk,dv,T,H", [(24, 40, 37, 3), (128, 100, 23, 1), (64, 128, 50, 2)])
def test_fp32_other_sizes_no_state(dk, dv, T, H):
    """Partial value slices (40, 100), ragged lengths, no S0 and no dL/dS_T."""
    inp = I.prefill_inputs("fp32_small", T=T, H=H, dk=dk, dv=dv)
    dO, _ = cotangents(1, T, H, dk, dv, torch.float32, seed=dk + dv, with_dst=False)
    check(inp, dO, None)


def test_bf16_head_size_128():
    inp = I.prefill_inputs("prefill_32k", T=96, H=2)          # slow gates, S0 ~ N(0, 0.01)
    dO, dST = cotangents(1, 96, 2, 128, 128, torch.bfloat16, seed=7)
    check(inp, dO, dST)


def test_bf16_batched_ragged():
    inp = I.prefill_inputs("prefill_4k", B=2, T=45, H=2)
    dO, dST = cotangents(2, 45, 2, 128, 128, torch.bfloat16, seed=8)
    check(inp, dO, dST)


def test_zero_length_copies_the_state_cotangent():
    q = torch.zeros(1, 0, 2, 16, device=DEV)
    la = torch.zeros(1, 0, 2, 16, device=DEV)
    beta = torch.zeros(1, 0, 2, device=DEV)
    dST = torch.randn(1, 2, 16, 16, device=DEV)
    got = kda.chunk_bwd(q, q, q, la, beta, q, None, dST)
    torch.cuda.synchronize()
    assert torch.equal(got["S0"], dST)


def test_autograd_through_the_library():
    """kda_prefill: torch.autograd gradients through chunk_fwd and chunk_bwd on the GPU."""
    x = I.prefill_inputs("fp32_small", T=40)
    x["S0"] = 0.1 * torch.randn(1, 2, 16, 16, generator=torch.Generator().manual_seed(4))
    t = {n: x[n].to(DEV).requires_grad_(True) for n in NAMES}
    out, S_T = kda.kda_prefill(t["q"], t["k"], t["v"], t["log_alpha"], t["beta"], t["S0"], chunk=16)
    g = torch.Generator().manual_seed(5)
    W1, W2 = torch.randn(tuple(out.shape), generator=g), torch.randn(tuple(S_T.shape), generator=g)
    ((out * W1.to(DEV)).sum() + (S_T * W2.to(DEV)).sum()).backward()
    torch.cuda.synchronize()
    ref = grad.backward(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], W1, S0=x["S0"], dS_T=W2)
    for n in NAMES:
        r = ref["d" + n]
        assert_close(t[n].grad, r, 1e-4 * max(1.0, float(np.abs(r).max())), 0.0, f"grad {n}")


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_strong_decay(dtype):
    """Channels with log a = -4, 0, -12 and -1e-3 (the strong-decay gate recipe)."""
    name = "fp32_small" if dtype == torch.float32 else "prefill_4k"
    inp = I.prefill_inputs(name, B=1, T=45, H=2, gate="strong", s0_std=0.1)
    B, T, H, dk = inp["q"].shape
    dO, dST = cotangents(B, T, H, dk, inp["v"].shape[-1], dtype, seed=77)
    check(inp, dO, dST)
