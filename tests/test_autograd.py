"""The torch.autograd wiring (gated_delta_rule_116_b200/autograd.py), on CPU.

The two library calls are replaced, for this test only, by stand-ins built on
the fp64 oracle (forward: oracle.forward, backward: oracle.grad.backward), so
that the test checks the wiring itself on CPU: which gradient reaches which
input, how an unused output or a missing S0 is handled, and that
torch.autograd's gradients equal the oracle's. The library path itself is
covered by the GPU tests.
"""
import numpy as np
import pytest
import torch

import kda_inputs as I
import oracle
from oracle import grad

kda = pytest.importorskip("gated_delta_rule_116_b200")
from gated_delta_rule_116_b200 import autograd as kag  # noqa: E402


@pytest.fixture
def oracle_backed(monkeypatch):
    def fwd(q, k, v, log_alpha, beta, S0=None, chunk=64, **_):
        o, s = oracle.forward(q.detach(), k.detach(), v.detach(), log_alpha.detach(), beta.detach(),
                              None if S0 is None else S0.detach())
        return torch.from_numpy(o).to(q.dtype), torch.from_numpy(s).float()

    def bwd(q, k, v, log_alpha, beta, grad_out, S0=None, grad_S_T=None, **_):
        g = grad.backward(q, k, v, log_alpha, beta, grad_out, S0=S0, dS_T=grad_S_T)
        t = lambda a, like: torch.from_numpy(a).to(like.dtype)
        S0_like = torch.zeros((), dtype=torch.float32)
        return dict(q=t(g["dq"], q), k=t(g["dk"], k), v=t(g["dv"], v), log_alpha=t(g["dlog_alpha"], log_alpha),
                    beta=t(g["dbeta"], beta), S0=t(g["dS0"], S0_like))

    monkeypatch.setattr(kag.binding, "chunk_fwd", fwd)
    monkeypatch.setattr(kag.binding, "chunk_bwd", bwd)


def leaves(x, names):
    return {n: x[n].clone().requires_grad_(True) for n in names}


@pytest.mark.parametrize("with_s0", [True, False])
def test_gradients_reach_the_right_inputs(oracle_backed, with_s0):
    x = I.prefill_inputs("fp32_small", T=20)
    if with_s0:
        x["S0"] = 0.1 * torch.randn(1, 2, 16, 16, generator=torch.Generator().manual_seed(1))
    names = ["q", "k", "v", "log_alpha", "beta"] + (["S0"] if with_s0 else [])
    t = leaves(x, names)
    out, S_T = kda.kda_prefill(t["q"], t["k"], t["v"], t["log_alpha"], t["beta"], t.get("S0"))
    g = torch.Generator().manual_seed(2)
    W1, W2 = torch.randn(out.shape, generator=g), torch.randn(S_T.shape, generator=g)
    (out * W1).sum().add((S_T * W2).sum()).backward()
    ref = grad.backward(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], W1, S0=x["S0"], dS_T=W2)
    for n in names:
        np.testing.assert_allclose(t[n].grad.double().numpy(), ref["d" + n], rtol=1e-5, atol=1e-6, err_msg=n)


def test_unused_output_gets_zero_cotangent(oracle_backed):
    x = I.prefill_inputs("fp32_small", T=12)
    t = leaves(x, ["q", "k", "v", "log_alpha", "beta"])
    _, S_T = kda.kda_prefill(t["q"], t["k"], t["v"], t["log_alpha"], t["beta"])
    W2 = torch.randn(S_T.shape, generator=torch.Generator().manual_seed(3))
    (S_T * W2).sum().backward()
    ref = grad.backward(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], torch.zeros(1, 12, 2, 16), dS_T=W2)
    np.testing.assert_allclose(t["k"].grad.double().numpy(), ref["dk"], rtol=1e-5, atol=1e-6)
    assert torch.all(t["q"].grad == 0)       # q only reaches the outputs
