"""The seeded input recipe (kda_inputs.py) against the workloads it stands for (CPU).

Shapes, dtypes, seeds and the distributions of every workload: q and k unit
rows, v ~ N(0,1), beta = sigmoid(N(0,1)), the three gate recipes, S0 and the
decode state cache. Expected moments come from numerical quadrature, not from
the generator.
"""
import math

import numpy as np
import pytest
import torch

import kda_inputs as I


def normal_expectation(f, mean=0.0):
    """E[f(X)] for X ~ N(mean, 1) by a fine trapezoid rule."""
    x = np.linspace(mean - 12, mean + 12, 200001)
    w = np.exp(-0.5 * (x - mean) ** 2) / math.sqrt(2 * math.pi)
    return float(np.trapezoid(f(x) * w, x))


softplus = lambda x: np.logaddexp(0.0, x)
sigmoid = lambda x: 1.0 / (1.0 + np.exp(-x))


def test_workload_table():
    W = I.WORKLOADS
    assert (W["fp32_small"].B, W["fp32_small"].T, W["fp32_small"].H, W["fp32_small"].dk,
            W["fp32_small"].chunk, W["fp32_small"].dtype) == (1, 64, 2, 16, 16, torch.float32)
    assert (W["prefill_4k"].B, W["prefill_4k"].T, W["prefill_4k"].H, W["prefill_4k"].dk,
            W["prefill_4k"].chunk, W["prefill_4k"].dtype) == (8, 4096, 32, 128, 64, torch.bfloat16)
    p32 = W["prefill_32k"]
    assert (p32.B, p32.T, p32.H, p32.dk, p32.dv, p32.chunk, p32.gate, p32.s0_std) == \
        (1, 32768, 32, 128, 128, 64, "slow", 0.01)
    p128 = W["prefill_128k"]
    assert (p128.B, p128.T, p128.H, p128.dk, p128.gate, p128.s0_std) == (1, 131072, 16, 128, "mixed", 0.0)
    dec = W["decode_256"]
    assert (dec.N, dec.H, dec.dk, dec.dv, dec.steps, dec.state_std, dec.dtype) == \
        (256, 32, 128, 128, 1000, 0.05, torch.bfloat16)
    assert len({w.seed for w in W.values()}) == len(W)


@pytest.mark.parametrize("name,gate_mean_arg", [("prefill_4k", 0.0), ("prefill_32k", -2.0)])
def test_prefill_distributions(name, gate_mean_arg):
    x = I.prefill_inputs(name, B=1, T=2048, H=8)
    q, k, v, la, beta = x["q"], x["k"], x["v"], x["log_alpha"], x["beta"]
    assert q.shape == (1, 2048, 8, 128) and q.dtype == torch.bfloat16 and v.dtype == torch.bfloat16
    for t in (q, k):
        n = t.float().norm(dim=-1)
        assert torch.all((n - 1).abs() < 1e-2)           # unit rows, then the bf16 cast
    vf = v.float()
    assert abs(vf.mean().item()) < 0.01 and abs(vf.std().item() - 1) < 0.01
    assert torch.all((beta > 0) & (beta < 1))
    assert abs(beta.mean().item() - normal_expectation(sigmoid)) < 5e-3
    assert torch.all(la <= 0)
    assert abs(la.mean().item() + normal_expectation(softplus, gate_mean_arg)) < 5e-3
    if name == "prefill_32k":
        assert x["S0"].shape == (1, 8, 128, 128) and abs(x["S0"].std().item() - 0.01) < 2e-4
    else:
        assert x["S0"] is None


def test_mixed_gates_half_slow_channels():
    x = I.prefill_inputs("prefill_128k", T=1024, H=4)
    la = x["log_alpha"]
    assert torch.all(la[..., :64] == -1e-3)
    fast = la[..., 64:]
    assert abs(fast.mean().item() + normal_expectation(softplus)) < 5e-3


def test_small_fp32_workload():
    x = I.prefill_inputs("fp32_small")
    assert x["q"].dtype == torch.float32 and x["q"].shape == (1, 64, 2, 16)
    assert torch.allclose(x["q"].norm(dim=-1), torch.ones(1, 64, 2), atol=1e-6)


def test_seeded_and_reproducible():
    a = I.prefill_inputs("prefill_4k", B=1, T=128, H=2)
    b = I.prefill_inputs("prefill_4k", B=1, T=128, H=2)
    c = I.prefill_inputs("prefill_32k", B=1, T=128, H=2)
    for n in ("q", "k", "v", "log_alpha", "beta"):
        assert torch.equal(a[n], b[n])
        assert not torch.equal(a[n].float(), c[n].float())


def test_decode_state_and_steps():
    st = I.decode_state(N=16, H=4)
    assert st.shape == (16, 4, 128, 128) and abs(st.std().item() - 0.05) < 1e-3
    s0 = I.decode_step_inputs("decode_256", 0, N=16, H=4)
    s0b = I.decode_step_inputs("decode_256", 0, N=16, H=4)
    s1 = I.decode_step_inputs("decode_256", 1, N=16, H=4)
    assert s0["q"].shape == (16, 4, 128) and s0["beta"].shape == (16, 4)
    assert torch.equal(s0["k"], s0b["k"]) and not torch.equal(s0["k"], s1["k"])
    assert torch.all(s0["log_alpha"] <= 0)


def test_strong_gate_recipe():
    """The edge-case recipe: fixed log a on channel classes c % 8 = 0..3, softplus elsewhere."""
    x = I.prefill_inputs("prefill_4k", B=1, T=256, H=2, gate="strong")
    la = x["log_alpha"]
    assert torch.all(la[..., 0::8] == -4.0) and torch.all(la[..., 1::8] == 0.0)
    assert torch.all(la[..., 2::8] == -12.0) and torch.all(la[..., 3::8] == np.float32(-1e-3))
    rest = torch.cat([la[..., c::8] for c in range(4, 8)], dim=-1)
    assert torch.all(rest < 0)
    assert abs(rest.mean().item() + normal_expectation(softplus)) < 2e-2
    # a 64-token chunk on a c % 8 == 0 channel decays by e^-256: beyond a chunk-midpoint anchor
    assert float(la[0, :64, 0, 0].sum()) == -256.0


def test_layer_inputs_recipe():
    """Raw q/k (not unit rows) and gate pre-activations whose -softplus gives the recipe's log a."""
    x = I.prefill_layer_inputs("prefill_128k", T=64, H=2)
    assert x["q"].dtype == torch.bfloat16 and x["gate"].dtype == torch.bfloat16
    assert not torch.allclose(x["q"].float().norm(dim=-1), torch.ones(1, 64, 2), atol=0.1)
    la = -torch.nn.functional.softplus(x["gate"].double())
    np.testing.assert_allclose(la[..., :64].numpy(), -1e-3, rtol=5e-3)   # bf16 of the fixed x
    s = I.prefill_layer_inputs("prefill_4k", B=1, T=32, H=1, gate="strong")
    las = -torch.nn.functional.softplus(s["gate"].double())
    np.testing.assert_allclose(las[..., 0::8].numpy(), -4.0, rtol=2e-2)
    assert float(las[..., 1::8].abs().max()) < 1e-12
    np.testing.assert_allclose(las[..., 2::8].numpy(), -12.0, rtol=2e-2)
    sl = I.prefill_layer_inputs("prefill_32k", T=2048, H=4)
    assert abs(sl["gate"].float().mean().item() + 2.0) < 0.02     # x ~ N(-2, 1): the slow recipe


def test_layer_extras_shapes_and_determinism():
    a = I.layer_extras("prefill_4k", B=1, T=5, H=2, conv_width=3)
    b = I.layer_extras("prefill_4k", B=1, T=5, H=2, conv_width=3)
    assert a["out_gate"].shape == (1, 5, 2, 128) and a["out_gate"].dtype == torch.bfloat16
    assert a["norm_weight"].shape == (128,) and a["norm_weight"].dtype == torch.float32
    assert a["conv_q"].shape == (2, 128, 3) and a["x_v"].shape == (1, 5, 2, 128)
    for key in ("out_gate", "norm_weight", "conv_q", "conv_k", "conv_v", "x_q", "x_k", "x_v"):
        assert torch.equal(a[key], b[key])
    assert abs(float(a["norm_weight"].mean()) - 1.0) < 0.05
