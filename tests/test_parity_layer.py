"""Parity of the layer steps around the recurrence with the fp64 layer oracle (GPU).

* ``kda_short_conv_swish`` (ShortConv + Swish) against ``oracle.layer.short_conv_swish``:
  dense and packed sequences (empty ones included), filters of 1..4 taps, bf16 and
  fp32. The kernel accumulates in fp32 from the given inputs and rounds once to the
  output type, so the bound is that rounding (bf16 round-to-nearest: at most 2^-8
  relative) plus a few fp32 ulps of the taps' sum and the Swish (2^-18 relative):
  |y - ref| <= (2^-8 + 2^-18) |ref| + 1e-6 for bf16, 1e-5 |ref| + 1e-6 for fp32.
* ``kda_layer_fwd`` (fused prologue, recurrence, per-head RMSNorm and sigmoid output
  gate) against ``oracle.layer.layer_core``. The epilogue scales each row of o by
  g_w sigmoid(z) / rms(o), so the recurrence's bound on o (2e-3 + 1e-2 |o|) carries
  over scaled by that factor, plus the bf16 rounding of the result:
  |out - ref| <= s (2e-3 + 1e-2 |o_ref|) + 2^-8 |ref|, s = |g_w sigmoid(z)| / rms(o_ref).
  S_T keeps the recurrence's bound.
* the two chained, as a layer runs them: the convolved bf16 q, k, v feed the layer.
"""
import numpy as np
import pytest
import torch

import kda_inputs as I
from kda_check import BF16_ATOL, BF16_RTOL, BF16_STATE_MAX_ABS, assert_close, to_np
from oracle import layer

kda = pytest.importorskip("gated_delta_rule_116_b200")
pytestmark = pytest.mark.gpu
DEV = "cuda"


def conv_bound(ref, dtype):
    r = np.abs(to_np(ref))
    return ((2.0 ** -8 + 2.0 ** -18) * r + 1e-6) if dtype == torch.bfloat16 else (1e-5 * r + 1e-6)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("W", [1, 2, 3, 4])
def test_short_conv_dense(dtype, W):
    ex = I.layer_extras("prefill_4k", B=2, T=37, H=3, conv_width=W)
    x = ex["x_q"].to(dtype)
    w = ex["conv_q"]
    y = kda.short_conv_swish(x.to(DEV), w.to(DEV))
    torch.cuda.synchronize()
    ref = layer.short_conv_swish(x, w)
    assert_close(y, ref, conv_bound(ref, dtype), 0.0, f"short conv dense W={W} {dtype}")


@pytest.mark.parametrize("lens", [[0, 1, 17, 40, 0, 3], [100], [16, 16, 16]])
def test_short_conv_packed(lens):
    ex = I.layer_extras("prefill_4k", B=1, T=int(sum(lens)), H=2)
    x = ex["x_k"][0]
    w = ex["conv_k"]
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lens)]), dtype=torch.int32)
    y = kda.short_conv_swish(x.to(DEV), w.to(DEV), cu.to(DEV))
    torch.cuda.synchronize()
    ref = layer.short_conv_swish(x, w, cu.numpy())
    assert_close(y, ref, conv_bound(ref, torch.bfloat16), 0.0, f"short conv packed {lens}")


def test_short_conv_leaves_gaps_untouched():
    """Tokens outside every packed sequence keep their output values."""
    ex = I.layer_extras("fp32_small", B=1, T=30, H=2)
    x = ex["x_v"][0].float()
    w = ex["conv_v"]
    cu = torch.tensor([2, 10, 10, 25], dtype=torch.int32)
    y = torch.full_like(x, 7.0).to(DEV)
    kda.short_conv_swish(x.to(DEV), w.to(DEV), cu.to(DEV), out=y)
    torch.cuda.synchronize()
    y = y.cpu()
    assert torch.all(y[:2] == 7.0) and torch.all(y[25:] == 7.0)
    ref = layer.short_conv_swish(x[2:25], w, np.array([0, 8, 8, 23]))
    assert_close(y[2:25], ref, conv_bound(ref, torch.float32), 0.0, "short conv between gaps")


def layer_check(inp, ex, eps=1e-6, what="layer"):
    g = {k: (v.to(DEV) if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    out, st = kda.layer_fwd(g["q"], g["k"], g["v"], g["gate"], g["beta"], ex["out_gate"].to(DEV),
                            ex["norm_weight"].to(DEV), g["S0"], eps=eps)
    torch.cuda.synchronize()
    o_ref, s_ref = layer.fused_forward(inp["q"], inp["k"], inp["v"], inp["gate"], inp["beta"], inp["S0"])
    ref = layer.rms_norm_gate(o_ref, ex["out_gate"], ex["norm_weight"], eps)
    gain = np.abs(to_np(ex["norm_weight"]) * layer.sigmoid(ex["out_gate"]))
    s = gain / np.sqrt(np.mean(o_ref * o_ref, axis=-1, keepdims=True) + eps)
    bound = s * (BF16_ATOL + BF16_RTOL * np.abs(o_ref)) + 2.0 ** -8 * np.abs(ref)
    assert_close(out, ref, bound, 0.0, f"{what} out")
    assert_close(st, s_ref, BF16_ATOL, BF16_RTOL, f"{what} S_T", max_abs=BF16_STATE_MAX_ABS)


@pytest.mark.parametrize("name,kw", [
    ("prefill_4k", dict(B=2, T=300, H=3)),
    ("prefill_32k", dict(T=700, H=2)),
    ("prefill_4k", dict(B=1, T=260, H=2, gate="strong", s0_std=0.05)),
    ("prefill_4k", dict(B=2, T=65, H=2)),
])
def test_layer_fwd_matches_oracle(name, kw):
    inp = I.prefill_layer_inputs(name, **kw)
    layer_check(inp, I.layer_extras(name, **kw))


def test_layer_eps_matters_for_small_rows():
    """With v scaled down so that o is small, eps changes the result; both eps agree with the oracle."""
    inp = I.prefill_layer_inputs("prefill_4k", B=1, T=100, H=2)
    inp["v"] = (inp["v"].float() * 1e-3).to(torch.bfloat16)
    ex = I.layer_extras("prefill_4k", B=1, T=100, H=2)
    layer_check(inp, ex, eps=1e-6, what="layer eps 1e-6")
    layer_check(inp, ex, eps=1e-2, what="layer eps 1e-2")


def test_layer_pipeline_conv_then_layer():
    """ShortConv + Swish on the projected q, k, v, then the layer on their bf16 results."""
    kw = dict(B=1, T=200, H=2)
    base = I.prefill_layer_inputs("prefill_4k", **kw)
    ex = I.layer_extras("prefill_4k", **kw)
    conv = {}
    for n in ("q", "k", "v"):
        y = kda.short_conv_swish(ex[f"x_{n}"].to(DEV), ex[f"conv_{n}"].to(DEV))
        torch.cuda.synchronize()
        ref = layer.short_conv_swish(ex[f"x_{n}"], ex[f"conv_{n}"])
        assert_close(y, ref, conv_bound(ref, torch.bfloat16), 0.0, f"pipeline conv {n}")
        conv[n] = y.cpu()
    inp = dict(base, q=conv["q"], k=conv["k"], v=conv["v"])
    layer_check(inp, ex, what="pipeline layer")


def test_layer_rejects_missing_epilogue_inputs():
    inp = I.prefill_layer_inputs("prefill_4k", B=1, T=64, H=1)
    ex = I.layer_extras("prefill_4k", B=1, T=64, H=1)
    g = {k: (v.to(DEV) if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    lib = kda.load()
    out = torch.empty_like(g["v"])
    rc = lib.kda_layer_fwd(g["q"].data_ptr(), g["k"].data_ptr(), g["v"].data_ptr(), g["gate"].data_ptr(),
                           g["beta"].data_ptr(), None, ex["norm_weight"].to(DEV).data_ptr(), 1e-6, None,
                           out.data_ptr(), None, 1, 64, 1, 128, 128, 64, kda.KDA_BF16, None, 0, None)
    assert rc == -1   # KDA_ERR_INVALID_ARG: out_gate is NULL
