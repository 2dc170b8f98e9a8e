"""The give-up path of the tensor-core prefill engine's bounded device waits (GPU).

Every wait of the cluster engine -- on a peer CTA's signal, on a TMA copy, on
an MMA -- is bounded. The host-set test hook ``binding.test_inject_wait_timeout``
makes launches give up on purpose: a short wait limit and one withheld "chunk
operands ready" signal, so the state-chain CTA's wait runs out. Nothing faults,
traps or hangs: the launch comes back, every CTA stops issuing copies and MMAs,
waits for those in flight and exits, ``device_status`` reports
KDA_ERR_DEVICE_TIMEOUT, and the next normal launch on the same context is
correct.
"""
import pytest
import torch

import kda_inputs as I
import oracle
from kda_check import assert_close, state_max_abs, tol_for

kda = pytest.importorskip("gated_delta_rule_116_b200")
from gated_delta_rule_116_b200 import binding  # noqa: E402

pytestmark = pytest.mark.gpu


def run(g):
    out, st = kda.chunk_fwd(g["q"], g["k"], g["v"], g["log_alpha"], g["beta"], g["S0"], chunk=64,
                            engine="tc_cluster")
    torch.cuda.synchronize()
    return out, st


def test_bounded_wait_gives_up_and_the_next_launch_is_correct():
    # 11 chunks per head: every producer CTA has more images than ring slots, so the
    # producers also wait on the state-chain CTA when it has given up
    inp = I.prefill_inputs("prefill_32k", B=2, T=700, H=3)
    g = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    kda.device_status()   # nothing pending from earlier launches
    old = binding.test_inject_wait_timeout(True)
    try:
        run(g)   # the launch itself succeeds; the failure is reported by the device
        with pytest.raises(kda.KdaError, match="KDA_ERR_DEVICE_TIMEOUT"):
            kda.device_status()
        run(g)   # a second give-up in a row is reported again
        with pytest.raises(kda.KdaError, match="KDA_ERR_DEVICE_TIMEOUT"):
            kda.device_status()
    finally:
        binding.test_inject_wait_timeout(old)
    out, st = run(g)
    kda.device_status()   # the flag was cleared and this launch did not give up
    ref_out, ref_st = oracle.forward(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"],
                                     inp["S0"])
    atol, rtol = tol_for(torch.bfloat16)
    assert_close(out, ref_out, atol, rtol, "out after a give-up")
    assert_close(st, ref_st, atol, rtol, "S_T after a give-up", max_abs=state_max_abs(torch.bfloat16))
