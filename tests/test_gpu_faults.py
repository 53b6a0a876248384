"""Failure detection on the GPU without faulting it.

Every wait in the grouped-GEMM pipeline is bounded. The library's test hook
(moe_set_test_stall) makes each CTA arm its first pipeline stage and never load
it, so the MMA's wait on that stage can only run out (a flag that nothing sets).
With a 50 ms limit the kernel must report MOE_DEV_TIMEOUT in the status word,
wait for its real copies and MMAs, free its tensor memory and return, and the
context must stay usable (the next call, hook off and default limit, is
correct). Nothing here traps, asserts or reads out of bounds on the device.
"""
import numpy as np
import pytest

import combine_warp_top_expert_b200 as moe
import moe_synth
import oracle
from parity_util import bits, close, f64

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("policy", [moe.GEMM_SINGLE, moe.GEMM_PAIR], ids=["single_tiles", "pair_tiles"])
def test_pipeline_wait_timeout_is_reported_and_context_survives(policy):
    import torch
    wl = moe_synth.workload("tiny")
    shape = moe.Shape(T=wl.T, d=wl.d, E=wl.E, k=wl.k, f=wl.f, R=wl.R)
    dv = moe_synth.device_inputs(wl)
    idx, gate, _ = oracle.route(moe_synth.host_logits(wl), wl.k)
    ref = oracle.dispatch(idx, wl.E, wl.R)
    x_np = moe_synth.host_x(wl)
    xp_np = oracle.permute_rows(x_np, ref["row_src"], wl.k)
    xp = torch.from_numpy(xp_np.view(np.int16)).cuda().view(torch.bfloat16)
    offs = torch.from_numpy(ref["expert_offsets"]).cuda()
    y = torch.zeros((shape.A, wl.d), dtype=torch.bfloat16, device="cuda")
    ws = moe.new_workspace(shape)
    old_policy = moe.set_gemm_policy(policy)
    try:
        moe.set_wait_timeout_ns(50_000_000)
        moe.set_test_stall(True)
        try:
            moe.moe_expert_ffn(shape, xp, offs, dv["w13"], dv["w2"], None, None, None, y, None, ws)
            status = moe.get_status(ws)
        finally:
            moe.set_test_stall(False)
            moe.set_wait_timeout_ns(0)
        assert status & moe.MOE_DEV_TIMEOUT
        # the context is still usable and the same call is now correct
        moe.clear_status(ws)
        moe.moe_expert_ffn(shape, xp, offs, dv["w13"], dv["w2"], None, None, None, y, None, ws)
        assert moe.get_status(ws) == 0
    finally:
        moe.set_gemm_policy(old_policy)
    y_ref, _ = oracle.expert_ffn(xp_np, ref["expert_offsets"], moe_synth.host_w13(wl), moe_synth.host_w2(wl))
    close(f64(bits(y)), y_ref, "y_perm after timeout")


def test_gathering_gemm_wait_timeout_is_reported_and_context_survives():
    """The bounded-wait path of the GEMM1 variant whose producer warp gathers rows of x."""
    import torch
    wl = moe_synth.workload("tiny")
    shape = moe.Shape(T=wl.T, d=wl.d, E=wl.E, k=wl.k, f=wl.f, R=wl.R)
    dv = moe_synth.device_inputs(wl)
    idx, _, _ = oracle.route(moe_synth.host_logits(wl), wl.k)
    ref = oracle.dispatch(idx, wl.E, wl.R)
    row_src = torch.from_numpy(ref["row_src"]).cuda()
    offs = torch.from_numpy(ref["expert_offsets"]).cuda()
    y = torch.zeros((shape.A, wl.d), dtype=torch.bfloat16, device="cuda")
    ws = moe.new_workspace(shape)

    def run():
        moe.moe_expert_gate_up_gather(shape, dv["x"], row_src, offs, dv["w13"], None, ws)
        moe.moe_expert_down(shape, offs, dv["w2"], None, y, None, ws)

    moe.set_wait_timeout_ns(50_000_000)
    moe.set_test_stall(True)
    try:
        run()
        status = moe.get_status(ws)
    finally:
        moe.set_test_stall(False)
        moe.set_wait_timeout_ns(0)
    assert status & moe.MOE_DEV_TIMEOUT
    moe.clear_status(ws)
    run()
    assert moe.get_status(ws) == 0
    xp_np = oracle.permute_rows(moe_synth.host_x(wl), ref["row_src"], wl.k)
    y_ref, _ = oracle.expert_ffn(xp_np, ref["expert_offsets"], moe_synth.host_w13(wl), moe_synth.host_w2(wl))
    close(f64(bits(y)), y_ref, "y_perm after a timeout in the gathering GEMM")
