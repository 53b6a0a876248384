"""Expert parallelism across GPUs, emulated on one GPU: R ranks' buffers on this device.

Page "Expert Parallelism" §1 and §4 "The All-to-All": every rank routes its own
tokens, the kernels store each row into the receive buffer of the rank that owns its
expert (moe_ep_dispatch), each rank runs its experts' grouped GEMM on what it
received, and combine loads every result row back from its owner (moe_ep_combine).
Here the R ranks' buffers are R allocations on one GPU and the ranks' calls are
issued phase by phase (every wait finds its signals already stored; no kernel waits
on one that has yet to run).

The reference is one single-GPU moe_layer call on the R batches taken as one batch
(rank after rank), with R logical ranks: each rank's receive buffer must equal that
call's x_perm slice of logical rank r bit for bit, its expert outputs the y_perm
slice, and its out the out rows of its tokens (the same rows go through the same
kernels, so the results are the same bits), over two layer calls in a row.
"""
import numpy as np
import pytest

import combine_warp_top_expert_b200 as moe
import moe_synth
from combine_warp_top_expert_b200 import ep

pytestmark = pytest.mark.gpu


def _bits(t):
    import torch
    return t.view(torch.int16) if t.dtype == torch.bfloat16 else t


@pytest.mark.parametrize("R,n_shared,cf", [(2, 0, 0.0), (4, 1, 0.0), (4, 0, 1.25), (8, 1, 1.0), (1, 0, 0.0)],
                         ids=["r2", "r4_shared", "r4_capacity", "r8_shared_capacity", "r1"])
def test_emulated_ranks_match_the_single_gpu_layer(R, n_shared, cf):
    import torch
    Tl, E, k, d, f = 160, 16, 4, 512, 256
    wl = moe_synth.Workload("ep", T=R * Tl, d=d, E=E, k=k, f=f, R=R, n_shared=n_shared, bias_kind="zipf",
                            zipf_s=0.8, seed=40 + R)
    cap = moe.capacity_for(cf, wl.T, k, E) if cf else 0
    dv = moe_synth.device_inputs(wl)
    old = moe.set_gemm_policy(moe.GEMM_SINGLE)  # one tile shape on both sides
    try:
        g_shape = moe.Shape(T=wl.T, d=d, E=E, k=k, f=f, R=R, n_shared=n_shared, capacity=cap)
        glob = moe.MoELayer(g_shape, dv["w13"], dv["w2"], dv.get("w13s"), dv.get("w2s"))
        g = {n: (t.clone() if t is not None else None) for n, t in glob(dv["logits"], dv["x"]).items()}
        assert moe.get_status(glob.ws) == 0
        Er = E // R
        peers = ep.EPPeers.emulated(R, E, d, rows_cap=R * Tl * k)
        l_shape = moe.Shape(T=Tl, d=d, E=E, k=k, f=f, R=R, n_shared=n_shared, capacity=cap)
        layers = [ep.EPMoELayer(l_shape, r, dv["w13"][r * Er:(r + 1) * Er].contiguous(),
                                dv["w2"][r * Er:(r + 1) * Er].contiguous(), peers,
                                dv.get("w13s"), dv.get("w2s")) for r in range(R)]
        logits = [dv["logits"][r * Tl:(r + 1) * Tl].contiguous() for r in range(R)]
        xs = [dv["x"][r * Tl:(r + 1) * Tl].contiguous() for r in range(R)]
        for call in range(2):
            for lay in layers:
                lay.out.zero_()
                peers.recv[lay.rank].zero_()
                peers.y[lay.rank].zero_()
            outs = ep.run_emulated(layers, logits, xs)
            torch.cuda.synchronize()
            for r, lay in enumerate(layers):
                assert lay.status() == 0, (call, r)
                assert lay.epoch == call + 1
                lo, hi = int(g["rank_offsets"][r]), int(g["rank_offsets"][r + 1])
                want_off = g["expert_offsets"][r * Er:(r + 1) * Er + 1] - lo
                assert torch.equal(lay.recv_offsets, want_off), (call, r)
                assert torch.equal(_bits(peers.recv[r][:hi - lo]), _bits(g["x_perm"][lo:hi])), (call, r)
                assert torch.equal(_bits(peers.y[r][:hi - lo]), _bits(g["y_perm"][lo:hi])), (call, r)
                # every assignment's row on its owner: the global row minus the owner's first row
                ga = g["assign_row"][r * Tl * k:(r + 1) * Tl * k].long()
                owner = lay.topk_idx.reshape(-1).long() // Er
                want_row = torch.where(ga >= 0, ga - g["rank_offsets"].long()[owner], torch.full_like(ga, -1))
                assert torch.equal(lay.send_row.long(), want_row), (call, r)
                assert torch.equal(lay.topk_idx, g["topk_idx"][r * Tl:(r + 1) * Tl])
                assert torch.equal(_bits(outs[r]), _bits(g["out"][r * Tl:(r + 1) * Tl])), (call, r)
                if n_shared:
                    assert torch.equal(_bits(lay.y_shared), _bits(g["y_shared"][r * Tl:(r + 1) * Tl]))
    finally:
        moe.set_gemm_policy(old)


def test_device_plan_equals_the_host_plan():
    """recv_offsets from the plan kernel against moe_ep_plan_host on the same counts."""
    import torch
    R, Tl, E, k, d, f = 4, 96, 32, 8, 256, 128
    wl = moe_synth.Workload("epp", T=R * Tl, d=d, E=E, k=k, f=f, R=R, bias_kind="zipf", zipf_s=1.2, seed=3)
    dv = moe_synth.device_inputs(wl)
    cap = moe.capacity_for(1.0, wl.T, k, E)
    peers = ep.EPPeers.emulated(R, E, d, rows_cap=R * Tl * k)
    l_shape = moe.Shape(T=Tl, d=d, E=E, k=k, f=f, R=R, capacity=cap)
    Er = E // R
    layers = [ep.EPMoELayer(l_shape, r, dv["w13"][r * Er:(r + 1) * Er].contiguous(),
                            dv["w2"][r * Er:(r + 1) * Er].contiguous(), peers) for r in range(R)]
    ep.run_emulated(layers, [dv["logits"][r * Tl:(r + 1) * Tl].contiguous() for r in range(R)],
                    [dv["x"][r * Tl:(r + 1) * Tl].contiguous() for r in range(R)])
    counts_all = np.stack([lay.expert_counts.cpu().numpy() for lay in layers])
    for r, lay in enumerate(layers):
        assert np.array_equal(peers.counts[r].cpu().numpy(), counts_all)   # every table holds every row
        plan = moe.ep_plan_host(R, E, r, cap, counts_all)
        assert np.array_equal(lay.recv_offsets.cpu().numpy(), plan["recv_offsets"])
        assert lay.status() == 0


def test_a_wait_nobody_signals_times_out_and_the_context_stays_usable():
    """moe_ep_wait on a slot no rank has signalled for this epoch: the bounded wait runs
    out, MOE_DEV_TIMEOUT is raised, and the next calls work."""
    import torch
    R = 2
    peers = ep.EPPeers.emulated(R, 8, 128, rows_cap=64)
    ws = moe.new_workspace(moe.Shape(T=16, d=128, E=8, k=2, f=128, R=R))
    old = moe.set_wait_timeout_ns(50_000_000)
    try:
        moe.moe_ep_signal(R, 0, moe.EP_SLOT_DONE, 7, peers)       # rank 1 never signals
        moe.moe_ep_wait(R, 1, moe.EP_SLOT_DONE, 7, peers, ws)
        assert moe.get_status(ws) & moe.MOE_DEV_TIMEOUT
        moe.clear_status(ws)
        moe.moe_ep_signal(R, 1, moe.EP_SLOT_DONE, 7, peers)
        moe.moe_ep_wait(R, 0, moe.EP_SLOT_DONE, 7, peers, ws)     # now both have signalled
        assert moe.get_status(ws) == 0
        torch.cuda.synchronize()
    finally:
        moe.set_wait_timeout_ns(old)
