"""The combine folded into the down GEMM's epilogue, against the separate combine.

The per-expert overlap of the page "Balancing and Beyond: Communication-Centric
Optimizations in Expert Parallelism" (key idea): combine starts as the experts'
outputs are produced instead of after the last one. The fused form sums each token's
rows in j order once its last row is stored, with the separate combine's arithmetic,
so every output must be bit for bit the same as moe_combine's, for every tile shape,
with a shared expert and with capacity drops (a token may then have no row at all),
over calls in a row (the counters are zeroed by each call's dispatch).
"""
import pytest

import combine_warp_top_expert_b200 as moe
import moe_synth

pytestmark = pytest.mark.gpu

CASES = [
    ("tiny", moe_synth.workload("tiny"), 0.0),
    ("shared_e16_k4", moe_synth.Workload("fsh", T=300, d=512, E=16, k=4, f=256, R=4, n_shared=1, bias_kind="zipf",
                                         zipf_s=1.0, seed=2), 0.0),
    ("capacity_all_dropped", moe_synth.Workload("fcap", T=400, d=256, E=8, k=2, f=256, R=2, bias_kind="zipf",
                                                zipf_s=2.5, seed=4), 0.5),
    ("capacity_shared", moe_synth.Workload("fcs", T=256, d=384, E=16, k=4, f=128, R=4, n_shared=1, bias_kind="hot",
                                           n_hot=3, beta=2.0, seed=6), 1.0),
    ("multi_tile_e8", moe_synth.Workload("fmt", T=4096, d=2048, E=8, k=2, f=512, R=4, bias_kind="zipf", zipf_s=0.5,
                                         seed=5), 0.0),
]


def _bits(t):
    import torch
    return t.view(torch.int16)


@pytest.mark.parametrize("policy", [moe.GEMM_SINGLE, moe.GEMM_PAIR], ids=["single", "pair"])
@pytest.mark.parametrize("name,wl,cf", CASES, ids=[c[0] for c in CASES])
def test_fused_combine_is_bit_identical_to_the_separate_combine(name, wl, cf, policy):
    import torch
    cap = moe.capacity_for(cf, wl.T, wl.k, wl.E) if cf else 0
    shape = moe.Shape(T=wl.T, d=wl.d, E=wl.E, k=wl.k, f=wl.f, R=wl.R, n_shared=wl.n_shared, capacity=cap)
    dv = moe_synth.device_inputs(wl)
    old_p = moe.set_gemm_policy(policy)
    try:
        ref_layer = moe.MoELayer(shape, dv["w13"], dv["w2"], dv.get("w13s"), dv.get("w2s"))
        ref = {n: t.clone() for n, t in ref_layer(dv["logits"], dv["x"]).items() if t is not None}
        assert moe.get_status(ref_layer.ws) == 0
        if name == "capacity_all_dropped":
            kept = (ref["assign_row"].view(wl.T, wl.k) >= 0).sum(1)
            assert (kept == 0).any()        # some token keeps no row: its output must be zero
        old = moe.set_fused_combine(True)
        try:
            layer = moe.MoELayer(shape, dv["w13"], dv["w2"], dv.get("w13s"), dv.get("w2s"))
            for call in range(2):
                layer.outs["out"].fill_(7)   # a stale value that must be overwritten everywhere
                outs = layer(dv["logits"], dv["x"])
                assert moe.get_status(layer.ws) == 0
                assert torch.equal(_bits(outs["out"]), _bits(ref["out"])), (name, call)
                assert torch.equal(_bits(outs["y_perm"][:int(ref["expert_offsets"][-1])]),
                                   _bits(ref["y_perm"][:int(ref["expert_offsets"][-1])]))
        finally:
            moe.set_fused_combine(old)
        # the standalone entry point on the same inputs
        o = layer.outs
        out2 = torch.full_like(o["out"], 3)
        moe.moe_expert_gate_up(shape, o["x_perm"], o["expert_offsets"], dv["w13"], dv["x"], dv.get("w13s"), layer.ws)
        moe.moe_expert_down_combine(shape, o["expert_offsets"], dv["w2"], dv.get("w2s"), o["row_src"], o["assign_row"],
                                    o["topk_gate"], o["y_perm"], o.get("y_shared"), out2, layer.ws)
        assert moe.get_status(layer.ws) == 0
        assert torch.equal(_bits(out2), _bits(ref["out"]))
    finally:
        moe.set_gemm_policy(old_p)
