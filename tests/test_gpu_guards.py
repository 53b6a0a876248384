"""Guard zones: no kernel of the layer writes outside the buffers it is given.

Every output buffer and the workspace are carved out of a larger allocation whose
bytes before and after the buffer (and the padding up to the next 256 bytes) hold
a known pattern; after the layer (and the separate entry points) run, every guard
byte must still hold it. Shapes cover ragged expert ends around the 32-, 128- and
256-row tile boundaries, every GEMM tile policy, capacity drops, the shared
expert and the path that gathers rows of x inside the GEMM.
"""
import numpy as np
import pytest

import combine_warp_top_expert_b200 as moe
import moe_synth
import oracle
from parity_util import bits, close, f64

pytestmark = pytest.mark.gpu

GUARD = 4096          # bytes on each side (keeps 256-byte alignment of the buffer)
PATTERN = 0xA5


class Guarded:
    """A tensor of `shape`/`dtype` inside a pattern-filled byte buffer."""

    def __init__(self, shape, dtype):
        import torch
        n = int(np.prod(shape)) * torch.empty((), dtype=dtype).element_size()
        self.n = n
        self.pad = -(-n // 256) * 256
        self.raw = torch.full((GUARD + self.pad + GUARD,), PATTERN, dtype=torch.uint8, device="cuda")
        self.t = self.raw[GUARD:GUARD + n].view(dtype).view(shape) if n else torch.empty(shape, dtype=dtype,
                                                                                         device="cuda")

    def intact(self) -> bool:
        import torch
        head = self.raw[:GUARD]
        tail = self.raw[GUARD + self.n:]
        return bool(torch.all(head == PATTERN).item()) and bool(torch.all(tail == PATTERN).item())


def _guarded_outputs(shape, x_perm=True):
    import torch
    i32, f32, bf = torch.int32, torch.float32, torch.bfloat16
    T, k, E, R, d, A = shape.T, shape.k, shape.E, shape.R, shape.d, shape.A
    spec = dict(topk_idx=((T, k), i32), topk_gate=((T, k), f32), expert_counts=((E,), i32),
                expert_offsets=((E + 1,), i32), rank_counts=((R,), i32), rank_offsets=((R + 1,), i32),
                row_src=((A,), i32), assign_row=((A,), i32), imbalance=((2,), f32), y_perm=((A, d), bf),
                out=((T, d), bf))
    if x_perm:
        spec["x_perm"] = ((A, d), bf)
    if shape.n_shared:
        spec["y_shared"] = ((T, d), bf)
    g = {n: Guarded(s, t) for n, (s, t) in spec.items()}
    outs = {n: (g[n].t if n in g else None) for n in moe._LAYER_OUTPUTS}
    return g, outs


def _ws(shape):
    ws = Guarded((moe.workspace_bytes(shape),), __import__("torch").uint8)
    ws.t.zero_()
    return ws


CASES = [
    # (workload, capacity factor, gather x rows in the GEMM)
    (moe_synth.Workload("g_tail", T=300, d=256, E=3, k=1, f=384, R=1, n_shared=1, bias_kind="hot", n_hot=1,
                        beta=4.0), None, False),
    (moe_synth.Workload("g_zipf", T=257, d=384, E=8, k=2, f=256, R=4, bias_kind="zipf", zipf_s=1.0), None, False),
    (moe_synth.Workload("g_cap", T=300, d=256, E=8, k=2, f=256, R=4, n_shared=1, bias_kind="zipf", zipf_s=1.0),
     1.25, False),
    (moe_synth.Workload("g_gather", T=200, d=256, E=16, k=4, f=256, R=4, n_shared=1, bias_kind="zipf",
                        zipf_s=1.0), None, True),
    (moe_synth.Workload("g_big", T=1100, d=512, E=4, k=2, f=512, R=2, bias_kind="hot", n_hot=1, beta=2.0), None,
     False),
]


@pytest.mark.parametrize("policy", [moe.GEMM_AUTO, moe.GEMM_SINGLE, moe.GEMM_PAIR],
                         ids=["auto", "single", "pair"])
@pytest.mark.parametrize("wl,cf,gather", CASES, ids=[c[0].name for c in CASES])
def test_layer_writes_stay_inside_their_buffers(wl, cf, gather, policy):
    cap = moe.capacity_for(cf, wl.T, wl.k, wl.E) if cf else 0
    shape = moe.Shape(T=wl.T, d=wl.d, E=wl.E, k=wl.k, f=wl.f, R=wl.R, n_shared=wl.n_shared, capacity=cap)
    dv = moe_synth.device_inputs(wl)
    g, outs = _guarded_outputs(shape, x_perm=not gather)
    ws = _ws(shape)
    old = moe.set_gemm_policy(policy)
    try:
        moe.moe_layer(shape, dv["logits"], dv["x"], dv["w13"], dv["w2"], dv.get("w13s"), dv.get("w2s"), outs, ws.t)
        status = moe.get_status(ws.t)
    finally:
        moe.set_gemm_policy(old)
    assert status == 0
    for n, b in g.items():
        assert b.intact(), f"{n}: a guard byte was overwritten"
    assert ws.intact(), "workspace guard overwritten"
    res = oracle.layer(moe_synth.host_x(wl), moe_synth.host_logits(wl), moe_synth.host_w13(wl),
                       moe_synth.host_w2(wl), wl.k, wl.R, moe_synth.host_w13s(wl) if wl.n_shared else None,
                       moe_synth.host_w2s(wl) if wl.n_shared else None, capacity=cap)
    close(f64(bits(outs["out"])), res["out"], "out (guarded buffers)")


def test_separate_entry_points_write_inside_their_buffers():
    """route -> dispatch -> gate/up -> down -> combine, each call on guarded buffers."""
    wl = moe_synth.Workload("g_steps", T=333, d=256, E=6, k=2, f=256, R=2, n_shared=1, bias_kind="zipf",
                            zipf_s=1.0)
    shape = moe.Shape(T=wl.T, d=wl.d, E=wl.E, k=wl.k, f=wl.f, R=wl.R, n_shared=wl.n_shared)
    dv = moe_synth.device_inputs(wl)
    g, o = _guarded_outputs(shape)
    ws = _ws(shape)
    moe.moe_route(shape, dv["logits"], o["topk_idx"], o["topk_gate"], ws.t)
    moe.moe_dispatch(shape, dv["x"], o["topk_idx"], o["expert_counts"], o["expert_offsets"], o["rank_counts"],
                     o["rank_offsets"], o["row_src"], o["assign_row"], o["x_perm"], o["imbalance"], ws.t)
    moe.moe_expert_gate_up(shape, o["x_perm"], o["expert_offsets"], dv["w13"], dv["x"], dv["w13s"], ws.t)
    moe.moe_expert_down(shape, o["expert_offsets"], dv["w2"], dv["w2s"], o["y_perm"], o["y_shared"], ws.t)
    moe.moe_combine(shape, o["y_perm"], o["assign_row"], o["topk_gate"], o["y_shared"], o["out"], ws.t)
    assert moe.get_status(ws.t) == 0
    for n, b in g.items():
        assert b.intact(), f"{n}: a guard byte was overwritten"
    assert ws.intact(), "workspace guard overwritten"


@pytest.mark.parametrize("policy", [moe.GEMM_SINGLE, moe.GEMM_PAIR], ids=["single", "pair"])
@pytest.mark.parametrize("wl,cf,gather", CASES, ids=[c[0].name for c in CASES])
def test_layer_with_the_fused_combine_writes_inside_its_buffers(wl, cf, gather, policy):
    """The combine folded into the down GEMM's epilogue (and the dispatch that zeroes its
    counters) writes out and the workspace's counters only inside their buffers."""
    cap = moe.capacity_for(cf, wl.T, wl.k, wl.E) if cf else 0
    shape = moe.Shape(T=wl.T, d=wl.d, E=wl.E, k=wl.k, f=wl.f, R=wl.R, n_shared=wl.n_shared, capacity=cap)
    dv = moe_synth.device_inputs(wl)
    g, outs = _guarded_outputs(shape, x_perm=not gather)
    ws = _ws(shape)
    old, old_f = moe.set_gemm_policy(policy), moe.set_fused_combine(True)
    try:
        moe.moe_layer(shape, dv["logits"], dv["x"], dv["w13"], dv["w2"], dv.get("w13s"), dv.get("w2s"), outs, ws.t)
        status = moe.get_status(ws.t)
    finally:
        moe.set_gemm_policy(old)
        moe.set_fused_combine(old_f)
    assert status == 0
    for n, b in g.items():
        assert b.intact(), f"{n}: a guard byte was overwritten"
    assert ws.intact(), "workspace guard overwritten"
    res = oracle.layer(moe_synth.host_x(wl), moe_synth.host_logits(wl), moe_synth.host_w13(wl),
                       moe_synth.host_w2(wl), wl.k, wl.R, moe_synth.host_w13s(wl) if wl.n_shared else None,
                       moe_synth.host_w2s(wl) if wl.n_shared else None, capacity=cap)
    close(f64(bits(outs["out"])), res["out"], "out (fused combine, guarded buffers)")
