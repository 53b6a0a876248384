"""GPU parity of each step against the CPU oracle, through the C ABI.

Inputs come from the seeded generator (host fill for the oracle, device fill or
a host->device copy for the GPU); every expected value comes from the oracle.
Routing, counts, offsets, permutation, x_perm and imbalance are compared bit
for bit; gates within 2^-20; bf16 outputs within rel-L2 5e-3 and max-abs
3e-2 * max|ref| (tests/parity_util.py).
"""
import numpy as np
import pytest

import combine_warp_top_expert_b200 as moe
import moe_synth
import oracle
from parity_util import GATE_TOL, bits, close, f64, np_i32

pytestmark = pytest.mark.gpu

WORKLOADS = ["tiny", "mixtral_prefill", "dsv3_decode", "qwen3_mixed", "dsv3_skewed_prefill"]


def _torch():
    import torch
    return torch


def _shape(wl):
    return moe.Shape(T=wl.T, d=wl.d, E=wl.E, k=wl.k, f=wl.f, R=wl.R, n_shared=wl.n_shared)


def _bf16_dev(a_bits):
    torch = _torch()
    return torch.from_numpy(np.ascontiguousarray(a_bits).view(np.int16)).cuda().view(torch.bfloat16)


def _gpu_route(shape, logits_np):
    torch = _torch()
    lg = torch.from_numpy(np.ascontiguousarray(logits_np, np.float32)).cuda()
    idx = torch.empty((shape.T, shape.k), dtype=torch.int32, device="cuda")
    gate = torch.empty((shape.T, shape.k), dtype=torch.float32, device="cuda")
    ws = moe.new_workspace(shape)
    moe.moe_route(shape, lg, idx, gate, ws)
    return np_i32(idx), gate.cpu().numpy(), moe.get_status(ws)


def _gpu_dispatch(shape, x_dev, idx_np):
    torch = _torch()
    i32 = torch.int32
    dev = "cuda"
    o = dict(expert_counts=torch.empty(shape.E, dtype=i32, device=dev),
             expert_offsets=torch.empty(shape.E + 1, dtype=i32, device=dev),
             rank_counts=torch.empty(shape.R, dtype=i32, device=dev),
             rank_offsets=torch.empty(shape.R + 1, dtype=i32, device=dev),
             row_src=torch.empty(shape.A, dtype=i32, device=dev),
             assign_row=torch.empty(shape.A, dtype=i32, device=dev),
             x_perm=torch.empty((shape.A, shape.d), dtype=torch.bfloat16, device=dev),
             imbalance=torch.empty(2, dtype=torch.float32, device=dev))
    ws = moe.new_workspace(shape)
    idx = torch.from_numpy(np.ascontiguousarray(idx_np, np.int32)).cuda()
    moe.moe_dispatch(shape, x_dev, idx, o["expert_counts"], o["expert_offsets"], o["rank_counts"],
                     o["rank_offsets"], o["row_src"], o["assign_row"], o["x_perm"], o["imbalance"], ws)
    o["status"] = moe.get_status(ws)
    return o


@pytest.fixture(params=[moe.DISPATCH_AUTO, moe.DISPATCH_TWO_PASS, moe.DISPATCH_ONE_PASS],
                ids=["auto", "two_pass", "one_pass"])
def dispatch_path(request):
    """Every dispatch path must give the same bits: the two-kernel path (histogram, last
    CTA's scan, permute) and the one-pass kernel (every CTA counts all ids itself)."""
    old = moe.set_dispatch_path(request.param)
    yield request.param
    moe.set_dispatch_path(old)


# ---------------------------------------------------------------------------
# generator: device fill == host fill
# ---------------------------------------------------------------------------

def test_device_fill_equals_host_fill():
    wl = moe_synth.workload("tiny").with_(n_shared=1)
    dv = moe_synth.device_inputs(wl)
    assert np.array_equal(bits(dv["x"]), moe_synth.host_x(wl))
    assert np.array_equal(dv["logits"].cpu().numpy().view(np.uint32), moe_synth.host_logits(wl).view(np.uint32))
    assert np.array_equal(bits(dv["w13"]), moe_synth.host_w13(wl))
    assert np.array_equal(bits(dv["w2"]), moe_synth.host_w2(wl))
    assert np.array_equal(bits(dv["w13s"]), moe_synth.host_w13s(wl))
    wl5 = moe_synth.workload("dsv3_skewed_prefill")
    lg = moe_synth.device_inputs(wl5, weights=False)["logits"]
    assert np.array_equal(lg.cpu().numpy().view(np.uint32), moe_synth.host_logits(wl5).view(np.uint32))


# ---------------------------------------------------------------------------
# route
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("name", WORKLOADS)
def test_route_matches_oracle(name):
    wl = moe_synth.workload(name)
    lg = moe_synth.host_logits(wl)
    idx, gate, status = _gpu_route(_shape(wl), lg)
    ridx, rgate, _ = oracle.route(lg, wl.k)
    assert status == 0
    assert np.array_equal(idx, ridx)
    assert np.max(np.abs(gate.astype(np.float64) - rgate)) <= GATE_TOL


@pytest.mark.parametrize("E,k", [(1, 1), (5, 3), (8, 8), (33, 4), (64, 2), (256, 8), (255, 7)])
def test_route_ties_signed_zeros_and_infinities(E, k):
    rng = np.random.default_rng(E * 7 + k)
    T = 777
    lg = rng.integers(-2, 3, size=(T, E)).astype(np.float32)           # exact ties everywhere
    lg[::5] = np.where(lg[::5] == 0, np.float32(-0.0), lg[::5])         # -0.0 ties +0.0
    lg[3] = -np.inf                                                      # all -inf: gates 1/k
    lg[4, : E // 2] = -np.inf
    shape = moe.Shape(T=T, d=128, E=E, k=k, f=128, R=1)
    idx, gate, status = _gpu_route(shape, lg)
    ridx, rgate, nan = oracle.route(lg, k)
    assert status == 0 and nan == 0
    assert np.array_equal(idx, ridx)
    assert np.max(np.abs(gate.astype(np.float64) - rgate)) <= GATE_TOL


@pytest.mark.parametrize("E,k", [(8, 2), (256, 8), (200, 5)])
def test_route_positive_infinity_orders_first(E, k):
    """+inf ranks above every finite logit, ties to the lower index among +inf; the gate
    of a +inf expert is NaN (inf - inf) on both sides, so gates are compared where finite."""
    rng = np.random.default_rng(E + k)
    T = 300
    lg = rng.normal(size=(T, E)).astype(np.float32)
    lg[::3, E // 2] = np.inf
    lg[1::3, [E - 1, 0]] = np.inf
    lg[5, :] = np.inf
    shape = moe.Shape(T=T, d=128, E=E, k=k, f=128, R=1)
    idx, gate, status = _gpu_route(shape, lg)
    ridx, rgate, nan = oracle.route(lg, k)
    assert status == 0 and nan == 0
    assert np.array_equal(idx, ridx)
    g = gate.astype(np.float64)
    assert np.array_equal(np.isnan(g), np.isnan(rgate))
    fin = ~np.isnan(rgate)
    assert np.max(np.abs(g[fin] - rgate[fin])) <= GATE_TOL


def test_route_nan_is_ordered_last_and_flagged():
    lg = np.random.default_rng(0).normal(size=(64, 16)).astype(np.float32)
    lg[7, 3] = np.nan
    lg[9, :] = np.nan
    shape = moe.Shape(T=64, d=128, E=16, k=4, f=128, R=1)
    idx, gate, status = _gpu_route(shape, lg)
    ridx, rgate, nan = oracle.route(lg, 4)
    assert nan == 17 and status & moe.MOE_DEV_NAN_LOGIT
    assert np.array_equal(idx, ridx)
    assert np.max(np.abs(gate.astype(np.float64) - rgate)) <= GATE_TOL


# ---------------------------------------------------------------------------
# dispatch
# ---------------------------------------------------------------------------

def _check_dispatch(o, ref, x_np=None, k=None):
    for n in ("expert_counts", "expert_offsets", "rank_counts", "rank_offsets", "row_src", "assign_row"):
        assert np.array_equal(np_i32(o[n]), ref[n]), n
    assert np.array_equal(o["imbalance"].cpu().numpy().view(np.uint32), ref["imbalance"].view(np.uint32))
    if x_np is not None:
        ref_xp = oracle.permute_rows(x_np, ref["row_src"], k)
        total = ref["expert_offsets"][-1]
        assert np.array_equal(bits(o["x_perm"])[:total], ref_xp[:total])


@pytest.mark.parametrize("name", WORKLOADS)
def test_dispatch_matches_oracle(name, dispatch_path):
    torch = _torch()
    wl = moe_synth.workload(name)
    shape = _shape(wl)
    ridx, _, _ = oracle.route(moe_synth.host_logits(wl), wl.k)
    ref = oracle.dispatch(ridx, wl.E, wl.R)
    x_dev = moe_synth.device_inputs(wl, weights=False)["x"]
    o = _gpu_dispatch(shape, x_dev, ridx)
    assert o["status"] == 0
    if wl.T * wl.d <= (1 << 24):
        _check_dispatch(o, ref, moe_synth.host_x(wl), wl.k)
    else:
        _check_dispatch(o, ref)
        # x_perm at full size: every row equals its token's row (property), checked on the device
        a = torch.arange(shape.A, device="cuda")
        rows = torch.from_numpy(ref["assign_row"]).cuda().long()
        xp = o["x_perm"].view(torch.int16)
        xs = x_dev.view(torch.int16)
        for c in torch.split(a, 1 << 14):
            assert torch.equal(xp[rows[c]], xs[c // wl.k])
        # and a sample of rows against the host-generated x, bit for bit
        samp = np.random.default_rng(1).choice(shape.A, 64, replace=False)
        toks = samp // wl.k
        got = bits(o["x_perm"][torch.from_numpy(ref["assign_row"][samp]).cuda().long()])
        assert np.array_equal(got, moe_synth.host_x(wl, toks))


def test_dispatch_worked_imbalance_example(dispatch_path):
    counts = np.array([140, 95, 78, 62, 48, 40, 31, 18])
    experts = np.repeat(np.arange(8), counts)
    np.random.default_rng(7).shuffle(experts)
    idx = experts.reshape(512, 1).astype(np.int32)
    x_np = moe_synth.host_x(moe_synth.Workload("p5", T=512, d=512, E=8, k=1, f=1024, R=8))
    for R, imb in ((8, (2.1875, 2.1875)), (2, (1.46484375, 2.1875))):
        shape = moe.Shape(T=512, d=512, E=8, k=1, f=1024, R=R)
        o = _gpu_dispatch(shape, _bf16_dev(x_np), idx)
        ref = oracle.dispatch(idx, 8, R)
        _check_dispatch(o, ref, x_np, 1)
        assert tuple(o["imbalance"].cpu().numpy().tolist()) == imb
        assert list(np_i32(o["expert_counts"])) == counts.tolist()


@pytest.mark.parametrize("T,E,k,R", [(0, 8, 2, 2), (1, 1, 1, 1), (1, 256, 8, 8), (1000, 37, 5, 1), (4099, 64, 3, 16),
                                     (2049, 8, 1, 4), (3000, 256, 8, 8)])
def test_dispatch_edge_shapes(T, E, k, R, dispatch_path):
    rng = np.random.default_rng(T + E)
    idx = rng.integers(0, E, size=(T, k)).astype(np.int32)   # repeats within a token allowed
    shape = moe.Shape(T=T, d=128, E=E, k=k, f=128, R=R)
    x_np = moe_synth.host_x(moe_synth.Workload("e", T=T, d=128, E=E, k=k, f=128, R=R))
    o = _gpu_dispatch(shape, _bf16_dev(x_np), idx)
    assert o["status"] == 0
    _check_dispatch(o, oracle.dispatch(idx, E, R), x_np, k)
    if T == 0:
        assert o["imbalance"].cpu().numpy().tolist() == [1.0, 1.0]


def test_dispatch_out_of_range_entries_are_skipped_and_flagged(dispatch_path):
    T, E, k = 300, 16, 2
    idx = np.random.default_rng(3).integers(0, E, size=(T, k)).astype(np.int32)
    idx[5, 1] = E
    idx[100, 0] = -3
    shape = moe.Shape(T=T, d=128, E=E, k=k, f=128, R=4)
    x_np = moe_synth.host_x(moe_synth.Workload("e", T=T, d=128, E=E, k=k, f=128, R=4))
    o = _gpu_dispatch(shape, _bf16_dev(x_np), idx)
    ref = oracle.dispatch(idx, E, 4)
    assert ref["skipped"] == 2 and o["status"] & moe.MOE_DEV_BOUNDS
    _check_dispatch(o, ref, x_np, k)


# ---------------------------------------------------------------------------
# combine
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("shared", [False, True])
@pytest.mark.parametrize("T,d,E,k", [(256, 512, 8, 2), (130, 1024, 64, 8), (1, 128, 4, 3)])
def test_combine_matches_oracle(T, d, E, k, shared):
    torch = _torch()
    wl = moe_synth.Workload("c", T=T, d=d, E=E, k=k, f=128, R=1, seed=11)
    idx, gate, _ = oracle.route(moe_synth.host_logits(wl), k)
    ref = oracle.dispatch(idx, E, 1)
    y_np = moe_synth.host_x(wl.with_(T=T * k, seed=12))     # any bf16 rows stand in for expert outputs
    ys_np = moe_synth.host_x(wl.with_(seed=13)) if shared else None
    shape = moe.Shape(T=T, d=d, E=E, k=k, f=128, R=1)
    out = torch.empty((T, d), dtype=torch.bfloat16, device="cuda")
    ws = moe.new_workspace(shape)
    moe.moe_combine(shape, _bf16_dev(y_np), torch.from_numpy(ref["assign_row"]).cuda(),
                    torch.from_numpy(gate).cuda(), _bf16_dev(ys_np) if shared else None, out, ws)
    assert moe.get_status(ws) == 0
    expect = oracle.combine(f64(y_np), ref["assign_row"], gate, f64(ys_np) if shared else None)
    close(f64(bits(out)), expect, "combine")
    # one bf16 rounding of an fp32 sum: within one bf16 ulp of the fp64 value
    assert np.all(np.abs(f64(bits(out)) - expect) <= 2.0 ** -7 * np.abs(expect) + 1e-6)


def test_dispatch_then_combine_k1_is_exact_identity():
    torch = _torch()
    wl = moe_synth.workload("tiny").with_(k=1)
    shape = _shape(wl)
    lg = moe_synth.host_logits(wl)
    ridx, rgate, _ = oracle.route(lg, 1)
    x_np = moe_synth.host_x(wl)
    o = _gpu_dispatch(shape, _bf16_dev(x_np), ridx)
    out = torch.empty((wl.T, wl.d), dtype=torch.bfloat16, device="cuda")
    ws = moe.new_workspace(shape)
    moe.moe_combine(shape, o["x_perm"], o["assign_row"], torch.from_numpy(rgate).cuda(), None, out, ws)
    assert np.array_equal(bits(out), x_np)


# ---------------------------------------------------------------------------
# expert FFN (grouped GEMM)
# ---------------------------------------------------------------------------

def _ffn_case(wl, idx=None):
    torch = _torch()
    shape = _shape(wl)
    x_np = moe_synth.host_x(wl)
    if idx is None:
        idx, _, _ = oracle.route(moe_synth.host_logits(wl), wl.k)
    ref = oracle.dispatch(idx, wl.E, wl.R)
    xp_np = oracle.permute_rows(x_np, ref["row_src"], wl.k)
    w13, w2 = moe_synth.host_w13(wl), moe_synth.host_w2(wl)
    w13s = moe_synth.host_w13s(wl) if wl.n_shared else None
    w2s = moe_synth.host_w2s(wl) if wl.n_shared else None
    y_ref, ys_ref = oracle.expert_ffn(xp_np, ref["expert_offsets"], w13, w2, x_np, w13s, w2s)
    y = torch.empty((shape.A, wl.d), dtype=torch.bfloat16, device="cuda")
    ys = torch.empty((wl.T, wl.d), dtype=torch.bfloat16, device="cuda") if wl.n_shared else None
    ws = moe.new_workspace(shape)
    moe.moe_expert_ffn(shape, _bf16_dev(xp_np), torch.from_numpy(ref["expert_offsets"]).cuda(), _bf16_dev(w13),
                       _bf16_dev(w2), _bf16_dev(x_np) if wl.n_shared else None,
                       _bf16_dev(w13s) if wl.n_shared else None, _bf16_dev(w2s) if wl.n_shared else None, y, ys, ws)
    assert moe.get_status(ws) == 0
    total = ref["expert_offsets"][-1]
    close(f64(bits(y))[:total], y_ref[:total], "y_perm")
    for e in range(wl.E):   # per expert too, so one bad expert cannot hide in the global norm
        r0, r1 = ref["expert_offsets"][e], ref["expert_offsets"][e + 1]
        if r1 > r0:
            close(f64(bits(y))[r0:r1], y_ref[r0:r1], f"y_perm expert {e}")
    if wl.n_shared:
        close(f64(bits(ys)), ys_ref, "y_shared")


@pytest.fixture(params=[moe.GEMM_AUTO, moe.GEMM_SINGLE, moe.GEMM_PAIR],
                ids=["auto_tiles", "single_tiles", "pair_tiles"])
def gemm_policy(request):
    old = moe.set_gemm_policy(request.param)
    yield request.param
    moe.set_gemm_policy(old)


def test_expert_ffn_tiny(gemm_policy):
    _ffn_case(moe_synth.workload("tiny"))


@pytest.mark.parametrize("wl", [
    # skewed: one expert with several m-tiles and a ragged tail, empty experts, shared expert, N=256 down tiles
    moe_synth.Workload("skew", T=300, d=256, E=6, k=2, f=384, R=2, n_shared=1, bias_kind="hot", n_hot=1, beta=3.0),
    # d % 256 != 0: 128-column down tiles
    moe_synth.Workload("d384", T=200, d=384, E=4, k=1, f=256, R=2),
    # one expert, top-1: a dense SwiGLU with a 2-row ragged tail
    moe_synth.Workload("dense", T=130, d=128, E=1, k=1, f=128, R=1),
    # many experts, few rows each (decode-like)
    moe_synth.Workload("decode", T=16, d=256, E=64, k=8, f=256, R=8, n_shared=1, bias_kind="zipf", zipf_s=1.2),
])
def test_expert_ffn_shapes(wl, gemm_policy):
    _ffn_case(wl)


def test_expert_ffn_with_empty_and_full_experts(gemm_policy):
    wl = moe_synth.Workload("emp", T=257, d=128, E=5, k=1, f=256, R=1)
    idx = np.zeros((257, 1), np.int32)
    idx[200:, 0] = 3          # experts 1, 2, 4 empty; expert 0 has 200 rows, expert 3 57
    _ffn_case(wl, idx)


@pytest.mark.parametrize("rows", [1, 15, 16, 17, 31, 32, 33, 63, 96, 127, 128, 129, 240, 255, 256, 257,
                                  383, 384, 385, 512, 513, 700])
def test_expert_ffn_tail_sizes(rows, gemm_policy):
    """Ragged ends of every size class around the 32-row store blocks and the 128/256-row tiles
    (and, for the split schedule, last blocks just under, at and over 128 rows after whole 256-row blocks)."""
    wl = moe_synth.Workload("tail", T=rows + 40, d=256, E=3, k=1, f=256, R=1, n_shared=1)
    idx = np.full((wl.T, 1), 2, np.int32)
    idx[:rows, 0] = 0          # expert 0: `rows` rows, expert 1 empty, expert 2: 40 rows
    _ffn_case(wl, idx)


@pytest.mark.parametrize("name,C", [("mixtral_prefill", 1.0), ("mixtral_prefill", 1.25), ("qwen3_mixed", 1.5),
                                    ("dsv3_skewed_prefill", 1.0), ("tiny", 2.0)])
def test_dispatch_with_capacity_matches_oracle(name, C, dispatch_path):
    wl = moe_synth.workload(name)
    cap = moe.capacity_for(C, wl.T, wl.k, wl.E)
    shape = moe.Shape(T=wl.T, d=wl.d, E=wl.E, k=wl.k, f=wl.f, R=wl.R, capacity=cap)
    ridx, _, _ = oracle.route(moe_synth.host_logits(wl), wl.k)
    ref = oracle.dispatch(ridx, wl.E, wl.R, capacity=cap)
    x_dev = moe_synth.device_inputs(wl, weights=False)["x"]
    o = _gpu_dispatch(shape, x_dev, ridx)
    assert o["status"] == 0
    _check_dispatch(o, ref, moe_synth.host_x(wl) if wl.T * wl.d <= (1 << 24) else None, wl.k)
    assert wl.T * wl.k - int(o["expert_offsets"][-1].item()) == ref["dropped"]


def _ffn_gather_case(wl, idx=None):
    """moe_expert_gate_up_gather (rows of x gathered through row_src) + moe_expert_down against the oracle."""
    torch = _torch()
    shape = _shape(wl)
    x_np = moe_synth.host_x(wl)
    if idx is None:
        idx, _, _ = oracle.route(moe_synth.host_logits(wl), wl.k)
    ref = oracle.dispatch(idx, wl.E, wl.R)
    xp_np = oracle.permute_rows(x_np, ref["row_src"], wl.k)
    w13, w2 = moe_synth.host_w13(wl), moe_synth.host_w2(wl)
    w13s = moe_synth.host_w13s(wl) if wl.n_shared else None
    w2s = moe_synth.host_w2s(wl) if wl.n_shared else None
    y_ref, ys_ref = oracle.expert_ffn(xp_np, ref["expert_offsets"], w13, w2, x_np, w13s, w2s)
    y = torch.empty((shape.A, wl.d), dtype=torch.bfloat16, device="cuda")
    ys = torch.empty((wl.T, wl.d), dtype=torch.bfloat16, device="cuda") if wl.n_shared else None
    ws = moe.new_workspace(shape)
    offs = torch.from_numpy(ref["expert_offsets"]).cuda()
    moe.moe_expert_gate_up_gather(shape, _bf16_dev(x_np), torch.from_numpy(ref["row_src"]).cuda(), offs,
                                  _bf16_dev(w13), _bf16_dev(w13s) if wl.n_shared else None, ws)
    moe.moe_expert_down(shape, offs, _bf16_dev(w2), _bf16_dev(w2s) if wl.n_shared else None, y, ys, ws)
    assert moe.get_status(ws) == 0
    total = ref["expert_offsets"][-1]
    for e in range(wl.E):
        r0, r1 = ref["expert_offsets"][e], ref["expert_offsets"][e + 1]
        if r1 > r0:
            close(f64(bits(y))[r0:r1], y_ref[r0:r1], f"y_perm expert {e} (gathered rows)")
    close(f64(bits(y))[:total], y_ref[:total], "y_perm (gathered rows)")
    if wl.n_shared:
        close(f64(bits(ys)), ys_ref, "y_shared")


@pytest.mark.parametrize("wl", [
    moe_synth.workload("tiny"),
    moe_synth.Workload("skew", T=300, d=256, E=6, k=2, f=384, R=2, n_shared=1, bias_kind="hot", n_hot=1, beta=3.0),
    moe_synth.Workload("decode", T=16, d=256, E=64, k=8, f=256, R=8, n_shared=1, bias_kind="zipf", zipf_s=1.2),
    moe_synth.Workload("d384", T=200, d=384, E=4, k=1, f=256, R=2),
])
def test_expert_ffn_gathering_rows_from_x(wl, gemm_policy):
    _ffn_gather_case(wl)


def test_index_only_dispatch_equals_full_dispatch(dispatch_path):
    torch = _torch()
    wl = moe_synth.workload("qwen3_mixed")
    shape = _shape(wl)
    ridx, _, _ = oracle.route(moe_synth.host_logits(wl), wl.k)
    full = _gpu_dispatch(shape, moe_synth.device_inputs(wl, weights=False)["x"], ridx)
    i32 = torch.int32
    o = {n: torch.full_like(full[n], -9) for n in ("expert_counts", "expert_offsets", "rank_counts", "rank_offsets",
                                                     "row_src", "assign_row", "imbalance")}
    ws = moe.new_workspace(shape)
    moe.moe_dispatch(shape, None, torch.from_numpy(ridx).cuda(), o["expert_counts"], o["expert_offsets"],
                     o["rank_counts"], o["rank_offsets"], o["row_src"], o["assign_row"], None, o["imbalance"], ws)
    assert moe.get_status(ws) == 0
    for n, t in o.items():
        assert torch.equal(t, full[n]), n


def test_gathering_gemm_reports_a_row_index_out_of_range():
    """A row_src entry past T*k is read as token 0 and raises MOE_DEV_BOUNDS (checked in the kernel)."""
    torch = _torch()
    wl = moe_synth.workload("tiny")
    shape = _shape(wl)
    idx, _, _ = oracle.route(moe_synth.host_logits(wl), wl.k)
    ref = oracle.dispatch(idx, wl.E, wl.R)
    row_src = ref["row_src"].copy()
    row_src[5] = shape.A + 1000
    ws = moe.new_workspace(shape)
    moe.moe_expert_gate_up_gather(shape, _bf16_dev(moe_synth.host_x(wl)), torch.from_numpy(row_src).cuda(),
                                  torch.from_numpy(ref["expert_offsets"]).cuda(), _bf16_dev(moe_synth.host_w13(wl)),
                                  None, ws)
    assert moe.get_status(ws) == moe.MOE_DEV_BOUNDS


def _random_dispatch_cases(n=24, seed=2024):
    rng = np.random.default_rng(seed)
    cases = []
    for _ in range(n):
        E = int(rng.integers(1, 257))
        k = int(rng.integers(1, min(E, 8) + 1))
        divisors = [r for r in range(1, min(E, 16) + 1) if E % r == 0]
        R = int(rng.choice(divisors))
        T = int(rng.integers(0, 5000))
        cap = int(rng.integers(1, max(2, T * k // E * 2))) if rng.random() < 0.4 and T else 0
        cases.append((T, E, k, R, cap, int(rng.integers(0, 2**31 - 1))))
    return cases


@pytest.mark.parametrize("T,E,k,R,cap,seed", _random_dispatch_cases())
def test_dispatch_random_shapes_bit_exact(T, E, k, R, cap, seed, dispatch_path):
    """Seeded random shapes (chunk boundaries, many or few experts, capacity drops) against the oracle."""
    torch = _torch()
    rng = np.random.default_rng(seed)
    idx = np.array([rng.permutation(E)[:k] for _ in range(T)], np.int32).reshape(T, k)
    shape = moe.Shape(T=T, d=128, E=E, k=k, f=128, R=R, capacity=cap)
    x_np = rng.integers(0, 1 << 16, size=(T, 128), dtype=np.uint64).astype(np.uint16)
    x_dev = torch.from_numpy(x_np.view(np.int16)).cuda().view(torch.bfloat16) if T else \
        torch.empty((0, 128), dtype=torch.bfloat16, device="cuda")
    o = _gpu_dispatch(shape, x_dev, idx)
    assert o["status"] == 0
    ref = oracle.dispatch(idx, E, R, capacity=cap)
    _check_dispatch(o, ref, x_np, k)
