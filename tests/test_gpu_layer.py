"""The whole layer (moe_layer) against the oracle, at oracle-sized and full sizes.

Full sizes (the workloads the benchmark times): inputs are filled on the device
by the seeded generator; routing, counts, offsets, permutation and imbalance are
compared bit for bit with the oracle over the whole batch, x_perm by a property
that holds at any size, and the floating-point outputs (out, y_perm rows) on a
sample of tokens that the oracle computes one by one from host-regenerated
inputs (only the sampled tokens' experts' weights are regenerated).
"""
import numpy as np
import pytest

import combine_warp_top_expert_b200 as moe
import moe_synth
import oracle
from parity_util import GATE_TOL, bits, close, f64, np_i32

pytestmark = pytest.mark.gpu


def _shape(wl):
    return moe.Shape(T=wl.T, d=wl.d, E=wl.E, k=wl.k, f=wl.f, R=wl.R, n_shared=wl.n_shared)


def _run_layer(wl):
    dv = moe_synth.device_inputs(wl)
    layer = moe.MoELayer(_shape(wl), dv["w13"], dv["w2"], dv.get("w13s"), dv.get("w2s"))
    outs = layer(dv["logits"], dv["x"])
    status = moe.get_status(layer.ws)
    return dv, layer, outs, status


def _check_routing(wl, outs):
    lg = moe_synth.host_logits(wl)
    ridx, rgate, _ = oracle.route(lg, wl.k)
    assert np.array_equal(np_i32(outs["topk_idx"]), ridx)
    assert np.max(np.abs(outs["topk_gate"].cpu().numpy().astype(np.float64) - rgate)) <= GATE_TOL
    ref = oracle.dispatch(ridx, wl.E, wl.R)
    for n in ("expert_counts", "expert_offsets", "rank_counts", "rank_offsets", "row_src", "assign_row"):
        assert np.array_equal(np_i32(outs[n]), ref[n]), n
    assert np.array_equal(outs["imbalance"].cpu().numpy().view(np.uint32), ref["imbalance"].view(np.uint32))
    return ridx, rgate, ref


def test_layer_tiny_full_parity():
    wl = moe_synth.workload("tiny")
    dv, layer, outs, status = _run_layer(wl)
    assert status == 0
    _check_routing(wl, outs)
    res = oracle.layer(moe_synth.host_x(wl), moe_synth.host_logits(wl), moe_synth.host_w13(wl),
                       moe_synth.host_w2(wl), wl.k, wl.R)
    assert np.array_equal(bits(outs["x_perm"]), res["x_perm"])
    close(f64(bits(outs["y_perm"])), res["y_perm"], "y_perm")
    close(f64(bits(outs["out"])), res["out"], "out")


def test_layer_with_shared_expert_full_parity():
    wl = moe_synth.Workload("sh", T=200, d=256, E=16, k=4, f=256, R=4, n_shared=1, bias_kind="zipf", zipf_s=1.0)
    dv, layer, outs, status = _run_layer(wl)
    assert status == 0
    _check_routing(wl, outs)
    res = oracle.layer(moe_synth.host_x(wl), moe_synth.host_logits(wl), moe_synth.host_w13(wl),
                       moe_synth.host_w2(wl), wl.k, wl.R, moe_synth.host_w13s(wl), moe_synth.host_w2s(wl))
    close(f64(bits(outs["y_shared"])), res["y_shared"], "y_shared")
    close(f64(bits(outs["out"])), res["out"], "out")


def test_layer_is_deterministic_across_calls():
    import torch
    wl = moe_synth.workload("tiny")
    dv, layer, outs, status = _run_layer(wl)
    first = {n: outs[n].clone() for n in ("x_perm", "y_perm", "out", "row_src", "topk_gate")}
    layer(dv["logits"], dv["x"])
    for n, t in first.items():
        a, b = t, layer.outs[n]
        if a.dtype == torch.bfloat16:
            a, b = a.view(torch.int16), b.view(torch.int16)
        assert torch.equal(a, b), n


def _sampled_parity(wl, outs, ridx, rgate, ref, n_tokens, seed=0):
    toks = np.sort(np.random.default_rng(seed).choice(wl.T, n_tokens, replace=False))
    x_rows = moe_synth.host_x(wl, toks)
    out_gpu = f64(bits(outs["out"][toks]))
    y_perm_gpu = outs["y_perm"]
    want = np.zeros((len(toks), wl.d))
    experts = sorted(set(ridx[toks].reshape(-1).tolist()))
    import torch
    for e in experts:
        sel = [(i, j) for i, t in enumerate(toks) for j in range(wl.k) if ridx[t, j] == e]
        y = oracle.swiglu(x_rows[[i for i, _ in sel]], moe_synth.host_w13(wl, e), moe_synth.host_w2(wl, e))
        rows = [ref["assign_row"][toks[i] * wl.k + j] for i, j in sel]
        close(f64(bits(y_perm_gpu[torch.tensor(rows, device="cuda").long()])), y, f"y_perm expert {e}")
        for (i, j), yr in zip(sel, y):
            want[i] += float(rgate[toks[i], j]) * yr
    if wl.n_shared:
        ys = oracle.swiglu(x_rows, moe_synth.host_w13s(wl), moe_synth.host_w2s(wl))
        close(f64(bits(outs["y_shared"][toks])), ys, "y_shared")
        want += ys
    close(out_gpu, want, "out")


@pytest.mark.parametrize("name,n_tokens", [("mixtral_prefill", 6), ("dsv3_decode", 6), ("qwen3_mixed", 8),
                                           ("dsv3_skewed_prefill", 3)])
def test_layer_full_size_sampled_parity(name, n_tokens):
    import torch
    wl = moe_synth.workload(name)
    dv, layer, outs, status = _run_layer(wl)
    assert status == 0
    ridx, rgate, ref = _check_routing(wl, outs)
    # x_perm: every assignment's row equals its token's row (any size)
    rows = torch.from_numpy(ref["assign_row"]).cuda().long()
    a = torch.arange(wl.T * wl.k, device="cuda")
    for c in torch.split(a, 1 << 14):
        assert torch.equal(outs["x_perm"].view(torch.int16)[rows[c]], dv["x"].view(torch.int16)[c // wl.k])
    assert torch.isfinite(outs["out"].float()).all()
    _sampled_parity(wl, outs, ridx, rgate, ref, n_tokens)
    del layer, outs, dv
    torch.cuda.empty_cache()


@pytest.mark.parametrize("policy", [moe.GEMM_SINGLE, moe.GEMM_PAIR], ids=["single_tiles", "pair_tiles"])
def test_layer_mixtral_sampled_parity_other_tiles(policy):
    old = moe.set_gemm_policy(policy)
    try:
        test_layer_full_size_sampled_parity("mixtral_prefill", 4)
    finally:
        moe.set_gemm_policy(old)


def test_layer_skewed_prefill_sampled_parity_pair_tiles():
    """Pair tiles on the skewed prefill: cold experts (~285 rows) end in half-height tiles, hot ones and the
    shared expert in full ones."""
    old = moe.set_gemm_policy(moe.GEMM_PAIR)
    try:
        test_layer_full_size_sampled_parity("dsv3_skewed_prefill", 3)
    finally:
        moe.set_gemm_policy(old)


def test_empty_batch_is_a_no_op():
    wl = moe_synth.workload("tiny").with_(T=0)
    dv, layer, outs, status = _run_layer(wl)
    assert status == 0
    assert np.all(np_i32(outs["expert_counts"]) == 0)
    assert outs["imbalance"].cpu().numpy().tolist() == [1.0, 1.0]


def test_inconsistent_offsets_are_reported_not_hung():
    import torch
    wl = moe_synth.workload("tiny")
    shape = _shape(wl)
    dv = moe_synth.device_inputs(wl)
    offs = torch.tensor([0, 100, 50, 300, 400, 450, 500, 510, 512], dtype=torch.int32, device="cuda")  # decreasing
    y = torch.zeros((shape.A, wl.d), dtype=torch.bfloat16, device="cuda")
    ws = moe.new_workspace(shape)
    xp = torch.zeros((shape.A, wl.d), dtype=torch.bfloat16, device="cuda")
    moe.moe_expert_ffn(shape, xp, offs, dv["w13"], dv["w2"], None, None, None, y, None, ws)
    assert moe.get_status(ws) & moe.MOE_DEV_COUNT_MISMATCH
    # the context stays usable
    dv2, layer, outs, status = _run_layer(wl)
    assert status == 0


def test_host_buffer_calls_overlap_and_match_device_calls():
    """forward_host (host tensors; copies on side streams, two rotating staging
    slots) gives each batch exactly the result of a device call, across calls in a
    row whose copies overlap each other's compute."""
    import torch
    old = moe.set_gemm_policy(moe.GEMM_SINGLE)
    try:
        wl = moe_synth.workload("tiny")
        batches = [moe_synth.device_inputs(wl.with_(seed=s), weights=(s == 0)) for s in range(3)]
        dv = batches[0]
        layer = moe.MoELayer(_shape(wl), dv["w13"], dv["w2"])
        want = []
        for b in batches:
            want.append(layer(b["logits"], b["x"])["out"].clone())
        hosts = [(b["logits"].cpu().pin_memory(), b["x"].cpu().pin_memory(),
                  torch.zeros((wl.T, wl.d), dtype=torch.bfloat16).pin_memory()) for b in batches]
        for lg_h, x_h, out_h in hosts:
            layer.forward_host(lg_h, x_h, out_h)
        torch.cuda.synchronize()
        for (_, _, out_h), w in zip(hosts, want):
            assert torch.equal(out_h.view(torch.int16), w.cpu().view(torch.int16))
    finally:
        moe.set_gemm_policy(old)


def test_layer_with_capacity_matches_oracle():
    import torch
    wl = moe_synth.Workload("capl", T=300, d=256, E=8, k=2, f=256, R=4, bias_kind="zipf", zipf_s=1.0)
    cap = moe.capacity_for(1.25, wl.T, wl.k, wl.E)
    shape = moe.Shape(T=wl.T, d=wl.d, E=wl.E, k=wl.k, f=wl.f, R=wl.R, capacity=cap)
    dv = moe_synth.device_inputs(wl)
    layer = moe.MoELayer(shape, dv["w13"], dv["w2"])
    outs = layer(dv["logits"], dv["x"])
    assert moe.get_status(layer.ws) == 0
    res = oracle.layer(moe_synth.host_x(wl), moe_synth.host_logits(wl), moe_synth.host_w13(wl),
                       moe_synth.host_w2(wl), wl.k, wl.R, capacity=cap)
    assert res["dropped"] > 0
    for n in ("expert_counts", "expert_offsets", "row_src", "assign_row"):
        assert np.array_equal(np_i32(outs[n]), res[n]), n
    close(f64(bits(outs["out"])), res["out"], "out with capacity")


def _run_layer_gather(wl, capacity=0):
    dv = moe_synth.device_inputs(wl)
    shape = moe.Shape(T=wl.T, d=wl.d, E=wl.E, k=wl.k, f=wl.f, R=wl.R, n_shared=wl.n_shared, capacity=capacity)
    layer = moe.MoELayer(shape, dv["w13"], dv["w2"], dv.get("w13s"), dv.get("w2s"), gather=True)
    outs = layer(dv["logits"], dv["x"])
    return dv, layer, outs, moe.get_status(layer.ws)


def test_layer_gathering_rows_full_parity():
    """x_perm not materialised: the grouped GEMM gathers the dispatched rows of x itself."""
    wl = moe_synth.Workload("gsh", T=200, d=256, E=16, k=4, f=256, R=4, n_shared=1, bias_kind="zipf", zipf_s=1.0)
    dv, layer, outs, status = _run_layer_gather(wl)
    assert status == 0 and outs["x_perm"] is None
    _check_routing(wl, outs)
    res = oracle.layer(moe_synth.host_x(wl), moe_synth.host_logits(wl), moe_synth.host_w13(wl),
                       moe_synth.host_w2(wl), wl.k, wl.R, moe_synth.host_w13s(wl), moe_synth.host_w2s(wl))
    close(f64(bits(outs["y_perm"])), res["y_perm"], "y_perm")
    close(f64(bits(outs["out"])), res["out"], "out")


@pytest.mark.parametrize("name,n_tokens", [("mixtral_prefill", 4), ("dsv3_skewed_prefill", 2), ("dsv3_decode", 4)])
def test_layer_gathering_rows_full_size_sampled(name, n_tokens):
    import torch
    wl = moe_synth.workload(name)
    dv, layer, outs, status = _run_layer_gather(wl)
    assert status == 0
    ridx, rgate, ref = _check_routing(wl, outs)
    _sampled_parity(wl, outs, ridx, rgate, ref, n_tokens, seed=3)
    del layer, outs, dv
    torch.cuda.empty_cache()


@pytest.mark.parametrize("name", ["qwen3_mixed", "dsv3_decode"])
def test_layer_gathering_rows_is_bit_identical_to_materialised_x_perm(name):
    """Same A rows, same MMA order: the gathering GEMM changes where rows come from, not the arithmetic."""
    import torch
    wl = moe_synth.workload(name)
    dv = moe_synth.device_inputs(wl)
    shape = moe.Shape(T=wl.T, d=wl.d, E=wl.E, k=wl.k, f=wl.f, R=wl.R, n_shared=wl.n_shared)
    a = moe.MoELayer(shape, dv["w13"], dv["w2"], dv.get("w13s"), dv.get("w2s"))(dv["logits"], dv["x"])
    b = moe.MoELayer(shape, dv["w13"], dv["w2"], dv.get("w13s"), dv.get("w2s"), gather=True)(dv["logits"], dv["x"])
    for n in ("row_src", "assign_row", "expert_offsets", "y_perm", "out"):
        assert torch.equal(a[n], b[n]), n


def test_layer_gathering_rows_with_capacity_matches_oracle():
    wl = moe_synth.Workload("capg", T=300, d=256, E=8, k=2, f=256, R=4, n_shared=1, bias_kind="zipf", zipf_s=1.0)
    cap = moe.capacity_for(1.25, wl.T, wl.k, wl.E)
    dv, layer, outs, status = _run_layer_gather(wl, capacity=cap)
    assert status == 0
    res = oracle.layer(moe_synth.host_x(wl), moe_synth.host_logits(wl), moe_synth.host_w13(wl),
                       moe_synth.host_w2(wl), wl.k, wl.R, moe_synth.host_w13s(wl), moe_synth.host_w2s(wl),
                       capacity=cap)
    assert res["dropped"] > 0
    for n in ("expert_counts", "expert_offsets", "row_src", "assign_row"):
        assert np.array_equal(np_i32(outs[n]), res[n]), n
    close(f64(bits(outs["out"])), res["out"], "out with capacity, gathered rows")


def _random_layer_cases(n=12, seed=77):
    rng = np.random.default_rng(seed)
    cases = []
    for i in range(n):
        E = int(rng.integers(1, 33))
        k = int(rng.integers(1, min(E, 8) + 1))
        R = int(rng.choice([r for r in range(1, E + 1) if E % r == 0]))
        T = int(rng.integers(1, 400))
        d = int(rng.choice([128, 256, 384, 512]))
        f = int(rng.choice([128, 256, 384]))
        n_shared = int(rng.integers(0, 2))
        cf = float(rng.choice([0.0, 0.0, 1.0, 1.5]))
        wl = moe_synth.Workload(f"rnd{i}", T=T, d=d, E=E, k=k, f=f, R=R, n_shared=n_shared, bias_kind="zipf",
                                zipf_s=float(rng.uniform(0.0, 1.5)), seed=i + 1)
        cases.append((wl, cf))
    return cases


@pytest.mark.parametrize("policy", [moe.GEMM_AUTO, moe.GEMM_SINGLE, moe.GEMM_PAIR], ids=["auto", "single", "pair"])
@pytest.mark.parametrize("wl,cf", _random_layer_cases(), ids=[c[0].name for c in _random_layer_cases()])
def test_layer_random_shapes_match_oracle(wl, cf, policy):
    """Seeded random shapes through the whole layer, under each tile policy, against the oracle
    (ragged groups of every size exercise the short A boxes of single-CTA tiles and the
    half-height pair tiles)."""
    cap = moe.capacity_for(cf, wl.T, wl.k, wl.E) if cf else 0
    shape = moe.Shape(T=wl.T, d=wl.d, E=wl.E, k=wl.k, f=wl.f, R=wl.R, n_shared=wl.n_shared, capacity=cap)
    dv = moe_synth.device_inputs(wl)
    old = moe.set_gemm_policy(policy)
    try:
        layer = moe.MoELayer(shape, dv["w13"], dv["w2"], dv.get("w13s"), dv.get("w2s"))
        outs = layer(dv["logits"], dv["x"])
        assert moe.get_status(layer.ws) == 0
    finally:
        moe.set_gemm_policy(old)
    res = oracle.layer(moe_synth.host_x(wl), moe_synth.host_logits(wl), moe_synth.host_w13(wl),
                       moe_synth.host_w2(wl), wl.k, wl.R, moe_synth.host_w13s(wl) if wl.n_shared else None,
                       moe_synth.host_w2s(wl) if wl.n_shared else None, capacity=cap)
    assert np.array_equal(np_i32(outs["topk_idx"]), res["topk_idx"])
    for n in ("expert_counts", "expert_offsets", "rank_counts", "rank_offsets", "row_src", "assign_row"):
        assert np.array_equal(np_i32(outs[n]), res[n]), n
    close(f64(bits(outs["out"])), res["out"], f"out {wl.name}")


@pytest.mark.parametrize("name", ["tiny", "qwen3_mixed", "dsv3_decode"])
def test_layer_is_bit_identical_with_and_without_launch_overlap(name):
    """Programmatic dependent launch changes when kernels start, not what they compute:
    every output of moe_layer, and of the five entry points called one by one, is bit for
    bit the same with the overlap on and off, over two calls in a row."""
    import torch
    wl = moe_synth.workload(name)
    dv = moe_synth.device_inputs(wl)
    shape = _shape(wl)
    names = ("topk_idx", "topk_gate", "expert_offsets", "row_src", "assign_row", "x_perm", "y_perm", "out",
             "imbalance")
    results = {}
    old = moe.set_pdl(True)
    try:
        for pdl in (True, False):
            moe.set_pdl(pdl)
            layer = moe.MoELayer(shape, dv["w13"], dv["w2"], dv.get("w13s"), dv.get("w2s"))
            for _ in range(2):
                outs = layer(dv["logits"], dv["x"])
            assert moe.get_status(layer.ws) == 0
            results[pdl] = {n: outs[n].clone() for n in names}
            o, ws = layer.outs, layer.ws
            moe.moe_route(shape, dv["logits"], o["topk_idx"], o["topk_gate"], ws)
            moe.moe_dispatch(shape, dv["x"], o["topk_idx"], o["expert_counts"], o["expert_offsets"],
                             o["rank_counts"], o["rank_offsets"], o["row_src"], o["assign_row"], o["x_perm"],
                             o["imbalance"], ws)
            moe.moe_expert_ffn(shape, o["x_perm"], o["expert_offsets"], dv["w13"], dv["w2"], dv["x"], dv.get("w13s"),
                               dv.get("w2s"), o["y_perm"], o.get("y_shared"), ws)
            moe.moe_combine(shape, o["y_perm"], o["assign_row"], o["topk_gate"], o.get("y_shared"), o["out"], ws)
            assert moe.get_status(ws) == 0
            for n in names:
                a, b = results[pdl][n], o[n]
                if a.dtype == torch.bfloat16:
                    a, b = a.view(torch.int16), b.view(torch.int16)
                assert torch.equal(a, b), (pdl, n)
    finally:
        moe.set_pdl(old)
    for n in names:
        a, b = results[True][n], results[False][n]
        if a.dtype == torch.bfloat16:
            a, b = a.view(torch.int16), b.view(torch.int16)
        assert torch.equal(a, b), n


@pytest.mark.parametrize("name", ["tiny", "qwen3_mixed", "dsv3_decode", "mixtral_prefill"])
def test_layer_is_bit_identical_on_both_dispatch_paths(name):
    """The one-pass dispatch kernel (which, inside moe_layer, loads rows of x before its
    wait on the router) and the two-kernel path place the same rows: every output of
    moe_layer is bit for bit the same, over two calls in a row, with the launch overlap
    on and off."""
    import torch
    wl = moe_synth.workload(name)
    dv = moe_synth.device_inputs(wl)
    shape = _shape(wl)
    names = ("topk_idx", "topk_gate", "expert_counts", "expert_offsets", "rank_counts", "rank_offsets", "row_src",
             "assign_row", "x_perm", "y_perm", "out", "imbalance")
    results = {}
    old_path, old_pdl = moe.set_dispatch_path(moe.DISPATCH_AUTO), moe.set_pdl(True)
    try:
        for path in (moe.DISPATCH_TWO_PASS, moe.DISPATCH_ONE_PASS):
            for pdl in (True, False):
                moe.set_dispatch_path(path)
                moe.set_pdl(pdl)
                layer = moe.MoELayer(shape, dv["w13"], dv["w2"], dv.get("w13s"), dv.get("w2s"))
                for _ in range(2):
                    outs = layer(dv["logits"], dv["x"])
                assert moe.get_status(layer.ws) == 0
                results[(path, pdl)] = {n: outs[n].clone() for n in names}
    finally:
        moe.set_dispatch_path(old_path)
        moe.set_pdl(old_pdl)
    base = results[(moe.DISPATCH_TWO_PASS, True)]
    for key, res in results.items():
        for n in names:
            a, b = base[n], res[n]
            if a.dtype == torch.bfloat16:
                a, b = a.view(torch.int16), b.view(torch.int16)
            assert torch.equal(a, b), (key, n)


@pytest.mark.parametrize("policy", [moe.GEMM_SINGLE, moe.GEMM_PAIR], ids=["single", "pair"])
@pytest.mark.parametrize("fused", [False, True], ids=["combine", "fused_combine"])
def test_stale_workspace_contents_never_reach_a_result(policy, fused):
    """Padding rows of h, the rows a short A box leaves in a pipeline stage, and every other
    scratch row past a group's real rows are computed on but never stored as results. With
    everything in the workspace past its 256-byte header (which holds the zeroed counters)
    set to 0xFF bytes (NaN in every bf16 of h) the layer gives the same bits as on a zeroed
    workspace, two calls in a row, on a batch of many one-tile groups and a few long ones."""
    import torch
    wl = moe_synth.Workload("stale", T=320, d=512, E=48, k=6, f=384, R=4, n_shared=1, bias_kind="zipf",
                            zipf_s=1.3, seed=31)
    shape = _shape(wl)
    dv = moe_synth.device_inputs(wl)
    names = ("topk_idx", "topk_gate", "expert_offsets", "row_src", "assign_row", "x_perm", "y_perm", "y_shared",
             "out")
    old_p, old_f = moe.set_gemm_policy(policy), moe.set_fused_combine(fused)
    try:
        results = []
        for fill in (0x00, 0xFF):
            layer = moe.MoELayer(shape, dv["w13"], dv["w2"], dv["w13s"], dv["w2s"])
            layer.ws[256:].fill_(fill)
            for _ in range(2):
                outs = layer(dv["logits"], dv["x"])
            torch.cuda.synchronize()
            assert moe.get_status(layer.ws) == 0
            results.append({n: outs[n].clone() for n in names})
    finally:
        moe.set_gemm_policy(old_p)
        moe.set_fused_combine(old_f)
    A = int(results[0]["expert_offsets"][-1])
    for n in names:
        a, b = results[0][n], results[1][n]
        if n in ("x_perm", "y_perm"):
            a, b = a[:A], b[:A]
        if a.dtype == torch.bfloat16:
            assert not torch.isnan(b.float()).any(), n
            a, b = a.view(torch.int16), b.view(torch.int16)
        assert torch.equal(a, b), n


def test_the_launch_counter_counts_each_kernel_of_a_layer_call():
    """moe_kernel_launches (the bench's `gpu_launches`): one moe_layer call launches route,
    dispatch (one kernel for T*k <= 16384, else histogram + permute), gate/up, down and
    combine; with the combine folded into the down GEMM the combine kernel is not launched
    (and dispatch takes its two-kernel form)."""
    import torch
    wl = moe_synth.workload("tiny")
    dv = moe_synth.device_inputs(wl)
    layer = moe.MoELayer(_shape(wl), dv["w13"], dv["w2"])
    cases = [(moe.DISPATCH_AUTO, False, 5), (moe.DISPATCH_ONE_PASS, False, 5), (moe.DISPATCH_TWO_PASS, False, 6),
             (moe.DISPATCH_AUTO, True, 5)]
    old_p, old_f = moe.set_dispatch_path(moe.DISPATCH_AUTO), moe.set_fused_combine(False)
    try:
        for path, fused, want in cases:
            moe.set_dispatch_path(path)
            moe.set_fused_combine(fused)
            before = moe.kernel_launches()
            layer(dv["logits"], dv["x"])
            assert moe.kernel_launches() - before == want, (path, fused)
        torch.cuda.synchronize()
        assert moe.get_status(layer.ws) == 0
    finally:
        moe.set_dispatch_path(old_p)
        moe.set_fused_combine(old_f)


def _soak_cases(n=40, seed=2026):
    """Seeded random layers, each with a random tile policy, dispatch path and combine form."""
    rng = np.random.default_rng(seed)
    cases = []
    for i in range(n):
        E = int(rng.integers(1, 65))
        k = int(rng.integers(1, min(E, 8) + 1))
        R = int(rng.choice([r for r in range(1, E + 1) if E % r == 0]))
        wl = moe_synth.Workload(f"soak{i}", T=int(rng.integers(1, 1500)), d=int(rng.choice([128, 256, 384, 512, 768])),
                                E=E, k=k, f=int(rng.choice([128, 256, 384, 512])), R=R,
                                n_shared=int(rng.integers(0, 2)), bias_kind="zipf",
                                zipf_s=float(rng.uniform(0.0, 1.6)), seed=5000 + i)
        cases.append((wl, float(rng.choice([0.0, 0.0, 1.0, 1.25, 2.0])), int(rng.choice([0, 1, 2])),
                      int(rng.choice([0, 1, 2])), bool(rng.integers(0, 2))))
    return cases


@pytest.mark.parametrize("wl,cf,policy,path,fused", _soak_cases(), ids=[c[0].name for c in _soak_cases()])
def test_layer_random_configurations_against_oracle(wl, cf, policy, path, fused):
    """Random shape x tile policy x dispatch path x combine form, on a workspace whose scratch
    starts as 0xFF bytes: indices bit-exact, `out` within tolerance of the oracle."""
    cap = moe.capacity_for(cf, wl.T, wl.k, wl.E) if cf else 0
    shape = moe.Shape(T=wl.T, d=wl.d, E=wl.E, k=wl.k, f=wl.f, R=wl.R, n_shared=wl.n_shared, capacity=cap)
    dv = moe_synth.device_inputs(wl)
    old = (moe.set_gemm_policy(policy), moe.set_dispatch_path(path), moe.set_fused_combine(fused))
    try:
        layer = moe.MoELayer(shape, dv["w13"], dv["w2"], dv.get("w13s"), dv.get("w2s"))
        layer.ws[256:].fill_(0xFF)
        outs = layer(dv["logits"], dv["x"])
        assert moe.get_status(layer.ws) == 0
    finally:
        moe.set_gemm_policy(old[0])
        moe.set_dispatch_path(old[1])
        moe.set_fused_combine(old[2])
    res = oracle.layer(moe_synth.host_x(wl), moe_synth.host_logits(wl), moe_synth.host_w13(wl),
                       moe_synth.host_w2(wl), wl.k, wl.R, moe_synth.host_w13s(wl) if wl.n_shared else None,
                       moe_synth.host_w2s(wl) if wl.n_shared else None, capacity=cap)
    assert np.array_equal(np_i32(outs["topk_idx"]), res["topk_idx"])
    for n in ("expert_counts", "expert_offsets", "rank_counts", "rank_offsets", "row_src", "assign_row"):
        assert np.array_equal(np_i32(outs[n]), res[n]), n
    close(f64(bits(outs["out"])), res["out"], f"out {wl.name}")
