"""Pins of the CPU oracle against things other than itself (no GPU).

Each test ties one oracle function to the page ("Expert Parallelism" tutorial,
learning-materials IX.05), to mathematics (brute force, closed forms,
invariants) or to an independent library computation (numpy dense SwiGLU), so
that a dropped term, a wrong sign or index, or a transposed operand anywhere in
the oracle fails at least one of them.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest

import moe_synth
import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _bf16(a):
    """fp32 -> bf16 bits (round to nearest even), test-side helper."""
    u = np.ascontiguousarray(a, np.float32).view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return u.astype(np.uint16)


def _f(b):
    return moe_synth.bf16_to_f32(b).astype(np.float64)


# ---------------------------------------------------------------------------
# router: top-k by brute force over ordered k-tuples (§1, §4 "Router output")
# ---------------------------------------------------------------------------

def _brute_topk(l, k):
    """Largest ordered k-tuple of distinct experts under (logit desc, index asc)."""
    best, best_key = None, None
    for tup in itertools.permutations(range(len(l)), k):
        key = tuple((l[e], -e) for e in tup)
        if best_key is None or key > best_key:
            best, best_key = tup, key
    return list(best)


@pytest.mark.parametrize("E,k", [(3, 1), (4, 2), (5, 3), (6, 2), (7, 4), (6, 6)])
def test_topk_matches_bruteforce_with_ties(E, k):
    rng = np.random.default_rng(100 + E * 10 + k)
    logits = rng.integers(-2, 3, size=(64, E)).astype(np.float32)  # many exact ties
    idx, _, nan = oracle.route(logits, k)
    assert nan == 0
    for t in range(logits.shape[0]):
        assert list(idx[t]) == _brute_topk([float(v) for v in logits[t]], k), t


def test_topk_signed_zero_ties_go_to_lower_index():
    for row in ([-0.0, 0.0, -1.0], [0.0, -0.0, -1.0]):
        idx, gate, _ = oracle.route(np.array([row], np.float32), 2)
        assert list(idx[0]) == [0, 1]
        assert gate[0, 0] == np.float32(0.5) and gate[0, 1] == np.float32(0.5)


def test_topk_matches_python_sort_on_arbitrary_floats():
    """Any float32 logits, special values mixed in (signed zeros, infinities, NaN,
    subnormals, the largest finite values): the selection equals Python's own sort by
    (logit descending with NaN as -inf, index ascending), and the NaN count is exact."""
    from hypothesis import given, settings, strategies as st

    special = st.sampled_from([0.0, -0.0, float("inf"), float("-inf"), float("nan"), 1e-45, -1e-45,
                               3.4028234663852886e38, -3.4028234663852886e38, 1.0, -1.0])
    value = st.one_of(st.floats(width=32), special)

    @st.composite
    def case(draw):
        E = draw(st.integers(1, 40))
        k = draw(st.integers(1, min(E, 8)))
        T = draw(st.integers(0, 5))
        return k, np.array([[draw(value) for _ in range(E)] for _ in range(T)], np.float32).reshape(T, E)

    @settings(max_examples=120, deadline=None)
    @given(case())
    def check(c):
        k, lg = c
        T, E = lg.shape
        idx, _, nan = oracle.route(lg, k)
        assert nan == int(np.isnan(lg).sum())
        for t in range(T):
            key = [float("-inf") if np.isnan(v) else float(v) for v in lg[t]]
            want = sorted(range(E), key=lambda e: (-key[e], e))[:k]
            assert list(idx[t]) == want, (lg[t], list(idx[t]), want)

    check()


def test_topk_nan_orders_as_minus_inf_and_is_counted():
    lg = np.array([[np.nan, 1.0, 0.5, -3.0]], np.float32)
    idx, _, nan = oracle.route(lg, 3)
    assert list(idx[0]) == [1, 2, 3] and nan == 1
    idx, gate, nan = oracle.route(np.full((1, 4), -np.inf, np.float32), 2)
    assert list(idx[0]) == [0, 1] and np.all(gate == np.float32(0.5))


# ---------------------------------------------------------------------------
# gates: closed forms and invariants
# ---------------------------------------------------------------------------

def test_gate_k1_is_exactly_one():
    lg = np.random.default_rng(1).normal(size=(200, 16)).astype(np.float32)
    _, gate, _ = oracle.route(lg, 1)
    assert np.all(gate == np.float32(1.0))


def test_gate_k2_is_logistic_of_logit_gap():
    lg = np.random.default_rng(2).normal(scale=3.0, size=(500, 9)).astype(np.float32)
    idx, gate, _ = oracle.route(lg, 2)
    l0 = lg[np.arange(500), idx[:, 0]].astype(np.float64)
    l1 = lg[np.arange(500), idx[:, 1]].astype(np.float64)
    g0 = 1.0 / (1.0 + np.exp(l1 - l0))  # two-way softmax == logistic of the gap
    assert np.max(np.abs(gate[:, 0] - g0)) <= 2.0 ** -24
    assert np.max(np.abs(gate[:, 1] - (1.0 - g0))) <= 2.0 ** -24


def test_gates_sum_to_one_and_are_non_increasing():
    lg = np.random.default_rng(3).normal(size=(300, 64)).astype(np.float32)
    _, gate, _ = oracle.route(lg, 8)
    assert np.max(np.abs(gate.astype(np.float64).sum(1) - 1.0)) <= 2.0 ** -22
    assert np.all(np.diff(gate, axis=1) <= 0)


# ---------------------------------------------------------------------------
# dispatch: the page's worked imbalance example (§5) and counting invariants
# ---------------------------------------------------------------------------

def _onehot_logits(counts, seed):
    experts = np.repeat(np.arange(len(counts)), counts)
    np.random.default_rng(seed).shuffle(experts)
    lg = np.full((experts.size, len(counts)), -1.0, np.float32)
    lg[np.arange(experts.size), experts] = 1.0
    return lg


def test_worked_imbalance_example_section5():
    g = json.load(open(os.path.join(GOLDEN, "expert_parallelism_s5_imbalance.json")))
    counts = np.array(g["counts"])
    assert counts.sum() == g["T"] and g["T"] // g["E"] == g["ideal_per_expert"]
    idx, _, _ = oracle.route(_onehot_logits(counts, 7), g["k"])
    # one GPU per expert (R = E): rank level == expert level == 140/64
    d8 = oracle.dispatch(idx, g["E"], 8)
    assert list(d8["expert_counts"]) == list(counts)
    assert list(d8["expert_offsets"]) == [0] + list(np.cumsum(counts))
    assert d8["imbalance"][0] == np.float32(140 / 64) == np.float32(2.1875)
    assert d8["imbalance"][1] == np.float32(2.1875)
    assert round(float(d8["imbalance"][0]), 1) == 2.2            # the page prints "2.2x"
    assert round(100.0 / float(d8["imbalance"][0])) == 46        # the page's 46% effective utilization
    # two logical ranks, experts {0..3} and {4..7}: 375 vs 137 against 256
    d2 = oracle.dispatch(idx, g["E"], 2)
    assert list(d2["rank_counts"]) == [375, 137]
    assert list(d2["rank_offsets"]) == [0, 375, 512]
    assert d2["imbalance"][0] == np.float32(1.46484375)
    assert d2["imbalance"][1] == np.float32(2.1875)


@pytest.mark.parametrize("T,E,k,R", [(1, 1, 1, 1), (37, 5, 3, 5), (200, 16, 4, 4), (129, 64, 8, 8)])
def test_dispatch_is_stable_counting_sort(T, E, k, R):
    rng = np.random.default_rng(T * 31 + E)
    idx = rng.integers(0, E, size=(T, k)).astype(np.int32)   # repeats allowed here
    d = oracle.dispatch(idx, E, R)
    A = T * k
    flat = idx.reshape(-1)
    # brute force: stable sort of assignments by expert
    assert list(d["row_src"]) == sorted(range(A), key=lambda a: (flat[a], a))
    assert np.all(d["assign_row"][d["row_src"]] == np.arange(A))
    assert np.all(d["row_src"][d["assign_row"]] == np.arange(A))
    assert d["expert_counts"].sum() == A
    assert list(d["expert_counts"]) == [int((flat == e).sum()) for e in range(E)]
    assert d["expert_offsets"][0] == 0 and d["expert_offsets"][E] == A
    per = E // R
    for r in range(R):
        assert d["rank_counts"][r] == sum(int((flat == e).sum()) for e in range(r * per, (r + 1) * per))
        assert d["rank_offsets"][r] == int((flat < r * per).sum())
    # every row of an expert's range holds that expert, in increasing assignment order
    for e in range(E):
        rows = d["row_src"][d["expert_offsets"][e]:d["expert_offsets"][e + 1]]
        assert np.all(flat[rows] == e) and np.all(np.diff(rows) > 0)
    mx_r = max(d["rank_counts"]) * R
    assert d["imbalance"][0] == np.float32(mx_r / A)


def test_dispatch_empty_batch_and_out_of_range_entries():
    d = oracle.dispatch(np.zeros((0, 2), np.int32), 4, 2)
    assert list(d["expert_counts"]) == [0] * 4 and list(d["imbalance"]) == [1.0, 1.0]
    idx = np.array([[0, 9], [-1, 1]], np.int32)
    d = oracle.dispatch(idx, 4, 2)
    assert d["skipped"] == 2 and list(d["expert_counts"]) == [1, 1, 0, 0]
    assert list(d["assign_row"]) == [0, -1, -1, 1]


def test_permute_rows_copies_token_rows_bit_exactly():
    wl = moe_synth.workload("tiny").with_(T=50)
    x = moe_synth.host_x(wl)
    idx, _, _ = oracle.route(moe_synth.host_logits(wl), wl.k)
    d = oracle.dispatch(idx, wl.E, wl.R)
    xp = oracle.permute_rows(x, d["row_src"], wl.k)
    a = np.arange(wl.A)
    assert np.array_equal(xp[d["assign_row"][a]], x[a // wl.k])


def test_communication_volume_section4():
    """x_perm is k*d*bytes per token: the page's Mixtral figures, 2.1 MB/layer and 67 MB/step."""
    g = json.load(open(os.path.join(GOLDEN, "expert_parallelism_s4_volume.json")))
    T, k, d = g["batch"], g["k"], g["d"]
    idx = np.tile(np.arange(k, dtype=np.int32), (T, 1))
    disp = oracle.dispatch(idx, 8, 4)
    xp = oracle.permute_rows(np.zeros((T, d), np.uint16), disp["row_src"], k)
    per_dir = xp.nbytes
    assert per_dir == T * k * d * g["bytes_per_element"] == 1_048_576
    assert round(2 * per_dir / 1e6, 1) == 2.1
    assert round(2 * per_dir * g["moe_layers"] / 1e6) == 67


# ---------------------------------------------------------------------------
# expert FFN: special cases that reduce to a dense SwiGLU (numpy fp64)
# ---------------------------------------------------------------------------

def _numpy_swiglu(xb, w13b, w2b):
    f = w2b.shape[1]
    x = _f(xb)
    wg, wu, wd = _f(w13b[:f]), _f(w13b[f:]), _f(w2b)
    a = x @ wg.T
    b = x @ wu.T
    return ((a * (1.0 / (1.0 + np.exp(-a)))) * b) @ wd.T


def test_silu_closed_form_values():
    # one row, d = 1, f = 1: y = w2 * silu(wg x) * (wu x)
    for xv, wg, wu, w2 in [(1.0, 0.0, 1.0, 1.0), (2.0, 1.0, 1.0, 1.0), (1.0, -3.0, 2.0, 0.5)]:
        y = oracle.swiglu(_bf16([[xv]]), _bf16([[wg], [wu]]), _bf16([[w2]]))
        a = wg * xv
        expect = w2 * (a / (1.0 + math.exp(-a))) * (wu * xv)
        assert abs(y[0, 0] - expect) <= 1e-15 * max(1.0, abs(expect))
    y = oracle.swiglu(_bf16([[1.0]]), _bf16([[0.0], [5.0]]), _bf16([[1.0]]))
    assert y[0, 0] == 0.0  # silu(0) = 0 kills the up branch


def test_one_expert_top1_layer_equals_dense_swiglu():
    """E = 1, k = 1: the MoE layer is a dense SwiGLU FFN (gate 1, identity permutation)."""
    wl = moe_synth.Workload("e1", T=33, d=48, E=1, k=1, f=80, R=1)
    x = moe_synth.host_x(wl)
    lg = moe_synth.host_logits(wl)
    w13, w2 = moe_synth.host_w13(wl), moe_synth.host_w2(wl)
    res = oracle.layer(x, lg, w13, w2, k=1, R=1)
    assert np.all(res["topk_gate"] == 1.0) and np.all(res["row_src"] == np.arange(wl.T))
    ref = _numpy_swiglu(x, w13[0], w2[0])
    assert np.max(np.abs(res["out"] - ref)) <= 1e-12 * np.max(np.abs(ref))


def test_each_expert_is_a_dense_swiglu_on_its_rows():
    wl = moe_synth.Workload("e4", T=40, d=32, E=4, k=2, f=48, R=2)
    x = moe_synth.host_x(wl)
    w13, w2 = moe_synth.host_w13(wl), moe_synth.host_w2(wl)
    idx, _, _ = oracle.route(moe_synth.host_logits(wl), wl.k)
    d = oracle.dispatch(idx, wl.E, wl.R)
    xp = oracle.permute_rows(x, d["row_src"], wl.k)
    y, _ = oracle.expert_ffn(xp, d["expert_offsets"], w13, w2)
    for e in range(wl.E):
        r0, r1 = d["expert_offsets"][e], d["expert_offsets"][e + 1]
        ref = _numpy_swiglu(xp[r0:r1], w13[e], w2[e])
        assert np.max(np.abs(y[r0:r1] - ref), initial=0.0) <= 1e-12 * max(1e-30, np.max(np.abs(ref), initial=0))


def test_shared_expert_is_dense_swiglu_on_all_tokens():
    wl = moe_synth.Workload("sh", T=20, d=32, E=2, k=1, f=64, R=1, n_shared=1)
    x = moe_synth.host_x(wl)
    w13, w2 = moe_synth.host_w13(wl), moe_synth.host_w2(wl)
    w13s, w2s = moe_synth.host_w13s(wl), moe_synth.host_w2s(wl)
    res = oracle.layer(x, moe_synth.host_logits(wl), w13, w2, 1, 1, w13s, w2s)
    ref = _numpy_swiglu(x, w13s, w2s)
    assert np.max(np.abs(res["y_shared"] - ref)) <= 1e-12 * np.max(np.abs(ref))


# ---------------------------------------------------------------------------
# combine: identity experts, exact pass-through, token-order metamorphic
# ---------------------------------------------------------------------------

def test_combine_with_identity_experts_returns_gate_sum_times_x():
    wl = moe_synth.workload("tiny").with_(T=64)
    x = moe_synth.host_x(wl)
    idx, gate, _ = oracle.route(moe_synth.host_logits(wl), wl.k)
    d = oracle.dispatch(idx, wl.E, wl.R)
    xp = oracle.permute_rows(x, d["row_src"], wl.k)
    out = oracle.combine(_f(xp), d["assign_row"], gate)
    expect = gate.astype(np.float64).sum(1, keepdims=True) * _f(x)
    assert np.max(np.abs(out - expect)) <= 1e-12


def test_dispatch_then_combine_k1_is_exact_identity():
    wl = moe_synth.workload("tiny").with_(T=64, k=1)
    x = moe_synth.host_x(wl)
    idx, gate, _ = oracle.route(moe_synth.host_logits(wl), 1)
    d = oracle.dispatch(idx, wl.E, wl.R)
    xp = oracle.permute_rows(x, d["row_src"], 1)
    out = oracle.combine(_f(xp), d["assign_row"], gate)
    assert np.array_equal(out, _f(x))


def test_layer_commutes_with_token_permutation():
    wl = moe_synth.Workload("perm", T=24, d=32, E=6, k=2, f=32, R=3)
    x, lg = moe_synth.host_x(wl), moe_synth.host_logits(wl)
    w13, w2 = moe_synth.host_w13(wl), moe_synth.host_w2(wl)
    p = np.random.default_rng(5).permutation(wl.T)
    a = oracle.layer(x, lg, w13, w2, wl.k, wl.R)["out"]
    b = oracle.layer(x[p], lg[p], w13, w2, wl.k, wl.R)["out"]
    assert np.max(np.abs(a[p] - b)) <= 1e-12


def test_sorted_path_equals_naive_per_token_loop():
    """Hands-on exercise C of §10: naive per-token loop vs sort-then-grouped-FFN."""
    wl = moe_synth.Workload("naive", T=30, d=32, E=5, k=2, f=48, R=5, n_shared=1)
    x, lg = moe_synth.host_x(wl), moe_synth.host_logits(wl)
    w13, w2 = moe_synth.host_w13(wl), moe_synth.host_w2(wl)
    w13s, w2s = moe_synth.host_w13s(wl), moe_synth.host_w2s(wl)
    res = oracle.layer(x, lg, w13, w2, wl.k, wl.R, w13s, w2s)
    naive = oracle.naive_token_loop(x, res["topk_idx"], res["topk_gate"], w13, w2, w13s, w2s)
    assert np.max(np.abs(res["out"] - naive)) <= 1e-12 * np.max(np.abs(naive))


# ---------------------------------------------------------------------------
# capacity factor (§5 "Mitigations" 1): keep the first `capacity` per expert
# ---------------------------------------------------------------------------

def test_capacity_on_the_worked_example():
    """C = 1.25 ("typical" on the page): capacity = 1.25 * 512 / 8 = 80 per expert."""
    g = json.load(open(os.path.join(GOLDEN, "expert_parallelism_s5_imbalance.json")))
    counts = np.array(g["counts"])
    idx, _, _ = oracle.route(_onehot_logits(counts, 7), 1)
    cap = math.ceil(1.25 * g["T"] / g["E"])
    assert cap == 80
    d = oracle.dispatch(idx, g["E"], g["E"], capacity=cap)
    kept = np.minimum(counts, cap)
    assert list(d["expert_counts"]) == kept.tolist() == [80, 80, 78, 62, 48, 40, 31, 18]
    assert d["dropped"] == int((counts - kept).sum()) == 75
    # the capacity bounds the imbalance: 80 * 8 / 437 instead of 140 * 8 / 512
    assert d["imbalance"][1] == np.float32(640 / 437)
    assert d["imbalance"][1] < np.float32(2.1875)


@pytest.mark.parametrize("T,E,k,cap", [(300, 8, 2, 50), (257, 16, 4, 1), (64, 5, 3, 1000), (129, 64, 8, 7)])
def test_capacity_keeps_the_first_assignments_in_order(T, E, k, cap):
    idx = np.random.default_rng(T + cap).integers(0, E, size=(T, k)).astype(np.int32)
    d = oracle.dispatch(idx, E, 1, capacity=cap)
    flat = idx.reshape(-1)
    keep = np.zeros(T * k, bool)
    for e in range(E):                       # brute force: the first `cap` of each expert, in order
        keep[np.flatnonzero(flat == e)[:cap]] = True
    assert np.array_equal(d["assign_row"] >= 0, keep)
    assert d["dropped"] == int((~keep).sum())
    assert list(d["row_src"][:keep.sum()]) == sorted(np.flatnonzero(keep), key=lambda a: (flat[a], a))
    assert np.all(d["row_src"][keep.sum():] == -1)
    if cap >= max(np.bincount(flat, minlength=E)):   # a capacity nobody reaches changes nothing
        free = oracle.dispatch(idx, E, 1)
        for n in ("expert_counts", "row_src", "assign_row"):
            assert np.array_equal(d[n], free[n])


def test_capacity_layer_equals_naive_loop_without_dropped_assignments():
    wl = moe_synth.Workload("cap", T=40, d=32, E=4, k=2, f=48, R=2, bias_kind="hot", n_hot=1, beta=2.0)
    x, lg = moe_synth.host_x(wl), moe_synth.host_logits(wl)
    w13, w2 = moe_synth.host_w13(wl), moe_synth.host_w2(wl)
    res = oracle.layer(x, lg, w13, w2, wl.k, wl.R, capacity=12)
    assert res["dropped"] > 0
    idx = res["topk_idx"].copy()
    idx.reshape(-1)[res["assign_row"] < 0] = -1          # a dropped assignment adds nothing
    naive = oracle.naive_token_loop(x, idx, res["topk_gate"], w13, w2)
    assert np.max(np.abs(res["out"] - naive)) <= 1e-12 * np.max(np.abs(naive))


# ---------------------------------------------------------------------------
# dispatch with capacity and ranks: randomised brute force (hypothesis)
# ---------------------------------------------------------------------------

def _brute_dispatch(flat, E, R, cap):
    """Stable sort by expert keeping each expert's first `cap` assignments (cap 0: all)."""
    A = len(flat)
    kept = [[] for _ in range(E)]
    for a in range(A):
        e = int(flat[a])
        if cap == 0 or len(kept[e]) < cap:
            kept[e].append(a)
    row_src = [a for e in range(E) for a in kept[e]]
    assign_row = [-1] * A
    for p, a in enumerate(row_src):
        assign_row[a] = p
    counts = [len(kept[e]) for e in range(E)]
    per = E // R
    rank_counts = [sum(counts[r * per:(r + 1) * per]) for r in range(R)]
    return row_src, assign_row, counts, rank_counts


def test_dispatch_matches_brute_force_on_random_shapes_with_capacity():
    from hypothesis import given, settings, strategies as st

    @st.composite
    def case(draw):
        E = draw(st.integers(1, 24))
        k = draw(st.integers(1, min(E, 8)))
        divisors = [r for r in range(1, E + 1) if E % r == 0]
        R = draw(st.sampled_from(divisors))
        T = draw(st.integers(0, 60))
        seed = draw(st.integers(0, 2**31 - 1))
        cap = draw(st.integers(0, max(1, T * k)))
        return T, E, k, R, cap, seed

    @settings(max_examples=80, deadline=None)
    @given(case())
    def check(c):
        T, E, k, R, cap, seed = c
        rng = np.random.default_rng(seed)
        idx = np.array([rng.permutation(E)[:k] for _ in range(T)], np.int32).reshape(T, k)
        d = oracle.dispatch(idx, E, R, capacity=cap)
        flat = idx.reshape(-1)
        row_src, assign_row, counts, rank_counts = _brute_dispatch(flat, E, R, cap)
        total = len(row_src)
        assert list(d["expert_counts"]) == counts
        assert list(d["expert_offsets"]) == [sum(counts[:e]) for e in range(E + 1)]
        assert list(d["rank_counts"]) == rank_counts
        assert list(d["rank_offsets"]) == [sum(rank_counts[:r]) for r in range(R + 1)]
        assert list(d["row_src"][:total]) == row_src and np.all(d["row_src"][total:] == -1)
        assert list(d["assign_row"]) == assign_row
        assert d["dropped"] == T * k - total
        if total:
            assert d["imbalance"][0] == np.float32(max(rank_counts) * R / total)
            assert d["imbalance"][1] == np.float32(max(counts) * E / total)
        else:
            assert list(d["imbalance"]) == [1.0, 1.0]

    check()
