"""The pins catch plausible mistakes: each test plants one mistake in a temporary
copy of the oracle's source (on the CPU), rebuilds it, and checks that the pin
written for that function fails on the mutant while it passes on the oracle.

Mutants: reversed tie-break, NaN ordered first instead of as -inf, wrong sign
in the gate exponent, softmax over all E logits instead of the k selected,
unstable (reversed) row order, imbalance denominator with the wrong count,
experts dealt to ranks round-robin instead of in contiguous blocks, rank
offsets not scaled by experts per rank, counts that still include dropped
assignments, token index taken as a % k in the row copy, swapped gate and up
halves, wrong silu sign, transposed down-projection index, gate dropped in
combine, shared-expert output dropped in combine, capacity keeping the last
instead of the first assignments.
"""
import importlib.util
import math
import os
import subprocess

import numpy as np
import pytest

import moe_synth
import oracle
from test_oracle_pins import _brute_topk, _numpy_swiglu, _onehot_logits

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "moe_oracle.cpp")


def _mutant(tmp_path, old: str, new: str):
    """Build the oracle with one textual change; return an oracle module bound to it."""
    text = open(SRC).read()
    assert text.count(old) == 1, old
    src = tmp_path / "mutant.cpp"
    src.write_text(text.replace(old, new))
    so = tmp_path / "libmutant.so"
    subprocess.run(["g++", "-std=c++17", "-O1", "-fopenmp", "-fPIC", "-shared", str(src), "-o", str(so)],
                   check=True)
    spec = importlib.util.spec_from_file_location("oracle_mutant", os.path.join(ROOT, "oracle", "__init__.py"))
    m = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(m)
    m.build = lambda force=False: str(so)
    return m


# ---- the pins, as functions of an oracle module: True when the pin holds ----

def pin_topk(o):
    rng = np.random.default_rng(105)
    lg = rng.integers(-2, 3, size=(64, 5)).astype(np.float32)
    idx, _, _ = o.route(lg, 3)
    return all(list(idx[t]) == _brute_topk([float(v) for v in lg[t]], 3) for t in range(64))


def pin_nan_last(o):
    """NaN orders as -inf: after every number, tied with -inf by index; each NaN counted."""
    lg = np.array([[np.nan, 1.0, 0.5, -3.0], [2.0, np.nan, np.nan, -np.inf]], np.float32)
    idx, _, nan = o.route(lg, 4)
    return list(idx[0]) == [1, 2, 3, 0] and list(idx[1]) == [0, 1, 2, 3] and nan == 3


def pin_gate_logistic(o):
    lg = np.random.default_rng(2).normal(scale=3.0, size=(200, 9)).astype(np.float32)
    idx, gate, _ = o.route(lg, 2)
    l0 = lg[np.arange(200), idx[:, 0]].astype(np.float64)
    l1 = lg[np.arange(200), idx[:, 1]].astype(np.float64)
    g0 = 1.0 / (1.0 + np.exp(l1 - l0))
    return (np.max(np.abs(gate[:, 0] - g0)) <= 2.0 ** -24 and np.max(np.abs(gate[:, 1] - (1.0 - g0))) <= 2.0 ** -24)


def pin_stable_sort(o):
    idx = np.random.default_rng(3).integers(0, 6, size=(50, 3)).astype(np.int32)
    d = o.dispatch(idx, 6, 2)
    flat = idx.reshape(-1)
    return list(d["row_src"]) == sorted(range(150), key=lambda a: (flat[a], a))


def pin_worked_example(o):
    counts = np.array([140, 95, 78, 62, 48, 40, 31, 18])
    idx, _, _ = oracle.route(_onehot_logits(counts, 7), 1)
    d2 = o.dispatch(idx, 8, 2)
    return d2["imbalance"][0] == np.float32(1.46484375) and d2["imbalance"][1] == np.float32(2.1875)


def pin_dense_swiglu(o):
    wl = moe_synth.Workload("e1", T=9, d=48, E=1, k=1, f=80, R=1)
    x, w13, w2 = moe_synth.host_x(wl), moe_synth.host_w13(wl), moe_synth.host_w2(wl)
    y = o.swiglu(x, w13[0], w2[0])
    ref = _numpy_swiglu(x, w13[0], w2[0])
    return np.max(np.abs(y - ref)) <= 1e-12 * np.max(np.abs(ref))


def pin_silu_closed_form(o):
    bf = lambda v: (np.array(v, np.float32).view(np.uint32) >> 16).astype(np.uint16)  # exact for these values
    y = o.swiglu(bf([[1.0]]), bf([[-3.0], [2.0]]), bf([[0.5]]))
    a = -3.0
    return abs(y[0, 0] - 0.5 * (a / (1.0 + math.exp(-a))) * 2.0) <= 1e-15


def pin_identity_experts(o):
    wl = moe_synth.workload("tiny").with_(T=32)
    x = moe_synth.host_x(wl)
    idx, gate, _ = o.route(moe_synth.host_logits(wl), wl.k)
    d = o.dispatch(idx, wl.E, wl.R)
    xp = o.permute_rows(x, d["row_src"], wl.k)
    f = moe_synth.bf16_to_f32
    out = o.combine(f(xp).astype(np.float64), d["assign_row"], gate)
    expect = gate.astype(np.float64).sum(1, keepdims=True) * f(x).astype(np.float64)
    return np.max(np.abs(out - expect)) <= 1e-12


def pin_capacity_first(o):
    idx = np.random.default_rng(9).integers(0, 4, size=(60, 2)).astype(np.int32)
    d = o.dispatch(idx, 4, 1, capacity=10)
    flat = idx.reshape(-1)
    keep = np.zeros(120, bool)
    for e in range(4):
        keep[np.flatnonzero(flat == e)[:10]] = True
    return bool(np.array_equal(d["assign_row"] >= 0, keep))


def pin_rank_offsets(o):
    """rank r's rows start after every row of the experts below r*E/R (numpy count)."""
    E, R = 12, 4
    idx = np.random.default_rng(11).integers(0, E, size=(90, 3)).astype(np.int32)
    d = o.dispatch(idx, E, R)
    n = np.bincount(idx.reshape(-1), minlength=E)
    want = [int(n[:r * E // R].sum()) for r in range(R + 1)]
    return list(d["rank_offsets"]) == want and list(d["rank_counts"]) == list(np.diff(want))


def pin_permute_token(o):
    """x_perm row p is the row of token a // k, a = row_src[p] (numpy indexing)."""
    k = 3
    idx = np.random.default_rng(12).integers(0, 5, size=(17, k)).astype(np.int32)
    d = o.dispatch(idx, 5, 1)
    x = np.random.default_rng(13).integers(0, 1 << 16, size=(17, 24)).astype(np.uint16)
    xp = o.permute_rows(x, d["row_src"], k)
    return bool(np.array_equal(xp, x[d["row_src"] // k]))


def pin_combine_shared(o):
    """zero expert outputs leave exactly the shared expert's output (weight one)."""
    idx = np.random.default_rng(14).integers(0, 4, size=(10, 2)).astype(np.int32)
    d = o.dispatch(idx, 4, 1)
    gate = np.random.default_rng(15).uniform(0.1, 0.9, size=(10, 2)).astype(np.float32)
    ys = np.random.default_rng(16).normal(size=(10, 8))
    out = o.combine(np.zeros((20, 8)), d["assign_row"], gate, ys)
    return bool(np.array_equal(out, ys))


def pin_capacity_counts(o):
    """with capacity c, expert e keeps min(n_e, c) rows and the offsets scan those."""
    idx = np.random.default_rng(17).integers(0, 5, size=(80, 2)).astype(np.int32)
    d = o.dispatch(idx, 5, 1, capacity=12)
    kept = np.minimum(np.bincount(idx.reshape(-1), minlength=5), 12)
    return (list(d["expert_counts"]) == list(kept)
            and list(d["expert_offsets"]) == [0] + list(np.cumsum(kept)))


MUTANTS = [
    ("reversed tie-break", "return ka > kb || (ka == kb && a < b);", "return ka > kb || (ka == kb && a > b);",
     pin_topk),
    ("NaN orders first", "return std::isnan(l) ? -std::numeric_limits<double>::infinity() : (double)l;",
     "return std::isnan(l) ? std::numeric_limits<double>::infinity() : (double)l;", pin_nan_last),
    ("gate exponent sign", "topk_gate[t * k + j] = (float)(std::exp(order_key(l[order[j]]) - l0) / s);",
     "topk_gate[t * k + j] = (float)(std::exp(l0 - order_key(l[order[j]])) / s);", pin_gate_logistic),
    ("unstable row order", "const int32_t p = offsets[e] + cursor[e]++;",
     "const int32_t p = offsets[e + 1] - 1 - cursor[e]++;", pin_stable_sort),
    ("imbalance denominator", "imbalance[1] = (float)((double)(max_e * E) / (double)total);",
     "imbalance[1] = (float)((double)(max_e * R) / (double)total);", pin_worked_example),
    ("gate and up swapped", "const float* wg = &w13f[(size_t)j * d];\n        const float* wu = &w13f[(size_t)(f + j) * d];",
     "const float* wu = &w13f[(size_t)j * d];\n        const float* wg = &w13f[(size_t)(f + j) * d];",
     pin_dense_swiglu),
    ("silu sign", "h[j] = a / (1.0 + std::exp(-a)) * b;", "h[j] = a / (1.0 + std::exp(a)) * b;",
     pin_silu_closed_form),
    ("transposed down projection", "const float* wd = &w2f[(size_t)o * f];\n        double acc = 0.0;\n        for (int32_t j = 0; j < f; ++j) acc += (double)wd[j] * h[j];",
     "double acc = 0.0;\n        for (int32_t j = 0; j < f; ++j) acc += (double)w2f[(size_t)j * d + o % d] * h[j];",
     pin_dense_swiglu),
    ("gate dropped in combine", "for (int32_t c = 0; c < d; ++c) o[c] += g * y_perm[p * d + c];",
     "for (int32_t c = 0; c < d; ++c) o[c] += y_perm[p * d + c];", pin_identity_experts),
    ("capacity keeps the last", "if (capacity > 0 && seen[e] >= capacity) {",
     "if (capacity > 0 && seen[e] < capacity) {", pin_capacity_first),
    ("softmax over all experts", "for (int32_t j = 0; j < k; ++j) s += std::exp(order_key(l[order[j]]) - l0);",
     "for (int32_t j = 0; j < E; ++j) s += std::exp(order_key(l[order[j]]) - l0);", pin_gate_logistic),
    ("ranks own interleaved experts",
     "for (int32_t e = r * per_rank; e < (r + 1) * per_rank; ++e) c += counts[e];",
     "for (int32_t e = r; e < E; e += R) c += counts[e];", pin_worked_example),
    ("rank offsets unscaled", "rank_offsets[r] = offsets[r * per_rank];", "rank_offsets[r] = offsets[r];",
     pin_rank_offsets),
    ("dropped assignments counted", "if (keep[a]) counts[topk_idx[a]] += 1;", "counts[topk_idx[a]] += 1;",
     pin_capacity_counts),
    ("token index by modulo", "const int64_t t = row_src[p] / k;", "const int64_t t = row_src[p] % k;",
     pin_permute_token),
    ("shared output dropped", "for (int32_t c = 0; c < d; ++c) o[c] += y_shared[t * d + c];",
     "for (int32_t c = 0; c < d; ++c) o[c] += 0.0 * y_shared[t * d + c];", pin_combine_shared),
]


@pytest.mark.parametrize("name,old,new,pin", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_pin_holds_on_oracle_and_fails_on_mutant(tmp_path, name, old, new, pin):
    assert pin(oracle), f"pin for '{name}' fails on the oracle itself"
    mutant = _mutant(tmp_path, old, new)
    assert not pin(mutant), f"pin did not catch the planted mistake: {name}"
