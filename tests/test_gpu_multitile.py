"""Element-wise parity of the persistent grouped GEMM when every CTA runs several tiles.

The grouped GEMM is persistent: a CTA (or CTA pair) claims tile after tile from a
counter and carries state from one tile to the next: the operand ring's stage and
phase, the tile queue's slot and phase, and which of its two TMEM accumulators the
tile uses (and that buffer's phase). All of it only shows up from a CTA's second
and third tile on. Every case here is sized so that the CTAs (the CTA pairs) run
at least 4 tiles each on average in both GEMMs (checked from the routed counts
before the comparison; tiles are claimed at run time, so a CTA's own count varies
around that mean), and y_perm, y_shared and out are compared element by element
with the oracle (the page "Expert Parallelism", §4 COMPUTE and COMBINE), under
both tile shapes: single-CTA tiles, and CTA-pair tiles with half-height last
blocks.

The full Mixtral-like workload (T 4096, d 4096, f 14336: about 50 single tiles per
CTA in gate/up, 7 to 8 pair tiles per cluster in down) is also compared in full:
every element of y_perm and out against the oracle's whole-layer run (about a
minute of host CPU).
"""
import functools

import numpy as np
import pytest

import combine_warp_top_expert_b200 as moe
import moe_synth
import oracle
from parity_util import bits, close, f64, np_i32

POLICIES = {"single": moe.GEMM_SINGLE, "pair": moe.GEMM_PAIR}

CASES = {
    # 8 experts, ~1024 rows each (Zipf-skewed): ragged expert ends, ~68 m-tiles of 128 rows
    "e8_k2": (moe_synth.Workload("mt_e8", T=4096, d=3072, E=8, k=2, f=1536, R=4, bias_kind="zipf",
                                 zipf_s=0.5, seed=5), 0.0),
    # 64 experts, top-8, 6 hot ones, a shared expert and a capacity factor of 1.25 (drops)
    "e64_k8_shared_cap": (moe_synth.Workload("mt_e64", T=1536, d=2048, E=64, k=8, f=1024, R=8, n_shared=1,
                                             bias_kind="hot", n_hot=6, beta=1.5, seed=9), 1.25),
}


def _sm_count():
    import torch
    return torch.cuda.get_device_properties(0).multi_processor_count


def _tiles(rows, tm):
    return -(-rows // tm)


def tiles_per_unit(counts, T, n_shared, d, f, policy, sms):
    """Mean tiles per CTA (single) or per CTA pair (pair) in the GEMM with fewer tiles,
    from the kernels' schedule: groups = experts (+ shared), m-tiles of 128 rows
    (single) or 256 rows with a half-height last block of <= 128 rows (pair), n-tiles
    of 128 h columns (gate/up) or 256 output columns (down)."""
    groups = list(counts) + ([T] * n_shared)
    tm, units = (128, sms) if policy == "single" else (256, sms // 2)
    return min(sum(_tiles(r, tm) for r in groups) * n_tiles_n / units for n_tiles_n in (f // 128, d // 256))


@functools.lru_cache(maxsize=None)
def _oracle_case(name):
    wl, cf = CASES[name]
    cap = moe.capacity_for(cf, wl.T, wl.k, wl.E) if cf else 0
    res = oracle.layer(moe_synth.host_x(wl), moe_synth.host_logits(wl), moe_synth.host_w13(wl),
                       moe_synth.host_w2(wl), wl.k, wl.R, moe_synth.host_w13s(wl) if wl.n_shared else None,
                       moe_synth.host_w2s(wl) if wl.n_shared else None, capacity=cap)
    return cap, res


@pytest.mark.gpu
@pytest.mark.parametrize("policy", list(POLICIES))
@pytest.mark.parametrize("case", list(CASES))
def test_multi_tile_layer_matches_oracle_element_by_element(case, policy):
    import torch
    wl, cf = CASES[case]
    cap, res = _oracle_case(case)
    counts = res["expert_counts"].tolist()
    per_unit = tiles_per_unit(counts, wl.T, wl.n_shared, wl.d, wl.f, policy, _sm_count())
    assert per_unit >= 4, f"only {per_unit:.1f} tiles per CTA/cluster: the case does not reach the persistent loop"
    if cf:
        assert res["dropped"] > 0
    shape = moe.Shape(T=wl.T, d=wl.d, E=wl.E, k=wl.k, f=wl.f, R=wl.R, n_shared=wl.n_shared, capacity=cap)
    dv = moe_synth.device_inputs(wl)
    old = moe.set_gemm_policy(POLICIES[policy])
    try:
        layer = moe.MoELayer(shape, dv["w13"], dv["w2"], dv.get("w13s"), dv.get("w2s"))
        outs = layer(dv["logits"], dv["x"])
        assert moe.get_status(layer.ws) == 0
    finally:
        moe.set_gemm_policy(old)
    for n in ("topk_idx", "expert_counts", "expert_offsets", "rank_counts", "rank_offsets", "row_src", "assign_row"):
        assert np.array_equal(np_i32(outs[n]), res[n]), n
    A = int(res["expert_offsets"][-1])                           # rows placed (drops excluded)
    close(f64(bits(outs["y_perm"][:A])), res["y_perm"][:A], f"y_perm {case} {policy}")
    if wl.n_shared:
        close(f64(bits(outs["y_shared"])), res["y_shared"], f"y_shared {case} {policy}")
    close(f64(bits(outs["out"])), res["out"], f"out {case} {policy}")
    # every expert on its own, so that one wrong group cannot hide in the whole tensor's norm
    off = res["expert_offsets"]
    y = f64(bits(outs["y_perm"][:A]))
    for e in range(wl.E):
        if off[e + 1] > off[e]:
            close(y[off[e]:off[e + 1]], res["y_perm"][off[e]:off[e + 1]], f"y_perm expert {e} {case} {policy}")
    del layer, outs, dv
    torch.cuda.empty_cache()


def test_tile_count_model_matches_a_hand_count():
    """The tiles-per-unit count used above, on a hand-worked case: two experts of 300 and
    100 rows, d = 512, f = 256 (2 n-tiles in either GEMM), 4 SMs. Single: (3 + 1) m-tiles
    x 2 = 8 tiles over 4 CTAs -> 2. Pair: (2 + 1) x 2 = 6 (the 44- and 100-row last
    blocks are half-height tiles) over 2 clusters -> 3. A shared expert is one more
    group of T rows."""
    assert tiles_per_unit([300, 100], 0, 0, 512, 256, "single", 4) == 2
    assert tiles_per_unit([300, 100], 0, 0, 512, 256, "pair", 4) == 3
    assert tiles_per_unit([300], 300, 1, 512, 256, "single", 4) == 3


@pytest.mark.gpu
def test_mixtral_prefill_full_output_matches_oracle():
    """Every element of y_perm and out at the benchmark's workload (default tile policy)."""
    import torch
    wl = moe_synth.workload("mixtral_prefill")
    shape = moe.Shape(T=wl.T, d=wl.d, E=wl.E, k=wl.k, f=wl.f, R=wl.R)
    dv = moe_synth.device_inputs(wl)
    layer = moe.MoELayer(shape, dv["w13"], dv["w2"])
    outs = layer(dv["logits"], dv["x"])
    assert moe.get_status(layer.ws) == 0
    y_gpu = f64(bits(outs["y_perm"]))
    out_gpu = f64(bits(outs["out"]))
    counts = np_i32(outs["expert_counts"]).tolist()
    del layer, outs, dv
    torch.cuda.empty_cache()
    assert tiles_per_unit(counts, wl.T, 0, wl.d, wl.f, "single", _sm_count()) >= 4
    res = oracle.layer(moe_synth.host_x(wl), moe_synth.host_logits(wl), moe_synth.host_w13(wl),
                       moe_synth.host_w2(wl), wl.k, wl.R)
    close(y_gpu, res["y_perm"], "y_perm mixtral_prefill (full)")
    close(out_gpu, res["out"], "out mixtral_prefill (full)")


# ---------------------------------------------------------------------------
# groups longer than one L2 band of m-tiles
# ---------------------------------------------------------------------------

BAND_BYTES = 24 << 20   # A rows per band of m-tiles (the kernels' tile order)


def band_m_tiles(tm, K):
    """m-tiles per band: the most whose A rows (tm rows x K bf16 each) fit BAND_BYTES."""
    return max(1, BAND_BYTES // (tm * K * 2))


BAND_CASES = {
    # gate/up reduces over d = 7168: 13 single (6 pair) m-tiles per band; the shared
    # expert's 4096 rows are 32 single (16 pair) m-tiles, 3 bands with a short last one
    "gate_up_bands": moe_synth.Workload("band_g", T=4096, d=7168, E=8, k=2, f=256, R=4, n_shared=1,
                                        bias_kind="zipf", zipf_s=1.0, seed=21),
    # down reduces over f = 7168: the same band sizes in the down GEMM
    "down_bands": moe_synth.Workload("band_d", T=4096, d=256, E=8, k=2, f=7168, R=4, n_shared=1,
                                     bias_kind="zipf", zipf_s=1.0, seed=22),
}


def test_band_model_on_a_hand_count():
    """24 MiB / (128 rows x 7168 x 2 bytes) = 13.7 -> 13 m-tiles per band; 256-row tiles: 6;
    a K of 2048 gives 48; a group of 32 m-tiles in 13-tile bands runs as 13 + 13 + 6."""
    assert band_m_tiles(128, 7168) == 13 and band_m_tiles(256, 7168) == 6
    assert band_m_tiles(128, 2048) == 48
    assert -(-32 // band_m_tiles(128, 7168)) == 3


@functools.lru_cache(maxsize=None)
def _oracle_band_case(name):
    wl = BAND_CASES[name]
    return oracle.layer(moe_synth.host_x(wl), moe_synth.host_logits(wl), moe_synth.host_w13(wl),
                        moe_synth.host_w2(wl), wl.k, wl.R, moe_synth.host_w13s(wl), moe_synth.host_w2s(wl))


@pytest.mark.gpu
@pytest.mark.parametrize("policy", list(POLICIES))
@pytest.mark.parametrize("case", list(BAND_CASES))
def test_groups_spanning_several_bands_match_oracle(case, policy):
    """The shared expert (and the largest routed experts) run their m-tiles in several
    bands, the last one short, in one of the GEMMs: every element of y_perm, y_shared
    and out against the oracle."""
    import torch
    wl = BAND_CASES[case]
    res = _oracle_band_case(case)
    tm = 128 if policy == "single" else 256
    K = wl.d if case == "gate_up_bands" else wl.f
    band = band_m_tiles(tm, K)
    m_shared = _tiles(wl.T, tm)
    assert m_shared >= 2 * band + 1 and m_shared % band != 0    # several bands, a short last one
    shape = moe.Shape(T=wl.T, d=wl.d, E=wl.E, k=wl.k, f=wl.f, R=wl.R, n_shared=1)
    dv = moe_synth.device_inputs(wl)
    old = moe.set_gemm_policy(POLICIES[policy])
    try:
        layer = moe.MoELayer(shape, dv["w13"], dv["w2"], dv["w13s"], dv["w2s"])
        outs = layer(dv["logits"], dv["x"])
        assert moe.get_status(layer.ws) == 0
    finally:
        moe.set_gemm_policy(old)
    close(f64(bits(outs["y_shared"])), res["y_shared"], f"y_shared {case} {policy}")
    off = res["expert_offsets"]
    y = f64(bits(outs["y_perm"]))
    for e in range(wl.E):
        if off[e + 1] > off[e]:
            close(y[off[e]:off[e + 1]], res["y_perm"][off[e]:off[e + 1]], f"y_perm expert {e} {case} {policy}")
    close(f64(bits(outs["out"])), res["out"], f"out {case} {policy}")
    # the shared expert's rows band by band, so that one misplaced band cannot hide
    ys = f64(bits(outs["y_shared"]))
    for b0 in range(0, wl.T, band * tm):
        close(ys[b0:b0 + band * tm], res["y_shared"][b0:b0 + band * tm], f"y_shared band at row {b0} {case}")
    del layer, outs, dv
    torch.cuda.empty_cache()
