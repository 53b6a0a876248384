"""The seeded input generator: reproducibility, distribution and workload structure (the per-rank
weight fill, marked gpu, needs a device)."""
import numpy as np
import pytest

import moe_synth
import oracle


def test_subsets_regenerate_bit_identically():
    wl = moe_synth.workload("tiny")
    x = moe_synth.host_x(wl)
    rows = np.array([0, 17, 255])
    assert np.array_equal(moe_synth.host_x(wl, rows), x[rows])
    lg = moe_synth.host_logits(wl)
    assert np.array_equal(moe_synth.host_logits(wl, rows), lg[rows])
    w13 = moe_synth.host_w13(wl)
    assert np.array_equal(moe_synth.host_w13(wl, 5), w13[5])
    assert np.array_equal(moe_synth.host_w2(wl, 3), moe_synth.host_w2(wl)[3])


def test_streams_are_independent_and_seeded():
    wl = moe_synth.workload("tiny")
    a = moe_synth.host_x(wl)
    b = moe_synth.host_x(wl.with_(seed=1))
    assert not np.array_equal(a, b)
    assert np.array_equal(a, moe_synth.host_x(wl))


def test_value_distribution():
    wl = moe_synth.workload("tiny")
    x = moe_synth.bf16_to_f32(moe_synth.host_x(wl)).astype(np.float64)
    assert abs(x.mean()) < 0.01 and abs(x.std() - 1.0) < 0.01
    w = moe_synth.bf16_to_f32(moe_synth.host_w13(wl)).astype(np.float64)
    assert abs(w.mean()) < 1e-4 and abs(w.std() - 0.02) < 2e-4
    # Irwin-Hall(4) support is bounded at sqrt(12) sigma
    assert np.abs(x).max() <= np.sqrt(12.0) * 1.01


def test_popularity_permutation_is_a_permutation():
    for name in ("mixtral_prefill", "dsv3_decode", "qwen3_mixed", "dsv3_skewed_prefill"):
        wl = moe_synth.workload(name)
        pi = moe_synth.popularity_perm(wl)
        assert sorted(pi.tolist()) == list(range(wl.E))


def test_qwen3_mixed_has_hot_and_cold_experts():
    wl = moe_synth.workload("qwen3_mixed")
    idx, _, _ = oracle.route(moe_synth.host_logits(wl), wl.k)
    c = np.bincount(idx.reshape(-1), minlength=wl.E)
    cold = c[moe_synth.popularity_perm(wl) >= wl.E // 2]
    assert c.max() > 160 and cold.min() < 20


def test_skewed_prefill_hot_share_is_half():
    wl = moe_synth.workload("dsv3_skewed_prefill")
    idx, _, _ = oracle.route(moe_synth.host_logits(wl), wl.k)
    c = np.bincount(idx.reshape(-1), minlength=wl.E)
    hot = moe_synth.popularity_perm(wl) < wl.n_hot
    assert wl.n_hot == 26 and 0.48 <= c[hot].sum() / c.sum() <= 0.52


@pytest.mark.gpu
def test_device_expert_weights_are_the_rows_of_the_full_tensors():
    """A rank's own experts' weights (expert parallelism) equal the matching rows of the full
    tensors, bit for bit (host fill, the same generator)."""
    import torch
    wl = moe_synth.Workload("w", T=4, d=128, E=8, k=2, f=128, R=4, n_shared=1)
    part = moe_synth.device_expert_weights(wl, 2, 6)
    assert np.array_equal(part["w13"].view(torch.int16).cpu().numpy().view(np.uint16), moe_synth.host_w13(wl)[2:6])
    assert np.array_equal(part["w2"].view(torch.int16).cpu().numpy().view(np.uint16), moe_synth.host_w2(wl)[2:6])
    assert np.array_equal(part["w13s"].view(torch.int16).cpu().numpy().view(np.uint16), moe_synth.host_w13s(wl))
