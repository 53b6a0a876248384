"""Expert parallelism across GPUs, host side (no GPU): the exchange plan and the whole
exchange with 2 and 4 gloo ranks.

Page "Expert Parallelism" §1 (rank r of R owns experts [r*E/R, (r+1)*E/R)) and §4
"The All-to-All": after the exchange every rank holds one contiguous run of rows per
expert it owns, and COMBINE brings every result back in the original order.

The plan (moe_ep_plan_host, the same arithmetic as the device plan kernel) is
pinned against an explicit placement: the R ranks' batches taken as one batch, rank
after rank, are sorted by expert (stable) as the single-GPU dispatch does, and every
row's place in its owner's slice is read off that list. The multi-process test runs
the exchange on the host with gloo: each rank routes its own tokens with the oracle,
the ranks all-gather their per-expert counts, each rank sends every row to the row
of its owner's receive buffer that the plan gives, the owners run the oracle's expert
FFN, and every rank sums the rows of its tokens in combine. The receive buffers must
equal, bit for bit, the slices of the oracle's single-GPU dispatch of the combined
batch, and every rank's output the oracle's layer output for its tokens.
"""
import os
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

import combine_warp_top_expert_b200 as moe

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def explicit_rows(counts_all, capacity):
    """For every (source s, expert e, p-th assignment of s to e): its row in the owner's
    receive buffer, or -1 if dropped, read off the explicit single-GPU ordering."""
    R, E = counts_all.shape
    Er = E // R
    entries = []                                  # global rows, sorted by expert, then source, then p
    for e in range(E):
        kept = 0
        for s in range(R):
            for p in range(int(counts_all[s, e])):
                keep = capacity == 0 or kept < capacity
                entries.append((e, s, p, keep))
                kept += 1
    row = {}
    owner_row = [0] * R
    for e, s, p, keep in entries:
        o = e // Er
        if keep:
            row[(s, e, p)] = owner_row[o]
            owner_row[o] += 1
        else:
            row[(s, e, p)] = -1
    return row, owner_row


@pytest.mark.parametrize("R,E,capacity,seed", [(1, 8, 0, 0), (2, 8, 0, 1), (4, 16, 0, 2), (4, 16, 3, 3),
                                               (8, 64, 5, 4), (2, 6, 1, 5), (3, 9, 0, 6)])
def test_plan_matches_the_explicit_single_gpu_placement(R, E, capacity, seed):
    rng = np.random.default_rng(seed)
    counts = rng.integers(0, 9, size=(R, E)).astype(np.int32)
    counts[rng.random((R, E)) < 0.2] = 0          # some experts get nothing from some ranks
    row, owner_rows = explicit_rows(counts, capacity)
    Er = E // R
    for me in range(R):
        plan = moe.ep_plan_host(R, E, me, capacity, counts)
        for e in range(E):
            for p in range(int(counts[me, e])):
                want = row[(me, e, p)]
                got = int(plan["row_base"][e]) + p if p < int(plan["keep"][e]) else -1
                assert got == want, (me, e, p)
        # this rank's experts: their rows in its receive buffer
        sizes = [sum(1 for (s, e2, p), r in row.items() if e2 == e and r >= 0) for e in range(me * Er, (me + 1) * Er)]
        assert plan["recv_offsets"].tolist() == np.concatenate([[0], np.cumsum(sizes)]).tolist()
        assert int(plan["recv_offsets"][-1]) == owner_rows[me]


def test_plan_rejects_invalid_arguments():
    c = np.zeros((2, 8), np.int32)
    for R, E, rank, cap in ((0, 8, 0, 0), (3, 8, 0, 0), (2, 8, 2, 0), (2, 8, -1, 0), (2, 8, 0, -1), (2, 300, 0, 0)):
        with pytest.raises(ValueError):
            moe.ep_plan_host(R, E, rank, cap, np.zeros((R, E), np.int32) if R > 0 else c)
    bad = c.copy()
    bad[1, 3] = -2
    with pytest.raises(ValueError):
        moe.ep_plan_host(2, 8, 0, 0, bad)


# ---------------------------------------------------------------------------
# the whole exchange with gloo ranks
# ---------------------------------------------------------------------------

def _rank_main(rank, R, port, wl_kw, capacity, q):
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    import torch
    import torch.distributed as dist

    import combine_warp_top_expert_b200 as moe
    import moe_synth
    import oracle
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=R)
    try:
        wl = moe_synth.Workload(**wl_kw)                   # the combined batch of R * T tokens
        T = wl.T // R
        E, k, d, Er = wl.E, wl.k, wl.d, wl.E // R
        toks = np.arange(rank * T, (rank + 1) * T)
        x = moe_synth.host_x(wl, toks)
        idx, gate, _ = oracle.route(moe_synth.host_logits(wl, toks), k)
        counts = np.bincount(idx.reshape(-1), minlength=E).astype(np.int32)
        allc = torch.empty((R * E,), dtype=torch.int32)
        dist.all_gather_into_tensor(allc, torch.from_numpy(counts))
        counts_all = allc.numpy().reshape(R, E)
        plan = moe.ep_plan_host(R, E, rank, capacity, counts_all)
        # every assignment's owner and row there (the dispatch kernel's arithmetic)
        seen = np.zeros(E, np.int64)
        send_row = np.full(T * k, -1, np.int64)
        for a in range(T * k):
            e = int(idx.reshape(-1)[a])
            p = int(seen[e])
            seen[e] += 1
            if p < int(plan["keep"][e]):
                send_row[a] = int(plan["row_base"][e]) + p
        owner = idx.reshape(-1) // Er
        rows_cap = R * T * k
        # the exchange: rows (with their destination row) to their owners
        send_n = [int(np.sum((owner == o) & (send_row >= 0))) for o in range(R)]
        order = [a for o in range(R) for a in range(T * k) if owner[a] == o and send_row[a] >= 0]
        recv_n_t = torch.empty(R, dtype=torch.int64)
        dist.all_to_all_single(recv_n_t, torch.tensor(send_n, dtype=torch.int64))
        recv_n = recv_n_t.tolist()
        rows_out = torch.from_numpy(np.array([send_row[a] for a in order], np.int64).reshape(-1))
        # bf16 bit patterns travel as int32 (gloo has no 16-bit integer type)
        data_out = torch.from_numpy(np.stack([x[a // k] for a in order]).astype(np.int32) if order else
                                    np.zeros((0, d), np.int32))
        rows_in = torch.empty(sum(recv_n), dtype=torch.int64)
        data_in = torch.empty((sum(recv_n), d), dtype=torch.int32)
        dist.all_to_all_single(rows_in, rows_out, recv_n, send_n)
        dist.all_to_all_single(data_in, data_out, recv_n, send_n)
        recv = np.zeros((rows_cap, d), np.uint16)
        recv[rows_in.numpy()] = data_in.numpy().astype(np.uint16)
        n_mine = int(plan["recv_offsets"][-1])
        # the single-GPU layout of the combined batch
        g_idx, g_gate, _ = oracle.route(moe_synth.host_logits(wl), k)
        g = oracle.dispatch(g_idx, E, R, capacity)
        g_xperm = oracle.permute_rows(moe_synth.host_x(wl), g["row_src"], k)
        lo, hi = int(g["rank_offsets"][rank]), int(g["rank_offsets"][rank + 1])
        layout_ok = bool(np.array_equal(recv[:n_mine], g_xperm[lo:hi]) and n_mine == hi - lo and
                         np.array_equal(plan["recv_offsets"], g["expert_offsets"][rank * Er:(rank + 1) * Er + 1] - lo))
        # expert compute on the owner, results back, combine in the original order
        w13 = moe_synth.host_w13(wl)[rank * Er:(rank + 1) * Er]
        w2 = moe_synth.host_w2(wl)[rank * Er:(rank + 1) * Er]
        y_recv, _ = oracle.expert_ffn(recv[:n_mine], plan["recv_offsets"], w13, w2)
        y_full = np.zeros((rows_cap, d), np.float64)
        y_full[:n_mine] = y_recv
        y_all = [torch.empty((rows_cap, d), dtype=torch.float64) for _ in range(R)]
        dist.all_gather(y_all, torch.from_numpy(y_full))
        out = np.zeros((T, d), np.float64)
        for t in range(T):
            for j in range(k):
                a = t * k + j
                if send_row[a] >= 0:
                    out[t] += float(gate[t, j]) * y_all[int(owner[a])].numpy()[send_row[a]]
        ref = oracle.layer(moe_synth.host_x(wl), moe_synth.host_logits(wl), moe_synth.host_w13(wl),
                           moe_synth.host_w2(wl), k, R, capacity=capacity)["out"][rank * T:(rank + 1) * T]
        q.put((rank, layout_ok, float(np.max(np.abs(out - ref))), n_mine, sum(recv_n)))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("R,capacity", [(2, 0), (4, 0), (4, 40)])
def test_exchange_with_gloo_ranks_gives_the_single_gpu_layout_and_output(R, capacity):
    wl_kw = dict(name="ep", T=48 * R, d=128, E=8, k=2, f=128, R=R, bias_kind="zipf", zipf_s=1.0, seed=11 + R)
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    sys.path.insert(0, ROOT)
    import bench
    port = bench.free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, R, port, wl_kw, capacity, q)) for r in range(R)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=240)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(R))
    assert [r[0] for r in res] == list(range(R))
    total = 0
    for rank, layout_ok, max_err, n_mine, n_recv in res:
        assert layout_ok, rank
        assert n_mine == n_recv                    # every row sent to this rank arrived at a distinct row
        assert max_err <= 1e-12, (rank, max_err)   # same fp64 rows, same j order: the same sums
        total += n_mine
    if capacity == 0:
        assert total == 48 * R * 2
