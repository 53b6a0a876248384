"""bench.py's multi-rank logic on CPU: world-size-2 gloo ranks (no GPU).

With N GPUs the benchmark runs N independent replicas of the layer ("replicas
only": the single-GPU path has no cross-GPU exchange). Each rank times its own
steps; the reported value is all ranks' tokens over the slowest rank's time.
"""
import os
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    import torch.distributed as dist

    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local_ms = [250.0, 400.0][rank]            # rank 1 is the slower replica
        mx = bench.max_over_ranks(local_ms, world)
        value = bench.aggregate_throughput(4096, 20, world, mx / 1e3)
        q.put((rank, mx, value, bench.replica_seed(0, rank)))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_report_max_time_and_total_tokens():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    sys.path.insert(0, ROOT)
    import bench
    port = bench.free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    for rank, mx, value, seed in res:
        assert mx == 400.0                          # the slowest rank sets the time
        assert value == pytest.approx(2 * 4096 * 20 / 0.4)
        assert seed == rank                         # each replica gets its own batch


def test_single_rank_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.5, 1) == 3.5
    assert bench.aggregate_throughput(128, 10, 1, 2.0) == 640.0


def test_max_affine_fit_recovers_known_regimes():
    """The regime fit of bench.py --regime-sweep recovers a known max-affine profile."""
    sys.path.insert(0, ROOT)
    import bench
    G, N, t = [], [], []
    for g in (1, 8, 32, 64, 148, 256):
        for n in (1, 8, 16, 32, 64, 128, 192, 256, 384, 512, 1024):
            G.append(g)
            N.append(g * n)
            t.append(max(0.01 + 0.0135 * g, 0.02 + 6.3e-5 * g * n))
    fit = bench.fit_max_affine(G, N, t)
    assert fit["b"] == pytest.approx(0.0135) and fit["beta"] == pytest.approx(6.3e-5)
    assert fit["n_star"] == pytest.approx(0.0135 / 6.3e-5) and fit["rel_rms"] < 1e-9


def test_gpus_flag_launches_that_many_ranks():
    """`bench.py --gpus 2` started directly (no WORLD_SIZE) re-launches itself as two ranks
    under torch.distributed.run; --rank-check makes each rank join a gloo group, agree on the
    slowest rank's time and report, without touching a GPU."""
    import json
    import subprocess
    env = {k: v for k, v in os.environ.items() if k not in ("WORLD_SIZE", "RANK", "LOCAL_RANK", "MASTER_PORT")}
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--gpus", "2", "--rank-check"],
                       capture_output=True, text=True, timeout=240, env=env)
    assert r.returncode == 0, r.stderr[-2000:]
    found = [json.loads(ln)["rank_check"] for ln in r.stdout.splitlines() if ln.startswith('{"rank_check"')]
    assert len(found) == 1                         # rank 0 prints every rank's report on one line
    lines = found[0]
    assert sorted(x["rank"] for x in lines) == [0, 1]
    for x in lines:
        assert x["world"] == 2 and x["gpus"] == 2
        assert x["max_ms"] == 200.0                # the slower rank's value, on every rank
        assert x["launches_all_ranks"] == 5 + 10   # every rank's count added up, on every rank
        assert x["seed"] == x["rank"]


def test_gpus_flag_must_match_world_size():
    import subprocess
    env = dict(os.environ, WORLD_SIZE="2", RANK="0", LOCAL_RANK="0")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--gpus", "3", "--rank-check"],
                       capture_output=True, text=True, timeout=120, env=env)
    assert r.returncode != 0
    assert "does not match WORLD_SIZE=2" in r.stderr
