"""Calibrate the router-bias strength of the skewed synthetic workloads.

Writes moe_synth/workloads.json. Calls only the oracle's router (and the
seeded generator for the logits), never the CUDA path.

  qwen3_mixed          Zipf(s=1.1) bias scaled by alpha: the smallest alpha >= 1
                       (bisection on the seed) for which the hottest expert gets
                       more than 160 assignments and the coldest half of the
                       experts has an expert with fewer than 20.
  dsv3_skewed_prefill  26 hot experts (10% of 256) get +beta: beta bisected on the
                       seed until the hot experts hold 48-52% of the assignments.

Run:  python -m oracle.calibrate_workloads
"""
import json
import os

import numpy as np

import moe_synth
import oracle

OUT = os.path.join(os.path.dirname(moe_synth.__file__), "workloads.json")


def _counts(wl):
    idx, _, _ = oracle.route(moe_synth.host_logits(wl), wl.k)
    return np.bincount(idx.reshape(-1), minlength=wl.E)


def _qwen_ok(wl):
    c = _counts(wl)
    pi = moe_synth.popularity_perm(wl)
    cold = c[pi >= wl.E // 2]
    return bool(c.max() > 160 and cold.min() < 20), c


def calibrate_qwen3(wl):
    ok, c = _qwen_ok(wl.with_(alpha=1.0))
    if ok:
        return 1.0, c
    lo, hi = 1.0, 8.0
    for _ in range(30):
        mid = 0.5 * (lo + hi)
        ok, c = _qwen_ok(wl.with_(alpha=mid))
        if ok:
            hi = mid
        else:
            lo = mid
    ok, c = _qwen_ok(wl.with_(alpha=hi))
    assert ok
    return hi, c


def _hot_share(wl):
    c = _counts(wl)
    pi = moe_synth.popularity_perm(wl)
    return float(c[pi < wl.n_hot].sum()) / float(c.sum()), c


def calibrate_skewed(wl):
    lo, hi = 0.0, 8.0
    for _ in range(40):
        mid = 0.5 * (lo + hi)
        share, c = _hot_share(wl.with_(beta=mid))
        if 0.49 <= share <= 0.51:
            return mid, share, c
        if share < 0.5:
            lo = mid
        else:
            hi = mid
    share, c = _hot_share(wl.with_(beta=mid))
    assert 0.48 <= share <= 0.52
    return mid, share, c


def main():
    wls = moe_synth.workloads()
    alpha, cq = calibrate_qwen3(wls["qwen3_mixed"])
    beta, share, cd = calibrate_skewed(wls["dsv3_skewed_prefill"])
    res = {
        "seed": 0,
        "qwen3_mixed": {"alpha": alpha, "max_count": int(cq.max()),
                        "experts_active": int((cq > 0).sum())},
        "dsv3_skewed_prefill": {"beta": beta, "hot_share": share, "max_count": int(cd.max()),
                                "experts_active": int((cd > 0).sum())},
    }
    with open(OUT, "w") as fh:
        json.dump(res, fh, indent=2)
        fh.write("\n")
    print(json.dumps(res, indent=2))


if __name__ == "__main__":
    main()
