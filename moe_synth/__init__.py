"""Seeded synthetic inputs for the MoE layer (test and benchmark infrastructure).

Shared by the CUDA path's tests/benchmark and by the CPU oracle's tests. It
holds no arithmetic of the MoE method: only the input recipe.

Recipe (per workload, seed 0 unless stated):
  x       [T, d]     bf16  ~ N(0, 1)     (Irwin-Hall(4) approximation, see synth.h)
  logits  [T, E]     fp32  ~ N(0, 1) + bias[e]
  w13     [E, 2f, d] bf16  ~ N(0, 0.02)  rows 0..f-1 = gate, f..2f-1 = up
  w2      [E, d, f]  bf16  ~ N(0, 0.02)
  w13s    [2f, d], w2s [d, f]  (shared expert, when n_shared = 1) ~ N(0, 0.02)

The router bias gives the skew the workloads name:
  zipf : bias[e] = -alpha * s * ln(1 + pi(e))   (pi = seeded permutation of 0..E-1,
         so popular experts are scattered over the logical ranks)
  hot  : bias[e] = beta if pi(e) < n_hot else 0  (n_hot hot experts)
alpha and beta are calibrated per seed (stored in workloads.json beside this file).

Every element is a pure function of (seed, tensor, index): the same values come
out of the host fill (numpy) and the device fill (torch CUDA tensor), bit for bit.
"""
from __future__ import annotations

import ctypes
import dataclasses
import json
import math
import os
import subprocess
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_DIR = os.path.join(_HERE, "lib")
_LIB_PATH = os.path.join(_LIB_DIR, "libmoe_synth.so")
_SRCS = [os.path.join(_HERE, "synth.cu"), os.path.join(_HERE, "synth.h")]

X, LOGITS, W13, W2, W13S, W2S, PERM = 1, 2, 3, 4, 5, 6, 7
IH4_SIGMA = 37837.2265747413
W_STD = 0.02


def build(force: bool = False) -> str:
    """Compile libmoe_synth.so in-tree (host fills + sm_100a device fills)."""
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= max(os.path.getmtime(s) for s in _SRCS)):
        return _LIB_PATH
    os.makedirs(_LIB_DIR, exist_ok=True)
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    cmd = ["nvcc", "-O3", "-std=c++17", "-shared", "-Xcompiler", "-fPIC,-fopenmp,-ffp-contract=off",
           "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo",
           os.path.join(_HERE, "synth.cu"), "-o", tmp, "-lgomp"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


_lib = None


def lib():
    global _lib
    if _lib is None:
        L = ctypes.CDLL(build())
        u64, u32, f32, vp = ctypes.c_uint64, ctypes.c_uint32, ctypes.c_float, ctypes.c_void_p
        L.synth_bits_at.restype = u64
        L.synth_bits_at.argtypes = [u64, u32, u64]
        L.synth_fill_normal_bf16_host.restype = ctypes.c_int
        L.synth_fill_normal_bf16_host.argtypes = [vp, u64, u64, u32, u64, f32]
        L.synth_fill_logits_host.restype = ctypes.c_int
        L.synth_fill_logits_host.argtypes = [vp, u64, u32, u64, u32, u64, f32, vp]
        L.synth_fill_normal_bf16_device.restype = ctypes.c_int
        L.synth_fill_normal_bf16_device.argtypes = [vp, u64, u64, u32, u64, f32, vp]
        L.synth_fill_logits_device.restype = ctypes.c_int
        L.synth_fill_logits_device.argtypes = [vp, u64, u32, u64, u32, u64, f32, vp, vp]
        _lib = L
    return _lib


# ---------------------------------------------------------------------------
# workloads
# ---------------------------------------------------------------------------

@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    T: int
    d: int
    E: int
    k: int
    f: int
    R: int
    n_shared: int = 0
    bias_kind: str = "none"     # none | zipf | hot
    zipf_s: float = 0.0
    alpha: float = 1.0
    n_hot: int = 0
    beta: float = 0.0
    seed: int = 0

    @property
    def A(self) -> int:
        return self.T * self.k

    def with_(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)

    def describe(self) -> dict:
        return dataclasses.asdict(self)


def _calibration() -> dict:
    p = os.path.join(_HERE, "workloads.json")
    if os.path.exists(p):
        with open(p) as fh:
            return json.load(fh)
    return {}


def workloads() -> dict:
    cal = _calibration()
    alpha_q = cal.get("qwen3_mixed", {}).get("alpha", 1.0)
    beta_d = cal.get("dsv3_skewed_prefill", {}).get("beta", 2.0)
    w = [
        Workload("tiny", T=256, d=512, E=8, k=2, f=1024, R=2),
        Workload("mixtral_prefill", T=4096, d=4096, E=8, k=2, f=14336, R=4, bias_kind="zipf", zipf_s=1.0),
        Workload("dsv3_decode", T=128, d=7168, E=256, k=8, f=2048, R=8, n_shared=1,
                 bias_kind="zipf", zipf_s=1.2),
        Workload("qwen3_mixed", T=512, d=4096, E=128, k=8, f=1536, R=8, bias_kind="zipf", zipf_s=1.1,
                 alpha=alpha_q),
        Workload("dsv3_skewed_prefill", T=16384, d=7168, E=256, k=8, f=2048, R=8, n_shared=1,
                 bias_kind="hot", n_hot=26, beta=beta_d),
    ]
    return {x.name: x for x in w}


def workload(name: str) -> Workload:
    return workloads()[name]


def popularity_perm(wl: Workload) -> np.ndarray:
    """pi: expert e -> popularity rank (0 = most popular), a seeded permutation."""
    L = lib()
    keys = np.array([L.synth_bits_at(wl.seed, PERM, e) for e in range(wl.E)], dtype=np.uint64)
    order = np.argsort(keys, kind="stable")
    pi = np.empty(wl.E, dtype=np.int64)
    pi[order] = np.arange(wl.E)
    return pi


def router_bias(wl: Workload) -> np.ndarray:
    if wl.bias_kind == "none":
        return np.zeros(wl.E, dtype=np.float32)
    pi = popularity_perm(wl)
    if wl.bias_kind == "zipf":
        return np.array([0.0 - wl.alpha * wl.zipf_s * math.log1p(float(p)) for p in pi], dtype=np.float32)
    if wl.bias_kind == "hot":
        return np.where(pi < wl.n_hot, np.float32(wl.beta), np.float32(0.0)).astype(np.float32)
    raise ValueError(wl.bias_kind)


def _c_unit() -> np.float32:
    return np.float32(1.0 / IH4_SIGMA)


def _c_w() -> np.float32:
    return np.float32(W_STD / IH4_SIGMA)


# ---------------------------------------------------------------------------
# host fills (numpy)
# ---------------------------------------------------------------------------

def _host_bf16(n: int, seed: int, tid: int, offset: int, c: np.float32) -> np.ndarray:
    out = np.empty(n, dtype=np.uint16)
    rc = lib().synth_fill_normal_bf16_host(out.ctypes.data, n, seed, tid, offset, float(c))
    assert rc == 0
    return out


def host_x(wl: Workload, rows: Optional[np.ndarray] = None) -> np.ndarray:
    """x as bf16 bit patterns, [T, d] (or the listed token rows)."""
    if rows is None:
        return _host_bf16(wl.T * wl.d, wl.seed, X, 0, _c_unit()).reshape(wl.T, wl.d)
    return np.stack([_host_bf16(wl.d, wl.seed, X, int(t) * wl.d, _c_unit()) for t in rows]) if len(rows) else \
        np.zeros((0, wl.d), np.uint16)


def host_logits(wl: Workload, rows: Optional[np.ndarray] = None) -> np.ndarray:
    bias = router_bias(wl)
    L = lib()
    if rows is None:
        out = np.empty((wl.T, wl.E), dtype=np.float32)
        assert L.synth_fill_logits_host(out.ctypes.data, wl.T, wl.E, wl.seed, LOGITS, 0, float(_c_unit()),
                                        bias.ctypes.data) == 0
        return out
    out = np.empty((len(rows), wl.E), dtype=np.float32)
    for i, t in enumerate(rows):
        assert L.synth_fill_logits_host(out[i:].ctypes.data, 1, wl.E, wl.seed, LOGITS, int(t), float(_c_unit()),
                                        bias.ctypes.data) == 0
    return out


def host_w13(wl: Workload, expert: Optional[int] = None) -> np.ndarray:
    per = 2 * wl.f * wl.d
    if expert is None:
        return _host_bf16(wl.E * per, wl.seed, W13, 0, _c_w()).reshape(wl.E, 2 * wl.f, wl.d)
    return _host_bf16(per, wl.seed, W13, expert * per, _c_w()).reshape(2 * wl.f, wl.d)


def host_w2(wl: Workload, expert: Optional[int] = None) -> np.ndarray:
    per = wl.d * wl.f
    if expert is None:
        return _host_bf16(wl.E * per, wl.seed, W2, 0, _c_w()).reshape(wl.E, wl.d, wl.f)
    return _host_bf16(per, wl.seed, W2, expert * per, _c_w()).reshape(wl.d, wl.f)


def host_w13s(wl: Workload) -> np.ndarray:
    return _host_bf16(2 * wl.f * wl.d, wl.seed, W13S, 0, _c_w()).reshape(2 * wl.f, wl.d)


def host_w2s(wl: Workload) -> np.ndarray:
    return _host_bf16(wl.d * wl.f, wl.seed, W2S, 0, _c_w()).reshape(wl.d, wl.f)


# ---------------------------------------------------------------------------
# device fills (torch CUDA tensors)
# ---------------------------------------------------------------------------

def device_inputs(wl: Workload, device="cuda", weights: bool = True) -> dict:
    """All inputs of the workload as CUDA tensors, filled on the device."""
    import torch
    L = lib()
    stream = torch.cuda.current_stream(device).cuda_stream
    out = {}

    def bf16(shape, tid, c):
        t = torch.empty(shape, dtype=torch.bfloat16, device=device)
        if t.numel():
            assert L.synth_fill_normal_bf16_device(t.data_ptr(), t.numel(), wl.seed, tid, 0, float(c), stream) == 0
        return t

    out["x"] = bf16((wl.T, wl.d), X, _c_unit())
    bias = torch.from_numpy(router_bias(wl)).to(device)
    lg = torch.empty((wl.T, wl.E), dtype=torch.float32, device=device)
    if lg.numel():
        assert L.synth_fill_logits_device(lg.data_ptr(), wl.T, wl.E, wl.seed, LOGITS, 0, float(_c_unit()),
                                          bias.data_ptr(), stream) == 0
    out["logits"] = lg
    if weights:
        out["w13"] = bf16((wl.E, 2 * wl.f, wl.d), W13, _c_w())
        out["w2"] = bf16((wl.E, wl.d, wl.f), W2, _c_w())
        if wl.n_shared:
            out["w13s"] = bf16((2 * wl.f, wl.d), W13S, _c_w())
            out["w2s"] = bf16((wl.d, wl.f), W2S, _c_w())
    torch.cuda.synchronize(device)
    return out


def device_expert_weights(wl: Workload, e0: int, e1: int, device="cuda") -> dict:
    """w13 [e1-e0, 2f, d] and w2 [e1-e0, d, f] of experts e0..e1-1 (and the shared expert's, if any),
    filled on the device with the same values as the full tensors' rows (expert parallelism:
    every rank holds its own experts only)."""
    import torch
    L = lib()
    stream = torch.cuda.current_stream(device).cuda_stream
    out = {}

    def bf16(shape, tid, offset):
        t = torch.empty(shape, dtype=torch.bfloat16, device=device)
        if t.numel():
            assert L.synth_fill_normal_bf16_device(t.data_ptr(), t.numel(), wl.seed, tid, offset, float(_c_w()),
                                                   stream) == 0
        return t

    n = e1 - e0
    out["w13"] = bf16((n, 2 * wl.f, wl.d), W13, e0 * 2 * wl.f * wl.d)
    out["w2"] = bf16((n, wl.d, wl.f), W2, e0 * wl.d * wl.f)
    if wl.n_shared:
        out["w13s"] = bf16((2 * wl.f, wl.d), W13S, 0)
        out["w2s"] = bf16((wl.d, wl.f), W2S, 0)
    torch.cuda.synchronize(device)
    return out


def bf16_to_f32(a: np.ndarray) -> np.ndarray:
    """Exact upcast of bf16 bit patterns."""
    return (a.astype(np.uint32) << 16).view(np.float32)
