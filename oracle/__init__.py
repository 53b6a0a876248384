"""CPU oracle of the MoE layer (ctypes binding of moe_oracle.cpp).

TEST INFRASTRUCTURE: only the tests, the smoke check and the benchmark's CPU
baseline leg import this package. It shares no code with the CUDA path.

Every function takes and returns numpy arrays. bf16 tensors are uint16 bit
patterns; floating-point results are fp64.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_DIR = os.path.join(_HERE, "lib")
_LIB_PATH = os.path.join(_LIB_DIR, "libmoe_oracle.so")
_SRC = os.path.join(_HERE, "moe_oracle.cpp")


def build(force: bool = False) -> str:
    """Compile the oracle with g++ (plain -O2, OpenMP over rows)."""
    if not force and os.path.exists(_LIB_PATH) and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC):
        return _LIB_PATH
    os.makedirs(_LIB_DIR, exist_ok=True)
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    subprocess.run(["g++", "-std=c++17", "-O2", "-fopenmp", "-fPIC", "-shared", _SRC, "-o", tmp], check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


_lib = None


def lib():
    global _lib
    if _lib is None:
        L = ctypes.CDLL(build())
        i64, i32, vp = ctypes.c_int64, ctypes.c_int32, ctypes.c_void_p
        L.oracle_route.restype = i64
        L.oracle_route.argtypes = [i64, i32, i32, vp, vp, vp]
        L.oracle_dispatch.restype = i64
        L.oracle_dispatch.argtypes = [i64, i32, i32, i32, vp, vp, vp, vp, vp, vp, vp, vp]
        L.oracle_dispatch_capacity.restype = i64
        L.oracle_dispatch_capacity.argtypes = [i64, i32, i32, i32, i32, vp, vp, vp, vp, vp, vp, vp, vp, vp]
        L.oracle_permute_rows.restype = None
        L.oracle_permute_rows.argtypes = [i64, i32, i32, vp, vp, vp]
        L.oracle_swiglu.restype = None
        L.oracle_swiglu.argtypes = [i64, i32, i32, vp, vp, vp, vp]
        L.oracle_expert_ffn.restype = None
        L.oracle_expert_ffn.argtypes = [i64, i32, i32, i32, i32, vp, vp, vp, vp, vp, vp, vp, vp, vp]
        L.oracle_combine.restype = None
        L.oracle_combine.argtypes = [i64, i32, i32, vp, vp, vp, vp, vp]
        L.oracle_naive_token_loop.restype = None
        L.oracle_naive_token_loop.argtypes = [i64, i32, i32, i32, i32, i32, vp, vp, vp, vp, vp, vp, vp, vp]
        _lib = L
    return _lib


def _c(a, dtype):
    a = np.ascontiguousarray(a, dtype=dtype)
    return a, a.ctypes.data


def route(logits: np.ndarray, k: int):
    """-> (topk_idx [T,k] int32, topk_gate [T,k] fp32, nan_count)."""
    logits, lp = _c(logits, np.float32)
    T, E = logits.shape
    idx = np.empty((T, k), np.int32)
    gate = np.empty((T, k), np.float32)
    n = lib().oracle_route(T, E, k, lp, idx.ctypes.data, gate.ctypes.data)
    return idx, gate, int(n)


def dispatch(topk_idx: np.ndarray, E: int, R: int, capacity: int = 0) -> dict:
    """capacity > 0: each expert keeps only its first `capacity` assignments."""
    topk_idx, ip = _c(topk_idx, np.int32)
    T, k = topk_idx.shape
    A = T * k
    out = dict(expert_counts=np.empty(E, np.int32), expert_offsets=np.empty(E + 1, np.int32),
               rank_counts=np.empty(R, np.int32), rank_offsets=np.empty(R + 1, np.int32),
               row_src=np.empty(A, np.int32), assign_row=np.empty(A, np.int32),
               imbalance=np.empty(2, np.float32))
    dropped = ctypes.c_int64(0)
    bad = lib().oracle_dispatch_capacity(T, E, k, R, capacity, ip, *(out[n].ctypes.data for n in (
        "expert_counts", "expert_offsets", "rank_counts", "rank_offsets", "row_src", "assign_row", "imbalance")),
        ctypes.addressof(dropped))
    out["skipped"] = int(bad)
    out["dropped"] = int(dropped.value)
    return out


def permute_rows(x: np.ndarray, row_src: np.ndarray, k: int) -> np.ndarray:
    x, xp = _c(x, np.uint16)
    row_src, rp = _c(row_src, np.int32)
    d = x.shape[1]
    xperm = np.zeros((row_src.shape[0], d), np.uint16)
    lib().oracle_permute_rows(row_src.shape[0], k, d, xp, rp, xperm.ctypes.data)
    return xperm


def swiglu(xrows: np.ndarray, w13: np.ndarray, w2: np.ndarray) -> np.ndarray:
    """One expert's SwiGLU FFN of bf16 rows -> fp64 [n, d]."""
    xrows, xp = _c(xrows, np.uint16)
    w13, w13p = _c(w13, np.uint16)
    w2, w2p = _c(w2, np.uint16)
    n, d = xrows.shape
    f = w2.shape[1]
    assert w13.shape == (2 * f, d) and w2.shape == (d, f)
    y = np.empty((n, d), np.float64)
    lib().oracle_swiglu(n, d, f, xp, w13p, w2p, y.ctypes.data)
    return y


def expert_ffn(x_perm, offsets, w13, w2, x=None, w13s=None, w2s=None):
    """-> (y_perm fp64 [A, d], y_shared fp64 [T, d] or None)."""
    x_perm, xpp = _c(x_perm, np.uint16)
    offsets, op = _c(offsets, np.int32)
    w13, w13p = _c(w13, np.uint16)
    w2, w2p = _c(w2, np.uint16)
    E, f2, d = w13.shape
    f = f2 // 2
    y_perm = np.zeros((x_perm.shape[0], d), np.float64)
    n_shared = 1 if w13s is not None else 0
    if n_shared:
        x, xp = _c(x, np.uint16)
        w13s, w13sp = _c(w13s, np.uint16)
        w2s, w2sp = _c(w2s, np.uint16)
        T = x.shape[0]
        y_shared = np.empty((T, d), np.float64)
        ysp = y_shared.ctypes.data
    else:
        T, xp, w13sp, w2sp, y_shared, ysp = 0, None, None, None, None, None
    lib().oracle_expert_ffn(T, d, E, f, n_shared, xpp, op, w13p, w2p, xp, w13sp, w2sp, y_perm.ctypes.data, ysp)
    return y_perm, y_shared


def combine(y_perm, assign_row, gate, y_shared=None) -> np.ndarray:
    y_perm, yp = _c(y_perm, np.float64)
    assign_row, ap = _c(assign_row, np.int32)
    gate, gp = _c(gate, np.float32)
    T, k = gate.shape
    d = y_perm.shape[1]
    ys = None
    if y_shared is not None:
        y_shared, ys = _c(y_shared, np.float64)
    out = np.empty((T, d), np.float64)
    lib().oracle_combine(T, k, d, yp, ap, gp, ys, out.ctypes.data)
    return out


def naive_token_loop(x, topk_idx, gate, w13, w2, w13s=None, w2s=None) -> np.ndarray:
    x, xp = _c(x, np.uint16)
    topk_idx, ip = _c(topk_idx, np.int32)
    gate, gp = _c(gate, np.float32)
    w13, w13p = _c(w13, np.uint16)
    w2, w2p = _c(w2, np.uint16)
    T, d = x.shape
    E, f2, _ = w13.shape
    k = topk_idx.shape[1]
    n_shared = 1 if w13s is not None else 0
    w13sp = w2sp = None
    if n_shared:
        w13s, w13sp = _c(w13s, np.uint16)
        w2s, w2sp = _c(w2s, np.uint16)
    out = np.empty((T, d), np.float64)
    lib().oracle_naive_token_loop(T, d, E, k, f2 // 2, n_shared, xp, ip, gp, w13p, w2p, w13sp, w2sp,
                                  out.ctypes.data)
    return out


def layer(x, logits, w13, w2, k, R, w13s=None, w2s=None, capacity: int = 0) -> dict:
    """The whole layer: route -> dispatch -> permute -> expert FFN -> combine."""
    E = w13.shape[0]
    idx, gate, nan = route(logits, k)
    disp = dispatch(idx, E, R, capacity)
    x_perm = permute_rows(x, disp["row_src"], k)
    y_perm, y_shared = expert_ffn(x_perm, disp["expert_offsets"], w13, w2, x, w13s, w2s)
    out = combine(y_perm, disp["assign_row"], gate, y_shared)
    res = dict(topk_idx=idx, topk_gate=gate, nan_count=nan, x_perm=x_perm, y_perm=y_perm, y_shared=y_shared,
               out=out)
    res.update(disp)
    return res
