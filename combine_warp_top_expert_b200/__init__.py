"""B200-native MoE layer: route -> dispatch -> grouped SwiGLU FFN -> combine.

Thin ctypes binding of libmoe_b200.so (the C ABI in include/moe.h). The
functions keep the ABI's names and only marshal arguments: every step runs in
the library's CUDA kernels. PyTorch supplies device memory and streams.
There is no CPU fallback: if the library is missing or cannot be loaded,
every call raises.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass
from typing import Optional

from . import build as _build

MOE_OK, MOE_ERR_INVALID_ARG, MOE_ERR_UNSUPPORTED, MOE_ERR_WORKSPACE, MOE_ERR_CUDA = range(5)
MOE_DEV_NAN_LOGIT, MOE_DEV_BOUNDS, MOE_DEV_TIMEOUT, MOE_DEV_COUNT_MISMATCH = 1, 2, 4, 8

LIB_PATH = _build.LIB_PATH

ABI_FUNCTIONS = (
    "moe_workspace_bytes", "moe_clear_status", "moe_get_status", "moe_route", "moe_dispatch", "moe_expert_ffn",
    "moe_combine", "moe_layer", "moe_status_string", "moe_last_cuda_error", "moe_set_wait_timeout_ns",
    "moe_expert_gate_up", "moe_expert_down", "moe_dispatch_static", "moe_set_gemm_policy",
    "moe_set_test_stall", "moe_expert_gate_up_gather", "moe_capacity_for", "moe_dispatch_static_scratch",
    "moe_set_pdl", "moe_ep_exchange_counts", "moe_ep_dispatch", "moe_ep_signal", "moe_ep_wait", "moe_ep_combine",
    "moe_ep_plan_host", "moe_expert_down_combine", "moe_set_fused_combine", "moe_set_dispatch_path",
    "moe_kernel_launches",
)
EP_SLOT_COUNTS, EP_SLOT_ROWS, EP_SLOT_OUTPUTS, EP_SLOT_DONE = 0, 1, 2, 3
GEMM_AUTO, GEMM_SINGLE, GEMM_PAIR = 0, 1, 2
DISPATCH_AUTO, DISPATCH_TWO_PASS, DISPATCH_ONE_PASS = 0, 1, 2


class MoEError(RuntimeError):
    def __init__(self, fn: str, code: int, msg: str):
        super().__init__(f"{fn} failed: {msg}")
        self.code = code


class moe_shape_t(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in ("T", "d", "E", "k", "f", "R", "n_shared", "capacity")]


class moe_layer_buffers_t(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in (
        "logits", "x", "w13", "w2", "w13s", "w2s", "topk_idx", "topk_gate", "expert_counts", "expert_offsets",
        "rank_counts", "rank_offsets", "row_src", "assign_row", "x_perm", "imbalance", "y_perm", "y_shared", "out")]


class moe_ep_peers_t(ctypes.Structure):
    _fields_ = [("counts", ctypes.c_void_p), ("recv_rows", ctypes.c_void_p), ("y_rows", ctypes.c_void_p),
                ("flags", ctypes.c_void_p), ("rows_cap", ctypes.c_int64)]


_lib = None


def load(build_if_missing: bool = True) -> ctypes.CDLL:
    """Load the in-tree libmoe_b200.so (building it with nvcc if absent)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH) or (build_if_missing and not _build.up_to_date()):
        if not build_if_missing:
            raise RuntimeError(f"libmoe_b200.so not built ({LIB_PATH}); run python -m combine_warp_top_expert_b200.build")
        _build.build()
    L = ctypes.CDLL(LIB_PATH)
    vp, sz, st = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int
    shp = ctypes.POINTER(moe_shape_t)
    L.moe_workspace_bytes.restype = sz
    L.moe_workspace_bytes.argtypes = [shp]
    L.moe_clear_status.restype = st
    L.moe_clear_status.argtypes = [vp, sz, vp]
    L.moe_get_status.restype = st
    L.moe_get_status.argtypes = [vp, sz, ctypes.POINTER(ctypes.c_uint32), vp]
    L.moe_route.restype = st
    L.moe_route.argtypes = [shp, vp, vp, vp, vp, sz, vp]
    L.moe_dispatch.restype = st
    L.moe_dispatch.argtypes = [shp] + [vp] * 10 + [vp, sz, vp]
    L.moe_dispatch_static.restype = st
    L.moe_dispatch_static.argtypes = [shp] + [vp] * 11 + [vp]
    L.moe_dispatch_static_scratch.restype = st
    L.moe_dispatch_static_scratch.argtypes = [ctypes.POINTER(ctypes.c_void_p), ctypes.POINTER(ctypes.c_size_t)]
    L.moe_capacity_for.restype = ctypes.c_int32
    L.moe_capacity_for.argtypes = [ctypes.c_int64, ctypes.c_int64, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32]
    L.moe_expert_ffn.restype = st
    L.moe_expert_ffn.argtypes = [shp] + [vp] * 9 + [vp, sz, vp]
    L.moe_expert_gate_up.restype = st
    L.moe_expert_gate_up.argtypes = [shp] + [vp] * 5 + [vp, sz, vp]
    L.moe_expert_gate_up_gather.restype = st
    L.moe_expert_gate_up_gather.argtypes = [shp] + [vp] * 5 + [vp, sz, vp]
    L.moe_expert_down.restype = st
    L.moe_expert_down.argtypes = [shp] + [vp] * 5 + [vp, sz, vp]
    L.moe_combine.restype = st
    L.moe_combine.argtypes = [shp] + [vp] * 5 + [vp, sz, vp]
    L.moe_layer.restype = st
    L.moe_layer.argtypes = [shp, ctypes.POINTER(moe_layer_buffers_t), vp, sz, vp]
    L.moe_status_string.restype = ctypes.c_char_p
    L.moe_status_string.argtypes = [st]
    L.moe_last_cuda_error.restype = ctypes.c_char_p
    L.moe_last_cuda_error.argtypes = []
    L.moe_set_gemm_policy.restype = ctypes.c_int
    L.moe_set_gemm_policy.argtypes = [ctypes.c_int]
    epp = ctypes.POINTER(moe_ep_peers_t)
    i32, u64 = ctypes.c_int32, ctypes.c_uint64
    L.moe_ep_exchange_counts.restype = st
    L.moe_ep_exchange_counts.argtypes = [shp, i32, u64, vp, vp, epp, vp, sz, vp]
    L.moe_ep_dispatch.restype = st
    L.moe_ep_dispatch.argtypes = [shp, i32, u64, vp, vp, vp, vp, epp, vp, sz, vp]
    L.moe_ep_signal.restype = st
    L.moe_ep_signal.argtypes = [i32, i32, i32, u64, epp, vp]
    L.moe_ep_wait.restype = st
    L.moe_ep_wait.argtypes = [i32, i32, i32, u64, epp, vp, sz, vp]
    L.moe_ep_combine.restype = st
    L.moe_ep_combine.argtypes = [shp, i32, u64, vp, vp, vp, vp, vp, epp, vp, sz, vp]
    L.moe_ep_plan_host.restype = i32
    L.moe_ep_plan_host.argtypes = [i32, i32, i32, i32, vp, vp, vp, vp]
    L.moe_expert_down_combine.restype = st
    L.moe_expert_down_combine.argtypes = [shp] + [vp] * 9 + [vp, sz, vp]
    L.moe_set_fused_combine.restype = ctypes.c_int
    L.moe_set_fused_combine.argtypes = [ctypes.c_int]
    L.moe_set_pdl.restype = ctypes.c_int
    L.moe_set_pdl.argtypes = [ctypes.c_int]
    L.moe_set_dispatch_path.restype = ctypes.c_int
    L.moe_set_dispatch_path.argtypes = [ctypes.c_int]
    L.moe_kernel_launches.restype = ctypes.c_uint64
    L.moe_kernel_launches.argtypes = []
    L.moe_set_test_stall.restype = ctypes.c_int
    L.moe_set_test_stall.argtypes = [ctypes.c_int]
    L.moe_set_wait_timeout_ns.restype = ctypes.c_uint64
    L.moe_set_wait_timeout_ns.argtypes = [ctypes.c_uint64]
    _lib = L
    return L


def _check(fn: str, code: int):
    if code != MOE_OK:
        L = load()
        msg = L.moe_status_string(code).decode()
        if code == MOE_ERR_CUDA:
            msg += " (" + L.moe_last_cuda_error().decode() + ")"
        raise MoEError(fn, code, msg)


@dataclass(frozen=True)
class Shape:
    T: int
    d: int
    E: int
    k: int
    f: int
    R: int
    n_shared: int = 0
    capacity: int = 0  # per-expert assignment limit, 0 = none

    @property
    def A(self) -> int:
        return self.T * self.k

    def c(self) -> moe_shape_t:
        return moe_shape_t(self.T, self.d, self.E, self.k, self.f, self.R, self.n_shared, self.capacity)


def capacity_for(C: float, T: int, k: int, E: int) -> int:
    """Per-expert capacity of a capacity factor C, computed by moe_capacity_for in the
    library (C is passed as an exact fraction with a denominator of at most 2^20)."""
    from fractions import Fraction
    q = Fraction(C).limit_denominator(1 << 20)
    c = load().moe_capacity_for(q.numerator, q.denominator, T, k, E)
    if c < 0:
        raise ValueError(f"no capacity for C={C}, T={T}, k={k}, E={E}")
    return c


def _ptr(t) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _stream(stream) -> Optional[int]:
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream


def _ws(ws):
    """(pointer, bytes) of a workspace: a contiguous uint8 CUDA tensor such as
    new_workspace returns. A host tensor would hand a host address to the kernels,
    so it is refused here."""
    import torch
    if ws is None:
        raise ValueError("ws must be a CUDA uint8 tensor (see new_workspace)")
    _dev(ws, torch.uint8, None, "ws")
    return ws.data_ptr(), ws.numel()


def _dev(t, dtype, shape, name, device: bool = True):
    """dtype, contiguity and shape of a buffer, then (device=True) that it lives on a CUDA device."""
    if t is None:
        return
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    if device and not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")


def workspace_bytes(shape: Shape) -> int:
    n = load().moe_workspace_bytes(ctypes.byref(shape.c()))
    if n == 0:
        raise MoEError("moe_workspace_bytes", MOE_ERR_INVALID_ARG, "invalid shape")
    return n


def new_workspace(shape: Shape, device="cuda"):
    """A zeroed device workspace (the status word starts clear)."""
    import torch
    return torch.zeros(workspace_bytes(shape), dtype=torch.uint8, device=device)


def clear_status(ws, stream=None):
    _check("moe_clear_status", load().moe_clear_status(*_ws(ws), _stream(stream)))


def get_status(ws, stream=None) -> int:
    bits = ctypes.c_uint32(0)
    _check("moe_get_status", load().moe_get_status(*_ws(ws), ctypes.byref(bits), _stream(stream)))
    return bits.value


def set_wait_timeout_ns(ns: int) -> int:
    return load().moe_set_wait_timeout_ns(ns)


def set_test_stall(enable: bool) -> int:
    """Test hook of the bounded-wait path (see moe_set_test_stall in include/moe.h)."""
    return load().moe_set_test_stall(1 if enable else 0)


def set_pdl(enable: bool) -> int:
    """Programmatic dependent launch of the library's kernels on (default) or off (see moe_set_pdl)."""
    return load().moe_set_pdl(1 if enable else 0)


def kernel_launches() -> int:
    """Kernels the library has launched in this process so far (see moe_kernel_launches)."""
    return int(load().moe_kernel_launches())


def set_dispatch_path(path: int) -> int:
    """DISPATCH_AUTO, DISPATCH_TWO_PASS or DISPATCH_ONE_PASS (see moe_set_dispatch_path); returns
    the previous path, -1 if `path` is unknown."""
    return load().moe_set_dispatch_path(int(path))


def set_fused_combine(enable: bool) -> int:
    """moe_layer folds the combine into the down GEMM's epilogue (see moe_set_fused_combine)."""
    return load().moe_set_fused_combine(1 if enable else 0)


def set_gemm_policy(policy: int) -> int:
    """GEMM_AUTO (chosen from the shape), GEMM_SINGLE (128-row single-CTA tiles) or GEMM_PAIR
    (256 x 256 CTA-pair tiles, a group's last block of <= 128 rows as a half-height pair tile)."""
    old = load().moe_set_gemm_policy(policy)
    if old < 0:
        raise ValueError(f"unknown GEMM policy {policy}")
    return old


def moe_route(shape: Shape, logits, topk_idx, topk_gate, ws, stream=None):
    import torch
    _dev(logits, torch.float32, (shape.T, shape.E), "logits")
    _dev(topk_idx, torch.int32, (shape.T, shape.k), "topk_idx")
    _dev(topk_gate, torch.float32, (shape.T, shape.k), "topk_gate")
    _check("moe_route", load().moe_route(ctypes.byref(shape.c()), _ptr(logits), _ptr(topk_idx), _ptr(topk_gate),
                                         *_ws(ws), _stream(stream)))


def moe_dispatch(shape: Shape, x, topk_idx, expert_counts, expert_offsets, rank_counts, rank_offsets, row_src,
                 assign_row, x_perm, imbalance, ws, stream=None):
    import torch
    i32, bf = torch.int32, torch.bfloat16
    _dev(x, bf, (shape.T, shape.d), "x")
    _dev(topk_idx, i32, (shape.T, shape.k), "topk_idx")
    _dev(expert_counts, i32, (shape.E,), "expert_counts")
    _dev(expert_offsets, i32, (shape.E + 1,), "expert_offsets")
    _dev(rank_counts, i32, (shape.R,), "rank_counts")
    _dev(rank_offsets, i32, (shape.R + 1,), "rank_offsets")
    _dev(row_src, i32, (shape.A,), "row_src")
    _dev(assign_row, i32, (shape.A,), "assign_row")
    _dev(x_perm, bf, (shape.A, shape.d), "x_perm")  # None: indices only
    _dev(imbalance, torch.float32, (2,), "imbalance")
    _check("moe_dispatch", load().moe_dispatch(
        ctypes.byref(shape.c()), _ptr(x), _ptr(topk_idx), _ptr(expert_counts), _ptr(expert_offsets),
        _ptr(rank_counts), _ptr(rank_offsets), _ptr(row_src), _ptr(assign_row), _ptr(x_perm), _ptr(imbalance),
        *_ws(ws), _stream(stream)))


def moe_expert_ffn(shape: Shape, x_perm, expert_offsets, w13, w2, x, w13s, w2s, y_perm, y_shared, ws, stream=None):
    import torch
    bf = torch.bfloat16
    _dev(x_perm, bf, (shape.A, shape.d), "x_perm")
    _dev(expert_offsets, torch.int32, (shape.E + 1,), "expert_offsets")
    _dev(w13, bf, (shape.E, 2 * shape.f, shape.d), "w13")
    _dev(w2, bf, (shape.E, shape.d, shape.f), "w2")
    _dev(y_perm, bf, (shape.A, shape.d), "y_perm")
    if shape.n_shared:
        _dev(x, bf, (shape.T, shape.d), "x")
        _dev(w13s, bf, (2 * shape.f, shape.d), "w13s")
        _dev(w2s, bf, (shape.d, shape.f), "w2s")
        _dev(y_shared, bf, (shape.T, shape.d), "y_shared")
    _check("moe_expert_ffn", load().moe_expert_ffn(
        ctypes.byref(shape.c()), _ptr(x_perm), _ptr(expert_offsets), _ptr(w13), _ptr(w2), _ptr(x), _ptr(w13s),
        _ptr(w2s), _ptr(y_perm), _ptr(y_shared), *_ws(ws), _stream(stream)))


def moe_expert_gate_up(shape: Shape, x_perm, expert_offsets, w13, x, w13s, ws, stream=None):
    """GEMM1 + SwiGLU into the workspace (first half of moe_expert_ffn)."""
    import torch
    bf = torch.bfloat16
    _dev(x_perm, bf, (shape.A, shape.d), "x_perm")
    _dev(expert_offsets, torch.int32, (shape.E + 1,), "expert_offsets")
    _dev(w13, bf, (shape.E, 2 * shape.f, shape.d), "w13")
    if shape.n_shared:
        _dev(x, bf, (shape.T, shape.d), "x")
        _dev(w13s, bf, (2 * shape.f, shape.d), "w13s")
    _check("moe_expert_gate_up", load().moe_expert_gate_up(
        ctypes.byref(shape.c()), _ptr(x_perm), _ptr(expert_offsets), _ptr(w13), _ptr(x), _ptr(w13s),
        *_ws(ws), _stream(stream)))


def moe_expert_gate_up_gather(shape: Shape, x, row_src, expert_offsets, w13, w13s, ws, stream=None):
    """GEMM1 + SwiGLU gathering its rows from x through row_src (no x_perm)."""
    import torch
    bf = torch.bfloat16
    _dev(x, bf, (shape.T, shape.d), "x")
    _dev(row_src, torch.int32, (shape.A,), "row_src")
    _dev(expert_offsets, torch.int32, (shape.E + 1,), "expert_offsets")
    _dev(w13, bf, (shape.E, 2 * shape.f, shape.d), "w13")
    if shape.n_shared:
        _dev(w13s, bf, (2 * shape.f, shape.d), "w13s")
    _check("moe_expert_gate_up_gather", load().moe_expert_gate_up_gather(
        ctypes.byref(shape.c()), _ptr(x), _ptr(row_src), _ptr(expert_offsets), _ptr(w13), _ptr(w13s),
        *_ws(ws), _stream(stream)))


def moe_expert_down(shape: Shape, expert_offsets, w2, w2s, y_perm, y_shared, ws, stream=None):
    """GEMM2 from the workspace's hidden rows (second half of moe_expert_ffn)."""
    import torch
    bf = torch.bfloat16
    _dev(expert_offsets, torch.int32, (shape.E + 1,), "expert_offsets")
    _dev(w2, bf, (shape.E, shape.d, shape.f), "w2")
    _dev(y_perm, bf, (shape.A, shape.d), "y_perm")
    if shape.n_shared:
        _dev(w2s, bf, (shape.d, shape.f), "w2s")
        _dev(y_shared, bf, (shape.T, shape.d), "y_shared")
    _check("moe_expert_down", load().moe_expert_down(
        ctypes.byref(shape.c()), _ptr(expert_offsets), _ptr(w2), _ptr(w2s), _ptr(y_perm), _ptr(y_shared),
        *_ws(ws), _stream(stream)))


def moe_expert_down_combine(shape: Shape, expert_offsets, w2, w2s, row_src, assign_row, topk_gate, y_perm, y_shared,
                            out, ws, stream=None):
    """GEMM2 with the combine folded into its epilogue: y_perm (y_shared) and out."""
    import torch
    bf = torch.bfloat16
    _dev(expert_offsets, torch.int32, (shape.E + 1,), "expert_offsets")
    _dev(w2, bf, (shape.E, shape.d, shape.f), "w2")
    _dev(row_src, torch.int32, (shape.A,), "row_src")
    _dev(assign_row, torch.int32, (shape.A,), "assign_row")
    _dev(topk_gate, torch.float32, (shape.T, shape.k), "topk_gate")
    _dev(y_perm, bf, (shape.A, shape.d), "y_perm")
    _dev(out, bf, (shape.T, shape.d), "out")
    if shape.n_shared:
        _dev(w2s, bf, (shape.d, shape.f), "w2s")
        _dev(y_shared, bf, (shape.T, shape.d), "y_shared")
    _check("moe_expert_down_combine", load().moe_expert_down_combine(
        ctypes.byref(shape.c()), _ptr(expert_offsets), _ptr(w2), _ptr(w2s), _ptr(row_src), _ptr(assign_row),
        _ptr(topk_gate), _ptr(y_perm), _ptr(y_shared), _ptr(out), *_ws(ws), _stream(stream)))


def moe_combine(shape: Shape, y_perm, assign_row, topk_gate, y_shared, out, ws, stream=None):
    import torch
    bf = torch.bfloat16
    _dev(y_perm, bf, (shape.A, shape.d), "y_perm")
    _dev(assign_row, torch.int32, (shape.A,), "assign_row")
    _dev(topk_gate, torch.float32, (shape.T, shape.k), "topk_gate")
    _dev(y_shared, bf, (shape.T, shape.d), "y_shared")
    _dev(out, bf, (shape.T, shape.d), "out")
    _check("moe_combine", load().moe_combine(
        ctypes.byref(shape.c()), _ptr(y_perm), _ptr(assign_row), _ptr(topk_gate), _ptr(y_shared), _ptr(out),
        *_ws(ws), _stream(stream)))


_LAYER_OUTPUTS = ("topk_idx", "topk_gate", "expert_counts", "expert_offsets", "rank_counts", "rank_offsets",
                  "row_src", "assign_row", "x_perm", "imbalance", "y_perm", "y_shared", "out")


def _layer_output_specs(shape: Shape) -> dict:
    """dtype and shape of every output buffer of moe_layer."""
    import torch
    i32, f32, bf = torch.int32, torch.float32, torch.bfloat16
    T, k, E, R, d, A = shape.T, shape.k, shape.E, shape.R, shape.d, shape.A
    return dict(topk_idx=(i32, (T, k)), topk_gate=(f32, (T, k)), expert_counts=(i32, (E,)),
                expert_offsets=(i32, (E + 1,)), rank_counts=(i32, (R,)), rank_offsets=(i32, (R + 1,)),
                row_src=(i32, (A,)), assign_row=(i32, (A,)), x_perm=(bf, (A, d)), imbalance=(f32, (2,)),
                y_perm=(bf, (A, d)), y_shared=(bf, (T, d)), out=(bf, (T, d)))


def alloc_layer_outputs(shape: Shape, device="cuda", x_perm: bool = True) -> dict:
    """Device buffers for every output of moe_layer (x_perm=False: the layer gathers
    rows of x inside the grouped GEMM and x_perm is not materialised)."""
    import torch
    i32, f32, bf = torch.int32, torch.float32, torch.bfloat16
    T, k, E, R, d, A = shape.T, shape.k, shape.E, shape.R, shape.d, shape.A
    o = dict(
        topk_idx=torch.empty((T, k), dtype=i32, device=device),
        topk_gate=torch.empty((T, k), dtype=f32, device=device),
        expert_counts=torch.empty((E,), dtype=i32, device=device),
        expert_offsets=torch.empty((E + 1,), dtype=i32, device=device),
        rank_counts=torch.empty((R,), dtype=i32, device=device),
        rank_offsets=torch.empty((R + 1,), dtype=i32, device=device),
        row_src=torch.empty((A,), dtype=i32, device=device),
        assign_row=torch.empty((A,), dtype=i32, device=device),
        x_perm=torch.empty((A, d), dtype=bf, device=device) if x_perm else None,
        imbalance=torch.empty((2,), dtype=f32, device=device),
        y_perm=torch.empty((A, d), dtype=bf, device=device),
        y_shared=torch.empty((T, d), dtype=bf, device=device) if shape.n_shared else None,
        out=torch.empty((T, d), dtype=bf, device=device),
    )
    return o


def moe_layer(shape: Shape, logits, x, w13, w2, w13s, w2s, outs: dict, ws, stream=None):
    """The whole layer on one stream, writing every buffer of `outs` (see alloc_layer_outputs)."""
    import torch
    bf = torch.bfloat16
    _dev(logits, torch.float32, (shape.T, shape.E), "logits")
    _dev(x, bf, (shape.T, shape.d), "x")
    _dev(w13, bf, (shape.E, 2 * shape.f, shape.d), "w13")
    _dev(w2, bf, (shape.E, shape.d, shape.f), "w2")
    if shape.n_shared:
        _dev(w13s, bf, (2 * shape.f, shape.d), "w13s")
        _dev(w2s, bf, (shape.d, shape.f), "w2s")
    specs = _layer_output_specs(shape)
    for n, (dtype, shp) in specs.items():  # every buffer's layout first, then where it lives
        if outs.get(n) is None:
            if n == "x_perm" or (n == "y_shared" and not shape.n_shared):
                continue  # x_perm None: rows gathered in GEMM1; no shared expert
            raise ValueError(f"outs[{n!r}] is required")
        _dev(outs[n], dtype, shp, f"outs[{n!r}]", device=False)
    for n, (dtype, shp) in specs.items():
        _dev(outs.get(n), dtype, shp, f"outs[{n!r}]")
    b = moe_layer_buffers_t(_ptr(logits), _ptr(x), _ptr(w13), _ptr(w2), _ptr(w13s), _ptr(w2s),
                            *(_ptr(outs.get(n)) for n in _LAYER_OUTPUTS))
    _check("moe_layer", load().moe_layer(ctypes.byref(shape.c()), ctypes.byref(b), *_ws(ws),
                                         _stream(stream)))
    return outs


class MoELayer:
    """Weights resident on the device plus a reusable workspace and output set."""

    def __init__(self, shape: Shape, w13, w2, w13s=None, w2s=None, device="cuda", gather: bool = False):
        """gather=True: no x_perm; the grouped GEMM gathers the dispatched rows of x itself."""
        self.shape = shape
        self.w13, self.w2, self.w13s, self.w2s = w13, w2, w13s, w2s
        self.gather = gather
        self.ws = new_workspace(shape, device)
        self.outs = alloc_layer_outputs(shape, device, x_perm=not gather)

    def __call__(self, logits, x, stream=None) -> dict:
        return moe_layer(self.shape, logits, x, self.w13, self.w2, self.w13s, self.w2s, self.outs, self.ws, stream)

    def forward_host(self, logits_host, x_host, out_host, stream=None):
        """Asynchronous end-to-end call with HOST tensors (pinned, for DMA).

        Enqueues, and returns without waiting: the copy of this batch's logits and x
        to the device (on a copy-in stream), the layer (on `stream`), and the copy of
        `out` back into out_host (on a copy-out stream). Call sync_host() (or
        torch.cuda.synchronize()) before reading out_host. Successive calls rotate
        between two device staging slots, so one batch's copies overlap its
        neighbours' compute, as in a serving loop; a slot is reused only after its
        previous compute and copy-out have finished (CUDA events)."""
        import torch
        s_comp = stream or torch.cuda.current_stream(self.ws.device)
        if not hasattr(self, "_slots"):
            dev = self.ws.device
            self._slots = [dict(outs=alloc_layer_outputs(self.shape, dev, x_perm=not self.gather),
                                x=torch.empty((self.shape.T, self.shape.d), dtype=torch.bfloat16, device=dev),
                                logits=torch.empty((self.shape.T, self.shape.E), dtype=torch.float32, device=dev),
                                ev_in=torch.cuda.Event(), ev_done=torch.cuda.Event(), ev_out=torch.cuda.Event(),
                                used=False) for _ in range(2)]
            self._s_in = torch.cuda.Stream(dev)
            self._s_out = torch.cuda.Stream(dev)
            self._slot = 0
        c = self._slots[self._slot]
        self._slot ^= 1
        if c["used"]:
            self._s_in.wait_event(c["ev_done"])   # the slot's inputs were consumed by its last compute
            s_comp.wait_event(c["ev_out"])        # the slot's last out has been copied back
        else:
            self._s_in.wait_stream(s_comp)
        c["used"] = True
        with torch.cuda.stream(self._s_in):
            c["logits"].copy_(logits_host, non_blocking=True)
            c["x"].copy_(x_host, non_blocking=True)
            c["ev_in"].record(self._s_in)
        s_comp.wait_event(c["ev_in"])
        moe_layer(self.shape, c["logits"], c["x"], self.w13, self.w2, self.w13s, self.w2s, c["outs"], self.ws, s_comp)
        c["ev_done"].record(s_comp)
        self._s_out.wait_event(c["ev_done"])
        with torch.cuda.stream(self._s_out):
            out_host.copy_(c["outs"]["out"], non_blocking=True)
            c["ev_out"].record(self._s_out)
        self._last_out = c["ev_out"]
        return out_host

    def sync_host(self):
        """Block until the last forward_host's copy-out has landed in host memory."""
        if getattr(self, "_last_out", None) is not None:
            self._last_out.synchronize()


# ---------------------------------------------------------------------------
# expert parallelism across GPUs (include/moe.h, "Expert parallelism across GPUs")
# ---------------------------------------------------------------------------

def ep_plan_host(R: int, E: int, rank: int, capacity: int, counts_all) -> dict:
    """The exchange plan of `rank` from all ranks' expert counts (int32 [R, E], host), as
    moe_ep_plan_host computes it: row_base [E], keep [E], recv_offsets [E/R + 1]."""
    import numpy as np
    c = np.ascontiguousarray(counts_all, dtype=np.int32)
    if c.shape != (R, E):
        raise ValueError(f"counts_all has shape {c.shape}, expected {(R, E)}")
    row_base, keep = np.empty(E, np.int32), np.empty(E, np.int32)
    recv_offsets = np.empty(E // R + 1 if R > 0 and E % R == 0 else 1, np.int32)
    rc = load().moe_ep_plan_host(R, E, rank, capacity, c.ctypes.data, row_base.ctypes.data, keep.ctypes.data,
                                 recv_offsets.ctypes.data)
    if rc != 0:
        raise ValueError(f"invalid plan arguments R={R} E={E} rank={rank} capacity={capacity}")
    return dict(row_base=row_base, keep=keep, recv_offsets=recv_offsets)


def moe_ep_exchange_counts(shape: Shape, rank: int, epoch: int, topk_idx, expert_counts, peers, ws, stream=None):
    import torch
    _dev(topk_idx, torch.int32, (shape.T, shape.k), "topk_idx")
    _dev(expert_counts, torch.int32, (shape.E,), "expert_counts")
    _check("moe_ep_exchange_counts", load().moe_ep_exchange_counts(
        ctypes.byref(shape.c()), rank, epoch, _ptr(topk_idx), _ptr(expert_counts), ctypes.byref(peers.c()),
        *_ws(ws), _stream(stream)))


def moe_ep_dispatch(shape: Shape, rank: int, epoch: int, x, topk_idx, send_row, recv_offsets, peers, ws, stream=None):
    import torch
    _dev(x, torch.bfloat16, (shape.T, shape.d), "x")
    _dev(topk_idx, torch.int32, (shape.T, shape.k), "topk_idx")
    _dev(send_row, torch.int32, (shape.A,), "send_row")
    _dev(recv_offsets, torch.int32, (shape.E // shape.R + 1,), "recv_offsets")
    _check("moe_ep_dispatch", load().moe_ep_dispatch(
        ctypes.byref(shape.c()), rank, epoch, _ptr(x), _ptr(topk_idx), _ptr(send_row), _ptr(recv_offsets),
        ctypes.byref(peers.c()), *_ws(ws), _stream(stream)))


def moe_ep_signal(R: int, rank: int, slot: int, epoch: int, peers, stream=None):
    _check("moe_ep_signal", load().moe_ep_signal(R, rank, slot, epoch, ctypes.byref(peers.c()), _stream(stream)))


def moe_ep_wait(R: int, rank: int, slot: int, epoch: int, peers, ws, stream=None):
    _check("moe_ep_wait", load().moe_ep_wait(R, rank, slot, epoch, ctypes.byref(peers.c()), *_ws(ws),
                                             _stream(stream)))


def moe_ep_combine(shape: Shape, rank: int, epoch: int, send_row, topk_idx, topk_gate, y_shared, out, peers, ws,
                   stream=None):
    import torch
    _dev(send_row, torch.int32, (shape.A,), "send_row")
    _dev(topk_idx, torch.int32, (shape.T, shape.k), "topk_idx")
    _dev(topk_gate, torch.float32, (shape.T, shape.k), "topk_gate")
    _dev(y_shared, torch.bfloat16, (shape.T, shape.d), "y_shared")
    _dev(out, torch.bfloat16, (shape.T, shape.d), "out")
    _check("moe_ep_combine", load().moe_ep_combine(
        ctypes.byref(shape.c()), rank, epoch, _ptr(send_row), _ptr(topk_idx), _ptr(topk_gate), _ptr(y_shared),
        _ptr(out), ctypes.byref(peers.c()), *_ws(ws), _stream(stream)))
