"""moe_dispatch_static: the dispatch step for callers that cannot allocate.

Some callers of this library cannot hand it a device workspace: an engine
plugin or serving runtime whose device memory is planned and owned by its own
arena, or a C/FFI caller with no CUDA allocator of its own. For them the library
offers moe_dispatch_static, which keeps its scratch in a fixed array compiled
into the library and allocates nothing.

This file is collected last on purpose. Through the C ABI it checks that two
calls in a row (different shapes, so the second call runs on scratch the first
one left behind) give exactly what moe_dispatch gives on the same inputs (bit
for bit, the bar for integer and byte outputs), that the status output is
per call, and that a shape needing more scratch than the array holds is refused
before anything runs. The test only allocates the caller's own buffers.
"""
import ctypes

import numpy as np
import pytest

import combine_warp_top_expert_b200 as moe
import moe_synth
import oracle

pytestmark = pytest.mark.gpu

OUTS = ("expert_counts", "expert_offsets", "rank_counts", "rank_offsets", "row_src", "assign_row", "x_perm",
        "imbalance")


def _buffers(shape):
    import torch
    i32 = torch.int32
    return dict(expert_counts=torch.full((shape.E,), -7, dtype=i32, device="cuda"),
                expert_offsets=torch.full((shape.E + 1,), -7, dtype=i32, device="cuda"),
                rank_counts=torch.full((shape.R,), -7, dtype=i32, device="cuda"),
                rank_offsets=torch.full((shape.R + 1,), -7, dtype=i32, device="cuda"),
                row_src=torch.full((shape.A,), -7, dtype=i32, device="cuda"),
                assign_row=torch.full((shape.A,), -7, dtype=i32, device="cuda"),
                x_perm=torch.zeros((shape.A, shape.d), dtype=torch.bfloat16, device="cuda"),
                imbalance=torch.zeros((2,), dtype=torch.float32, device="cuda"))


def _static_call(shape, x, idx, b, status):
    lib = moe.load()
    import torch
    rc = lib.moe_dispatch_static(ctypes.byref(shape.c()), x.data_ptr(), idx.data_ptr(),
                                 *(b[n].data_ptr() for n in OUTS), status.data_ptr(),
                                 torch.cuda.current_stream().cuda_stream)
    assert rc == moe.MOE_OK, lib.moe_status_string(rc)


def _reference_call(shape, x, idx, b):
    ws = moe.new_workspace(shape)
    moe.moe_dispatch(shape, x, idx, *(b[n] for n in OUTS), ws)
    return moe.get_status(ws)


def _case(wl, idx_np=None):
    import torch
    shape = moe.Shape(T=wl.T, d=wl.d, E=wl.E, k=wl.k, f=wl.f, R=wl.R)
    x = moe_synth.device_inputs(wl, weights=False)["x"]
    if idx_np is None:
        idx_np, _, _ = oracle.route(moe_synth.host_logits(wl), wl.k)
    idx = torch.from_numpy(np.ascontiguousarray(idx_np, np.int32)).cuda()
    return shape, x, idx


def _same(a, b):
    import torch
    for n in OUTS:
        u, v = a[n], b[n]
        if u.dtype == torch.bfloat16:
            u, v = u.view(torch.int16), v.view(torch.int16)
        assert torch.equal(u, v), n


def test_static_dispatch_matches_workspace_dispatch_on_two_calls_in_a_row():
    import torch
    status = torch.full((1,), 0xFFFF, dtype=torch.int32, device="cuda")
    cases = [_case(moe_synth.workload("qwen3_mixed")), _case(moe_synth.workload("tiny"))]
    for shape, x, idx in cases:
        got, want = _buffers(shape), _buffers(shape)
        _static_call(shape, x, idx, got, status)
        ref_status = _reference_call(shape, x, idx, want)
        torch.cuda.synchronize()
        _same(got, want)
        assert int(status.item()) == ref_status == 0


def test_static_dispatch_reports_per_call_status_and_refuses_oversized_shapes():
    import torch
    wl = moe_synth.workload("tiny")
    idx_np, _, _ = oracle.route(moe_synth.host_logits(wl), wl.k)
    bad = idx_np.copy()
    bad[3, 1] = wl.E + 5                      # out of range: skipped and flagged
    status = torch.zeros((1,), dtype=torch.int32, device="cuda")
    shape, x, idx = _case(wl, bad)
    got, want = _buffers(shape), _buffers(shape)
    _static_call(shape, x, idx, got, status)
    ref_status = _reference_call(shape, x, idx, want)
    _same(got, want)
    assert int(status.item()) == ref_status == moe.MOE_DEV_BOUNDS
    shape, x, idx = _case(wl, idx_np)         # the next call starts from a clear status word
    got = _buffers(shape)
    _static_call(shape, x, idx, got, status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    # 131072 tokens x top-8 needs 4 MiB of in-chunk ranks: more than the 1 MiB array
    big = moe.Shape(T=131072, d=128, E=256, k=8, f=128, R=8)
    lib = moe.load()
    fake = 1 << 20
    rc = lib.moe_dispatch_static(ctypes.byref(big.c()), *([fake] * 10), None, None)
    assert rc == moe.MOE_ERR_UNSUPPORTED
