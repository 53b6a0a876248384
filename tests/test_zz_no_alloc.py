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
per call, that a call is not thrown off by what an earlier call left in the
array's header (a non-zero last-chunk ticket), that the largest workload (64
histogram chunks) and the index-only form (x_perm NULL) match too, that the
one-pass and the two-kernel dispatch paths give the same bits through it, and
that a shape needing more scratch than the array holds is refused before
anything runs. The test only allocates the caller's own buffers.
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
    ptr = lambda t: None if t is None else t.data_ptr()  # noqa: E731
    rc = lib.moe_dispatch_static(ctypes.byref(shape.c()), ptr(x), idx.data_ptr(),
                                 *(ptr(b[n]) for n in OUTS), status.data_ptr(),
                                 torch.cuda.current_stream().cuda_stream)
    assert rc == moe.MOE_OK, lib.moe_status_string(rc)


def _reference_call(shape, x, idx, b, path=None):
    """moe_dispatch with a workspace (on `path`, else the current dispatch path)."""
    old = moe.set_dispatch_path(path) if path is not None else None
    try:
        ws = moe.new_workspace(shape)
        moe.moe_dispatch(shape, x, idx, *(b[n] for n in OUTS), ws)
        return moe.get_status(ws)
    finally:
        if old is not None:
            moe.set_dispatch_path(old)


@pytest.fixture
def two_pass():
    """The ticket tests run the two-kernel path (the one-pass kernel has no ticket)."""
    old = moe.set_dispatch_path(moe.DISPATCH_TWO_PASS)
    yield
    moe.set_dispatch_path(old)


def _scratch():
    """Device address and size of the library's fixed scratch array (current device)."""
    addr, size = ctypes.c_void_p(0), ctypes.c_size_t(0)
    assert moe.load().moe_dispatch_static_scratch(ctypes.byref(addr), ctypes.byref(size)) == moe.MOE_OK
    return addr.value, size.value


def _scratch_header():
    """The array's 256-byte header (status word at 0, last-chunk ticket at 64) as uint32."""
    import torch
    from cuda.bindings import runtime as rt
    torch.cuda.synchronize()
    addr, _ = _scratch()
    host = np.zeros(64, np.uint32)
    err, = rt.cudaMemcpy(host.ctypes.data, addr, 256, rt.cudaMemcpyKind.cudaMemcpyDeviceToHost)
    assert err == rt.cudaError_t.cudaSuccess
    return host


def _poison_scratch_header(ticket: int, status: int):
    import torch
    from cuda.bindings import runtime as rt
    torch.cuda.synchronize()
    addr, _ = _scratch()
    host = np.zeros(64, np.uint32)
    host[0], host[16] = status, ticket
    err, = rt.cudaMemcpy(addr, host.ctypes.data, 256, rt.cudaMemcpyKind.cudaMemcpyHostToDevice)
    assert err == rt.cudaError_t.cudaSuccess


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


@pytest.mark.parametrize("path", ["auto", "two_pass", "one_pass"])
def test_static_dispatch_matches_workspace_dispatch_on_two_calls_in_a_row(path):
    """Static calls on each dispatch path against the workspace call on the two-kernel path."""
    import torch
    status = torch.full((1,), 0xFFFF, dtype=torch.int32, device="cuda")
    cases = [_case(moe_synth.workload("qwen3_mixed")), _case(moe_synth.workload("tiny"))]
    p = {"auto": moe.DISPATCH_AUTO, "two_pass": moe.DISPATCH_TWO_PASS, "one_pass": moe.DISPATCH_ONE_PASS}[path]
    old = moe.set_dispatch_path(p)
    try:
        for shape, x, idx in cases:
            got, want = _buffers(shape), _buffers(shape)
            _static_call(shape, x, idx, got, status)
            ref_status = _reference_call(shape, x, idx, want, moe.DISPATCH_TWO_PASS)
            torch.cuda.synchronize()
            _same(got, want)
            assert int(status.item()) == ref_status == 0
    finally:
        moe.set_dispatch_path(old)


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


def _chunks(shape):
    per = max(1, 2048 // shape.k)
    return -(-shape.T // per)


def test_static_dispatch_ignores_a_stale_ticket_and_status_left_in_the_header(two_pass):
    """A call that was interrupted or raced could leave the last-chunk ticket and the
    status word non-zero; the next call zeroes the header first and is still exact."""
    import torch
    wl = moe_synth.workload("qwen3_mixed").with_(T=1280)      # 1280 * 8 / 2048 = 5 chunks
    shape, x, idx = _case(wl)
    assert _chunks(shape) == 5
    _poison_scratch_header(ticket=3, status=moe.MOE_DEV_TIMEOUT)
    status = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    got, want = _buffers(shape), _buffers(shape)
    _static_call(shape, x, idx, got, status)
    ref_status = _reference_call(shape, x, idx, want)
    torch.cuda.synchronize()
    _same(got, want)
    assert int(status.item()) == ref_status == 0
    hdr = _scratch_header()
    assert hdr[16] == 0 and hdr[0] == 0                        # ticket back at zero, no status bits


def test_static_dispatch_three_then_two_chunks_leaves_the_ticket_at_zero(two_pass):
    import torch
    status = torch.zeros((1,), dtype=torch.int32, device="cuda")
    for T in (768, 512):                                      # k = 8: 3 chunks, then 2
        wl = moe_synth.workload("qwen3_mixed").with_(T=T)
        shape, x, idx = _case(wl)
        assert _chunks(shape) == T // 256
        got, want = _buffers(shape), _buffers(shape)
        _static_call(shape, x, idx, got, status)
        _reference_call(shape, x, idx, want)
        torch.cuda.synchronize()
        _same(got, want)
        assert _scratch_header()[16] == 0


def test_static_dispatch_skewed_prefill_shape_64_chunks():
    """The largest workload (T 16384, top-8, E 256: 64 chunks, 590,080 bytes of scratch)."""
    import torch
    wl = moe_synth.workload("dsv3_skewed_prefill")
    shape, x, idx = _case(wl)
    assert _chunks(shape) == 64
    status = torch.zeros((1,), dtype=torch.int32, device="cuda")
    got, want = _buffers(shape), _buffers(shape)
    _static_call(shape, x, idx, got, status)
    ref_status = _reference_call(shape, x, idx, want)
    torch.cuda.synchronize()
    _same(got, want)
    assert int(status.item()) == ref_status == 0
    del got, want, x
    torch.cuda.empty_cache()


def test_static_dispatch_index_only():
    """x_perm = NULL (and x = NULL): indices, counts, offsets and imbalance only."""
    import torch
    wl = moe_synth.workload("qwen3_mixed")
    shape, x, idx = _case(wl)
    status = torch.zeros((1,), dtype=torch.int32, device="cuda")
    got, want = _buffers(shape), _buffers(shape)
    got["x_perm"] = None
    _static_call(shape, None, idx, got, status)
    _reference_call(shape, x, idx, want)
    torch.cuda.synchronize()
    for n in OUTS:
        if n != "x_perm":
            u, v = got[n], want[n]
            assert torch.equal(u, v), n
    assert int(status.item()) == 0
