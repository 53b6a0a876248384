"""The C ABI library: loads, exports every declared symbol, validates on the host (no GPU).

Every call here fails validation before anything is launched, so no CUDA device
is touched.
"""
import ctypes
import os
import re

import pytest

import combine_warp_top_expert_b200 as moe

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moe.h")

TINY = moe.Shape(T=256, d=512, E=8, k=2, f=1024, R=2)
FAKE = 1 << 20  # an aligned, never-dereferenced address


def declared_functions():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w+\*?\s+\*?(moe_\w+)\s*\(", text, re.M)))


def test_library_loads_and_exports_every_declared_symbol():
    lib = moe.load()
    names = declared_functions()
    assert set(names) >= {"moe_route", "moe_dispatch", "moe_expert_ffn", "moe_combine", "moe_layer"}
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(moe.ABI_FUNCTIONS)


def test_workspace_bytes_layout():
    lib = moe.load()
    n = moe.workspace_bytes(TINY)
    A = TINY.T * TINY.k
    chunks = -(-TINY.T // (2048 // TINY.k))
    h_rows = 256 * (A // 256 + min(TINY.E, A))
    ep_scratch = -(-(6 * 256 + 4) * 4 // 256) * 256                 # expert-parallel plan and local scan
    combine_counters = -(-TINY.T * (TINY.d // 64) * 4 // 256) * 256  # the combine folded into GEMM2
    expect = (256 + (-(-chunks * TINY.E * 4 // 256) * 256) + (-(-A * 4 // 256) * 256) + ep_scratch
              + combine_counters + (-(-h_rows * TINY.f * 2 // 256) * 256))
    assert n == expect
    # shared expert adds its padded hidden rows
    sh = moe.Shape(T=256, d=512, E=8, k=2, f=1024, R=2, n_shared=1)
    assert moe.workspace_bytes(sh) == n + 256 * TINY.f * 2   # ceil(256 / 256) blocks of 256 rows
    # empty batch still has the status header
    assert moe.workspace_bytes(moe.Shape(T=0, d=512, E=8, k=2, f=1024, R=2)) >= 256
    for bad in (moe.Shape(-1, 512, 8, 2, 1024, 2), moe.Shape(8, 512, 8, 9, 1024, 2), moe.Shape(8, 512, 8, 2, 1024, 3),
                moe.Shape(8, 500, 8, 2, 1024, 2), moe.Shape(8, 512, 300, 2, 1024, 2),
                moe.Shape(8, 512, 8, 2, 1024, 2, n_shared=2)):
        assert lib.moe_workspace_bytes(ctypes.byref(bad.c())) == 0


@pytest.mark.parametrize("shape,code", [
    (moe.Shape(T=8, d=512, E=8, k=0, f=1024, R=2), moe.MOE_ERR_INVALID_ARG),
    (moe.Shape(T=8, d=512, E=4, k=5, f=1024, R=2), moe.MOE_ERR_INVALID_ARG),
    (moe.Shape(T=8, d=512, E=8, k=2, f=1024, R=3), moe.MOE_ERR_INVALID_ARG),
    (moe.Shape(T=8, d=512, E=8, k=2, f=1024, R=2, n_shared=3), moe.MOE_ERR_INVALID_ARG),
    (moe.Shape(T=8, d=520, E=8, k=2, f=1024, R=2), moe.MOE_ERR_UNSUPPORTED),
    (moe.Shape(T=8, d=512, E=8, k=2, f=1000, R=2), moe.MOE_ERR_UNSUPPORTED),
    (moe.Shape(T=8, d=512, E=512, k=2, f=1024, R=2), moe.MOE_ERR_UNSUPPORTED),
    (moe.Shape(T=8, d=512, E=16, k=9, f=1024, R=2), moe.MOE_ERR_UNSUPPORTED),
])
def test_invalid_shapes_are_rejected_before_launch(shape, code):
    lib = moe.load()
    s = ctypes.byref(shape.c())
    assert lib.moe_route(s, FAKE, FAKE, FAKE, FAKE, 1 << 30, None) == code
    assert lib.moe_dispatch(s, *([FAKE] * 10), FAKE, 1 << 30, None) == code
    assert lib.moe_expert_ffn(s, *([FAKE] * 9), FAKE, 1 << 30, None) == code
    assert lib.moe_combine(s, *([FAKE] * 5), FAKE, 1 << 30, None) == code


SHAPE_CHECKS = [
    ("T<0", dict(T=-1), moe.MOE_ERR_INVALID_ARG),
    ("d<1", dict(d=0), moe.MOE_ERR_INVALID_ARG),
    ("f<1", dict(f=0), moe.MOE_ERR_INVALID_ARG),
    ("E<1", dict(E=0), moe.MOE_ERR_INVALID_ARG),
    ("R<1", dict(R=0), moe.MOE_ERR_INVALID_ARG),
    ("capacity<0", dict(capacity=-1), moe.MOE_ERR_INVALID_ARG),
    ("T*k>2^27", dict(T=(1 << 26) + 1), moe.MOE_ERR_UNSUPPORTED),
    ("d>65536", dict(d=65536 + 128), moe.MOE_ERR_UNSUPPORTED),
    ("f>65536", dict(f=65536 + 128), moe.MOE_ERR_UNSUPPORTED),
]


@pytest.mark.parametrize("kw,code", [c[1:] for c in SHAPE_CHECKS], ids=[c[0] for c in SHAPE_CHECKS])
def test_every_shape_check_holds_at_every_entry_point(kw, code):
    """Each shape rule rejects the shape at every entry point, and the workspace size is 0."""
    lib = moe.load()
    base = dict(T=8, d=512, E=8, k=2, f=1024, R=2)
    base.update(kw)
    s = ctypes.byref(moe.Shape(**base).c())
    assert lib.moe_workspace_bytes(s) == 0
    assert lib.moe_route(s, FAKE, FAKE, FAKE, FAKE, 1 << 30, None) == code
    assert lib.moe_dispatch(s, *([FAKE] * 10), FAKE, 1 << 30, None) == code
    assert lib.moe_dispatch_static(s, *([FAKE] * 10), None, None) == code
    assert lib.moe_expert_ffn(s, *([FAKE] * 9), FAKE, 1 << 30, None) == code
    assert lib.moe_expert_gate_up(s, *([FAKE] * 5), FAKE, 1 << 30, None) == code
    assert lib.moe_expert_gate_up_gather(s, *([FAKE] * 5), FAKE, 1 << 30, None) == code
    assert lib.moe_expert_down(s, *([FAKE] * 5), FAKE, 1 << 30, None) == code
    assert lib.moe_combine(s, *([FAKE] * 5), FAKE, 1 << 30, None) == code
    b = moe.moe_layer_buffers_t(*([FAKE] * len(moe.moe_layer_buffers_t._fields_)))
    assert lib.moe_layer(s, ctypes.byref(b), FAKE, 1 << 30, None) == code


def test_misaligned_operands_are_rejected_before_launch():
    """Every bf16 operand must start on a 16-byte boundary (16-byte vector and TMA access)."""
    lib = moe.load()
    s = ctypes.byref(TINY.c())
    bad, ws, inv = FAKE + 8, (FAKE, 1 << 30), moe.MOE_ERR_INVALID_ARG
    # moe_dispatch: x_perm (x is covered above)
    assert lib.moe_dispatch(s, FAKE, *([FAKE] * 7), bad, FAKE, *ws, None) == inv
    # moe_expert_gate_up(x_perm, expert_offsets, w13, x, w13s)
    assert lib.moe_expert_gate_up(s, bad, FAKE, FAKE, FAKE, None, *ws, None) == inv
    assert lib.moe_expert_gate_up(s, FAKE, FAKE, bad, FAKE, None, *ws, None) == inv
    # moe_expert_gate_up_gather(x, row_src, expert_offsets, w13, w13s)
    assert lib.moe_expert_gate_up_gather(s, bad, FAKE, FAKE, FAKE, None, *ws, None) == inv
    assert lib.moe_expert_gate_up_gather(s, FAKE, FAKE, FAKE, bad, None, *ws, None) == inv
    # moe_expert_down(expert_offsets, w2, w2s, y_perm, y_shared)
    assert lib.moe_expert_down(s, FAKE, bad, None, FAKE, None, *ws, None) == inv
    assert lib.moe_expert_down(s, FAKE, FAKE, None, bad, None, *ws, None) == inv
    # moe_expert_ffn(x_perm, expert_offsets, w13, w2, x, w13s, w2s, y_perm, y_shared)
    for i in (0, 2, 3, 7):
        p = [FAKE, FAKE, FAKE, FAKE, None, None, None, FAKE, None]
        p[i] = bad
        assert lib.moe_expert_ffn(s, *p, *ws, None) == inv, i
    # moe_combine(y_perm, assign_row, topk_gate, y_shared, out)
    assert lib.moe_combine(s, bad, FAKE, FAKE, None, FAKE, *ws, None) == inv
    assert lib.moe_combine(s, FAKE, FAKE, FAKE, bad, FAKE, *ws, None) == inv
    assert lib.moe_combine(s, FAKE, FAKE, FAKE, None, bad, *ws, None) == inv
    # moe_layer: each bf16 buffer in turn
    for name in ("x", "w13", "w2", "w13s", "w2s", "x_perm", "y_perm", "y_shared", "out"):
        b = moe.moe_layer_buffers_t(*([FAKE] * len(moe.moe_layer_buffers_t._fields_)))
        setattr(b, name, bad)
        assert lib.moe_layer(s, ctypes.byref(b), *ws, None) == inv, name


def test_null_pointers_and_small_workspace_are_rejected():
    lib = moe.load()
    s = ctypes.byref(TINY.c())
    assert lib.moe_route(None, FAKE, FAKE, FAKE, FAKE, 1 << 30, None) == moe.MOE_ERR_INVALID_ARG
    assert lib.moe_route(s, None, FAKE, FAKE, FAKE, 1 << 30, None) == moe.MOE_ERR_INVALID_ARG
    assert lib.moe_route(s, FAKE, FAKE, FAKE, FAKE, 16, None) == moe.MOE_ERR_WORKSPACE
    assert lib.moe_route(s, FAKE, FAKE, FAKE, FAKE + 8, 1 << 30, None) == moe.MOE_ERR_WORKSPACE
    assert lib.moe_dispatch(s, FAKE + 2, *([FAKE] * 9), FAKE, 1 << 30, None) == moe.MOE_ERR_INVALID_ARG
    assert lib.moe_expert_ffn(s, *([FAKE] * 9), FAKE, 100, None) == moe.MOE_ERR_WORKSPACE
    sh = ctypes.byref(moe.Shape(T=8, d=512, E=8, k=2, f=1024, R=2, n_shared=1).c())
    assert lib.moe_expert_ffn(sh, FAKE, FAKE, FAKE, FAKE, None, None, None, FAKE, None, FAKE, 1 << 30,
                              None) == moe.MOE_ERR_INVALID_ARG
    assert lib.moe_combine(s, None, FAKE, FAKE, None, FAKE, FAKE, 1 << 30, None) == moe.MOE_ERR_INVALID_ARG
    assert lib.moe_layer(s, None, FAKE, 1 << 30, None) == moe.MOE_ERR_INVALID_ARG
    b = moe.moe_layer_buffers_t()
    assert lib.moe_layer(s, ctypes.byref(b), FAKE, 1 << 30, None) == moe.MOE_ERR_INVALID_ARG
    bits = ctypes.c_uint32()
    assert lib.moe_get_status(FAKE, 1 << 30, None, None) == moe.MOE_ERR_INVALID_ARG
    assert lib.moe_get_status(FAKE + 1, 1 << 30, ctypes.byref(bits), None) == moe.MOE_ERR_WORKSPACE
    assert lib.moe_clear_status(None, 1 << 30, None) == moe.MOE_ERR_WORKSPACE


def test_status_strings_and_timeout_knob():
    lib = moe.load()
    assert lib.moe_status_string(0) == b"MOE_OK"
    assert lib.moe_status_string(4) == b"MOE_ERR_CUDA"
    assert lib.moe_status_string(99) == b"MOE_ERR_UNKNOWN"
    old = lib.moe_set_wait_timeout_ns(12345)
    assert old == 2_000_000_000
    assert lib.moe_set_wait_timeout_ns(0) == 12345
    assert lib.moe_set_wait_timeout_ns(0) == 2_000_000_000
    assert lib.moe_set_gemm_policy(1) == 0
    assert lib.moe_set_gemm_policy(7) == -1
    assert lib.moe_set_gemm_policy(2) == 1
    assert lib.moe_set_gemm_policy(3) == -1                       # the split schedule is gone
    assert lib.moe_set_gemm_policy(0) == 2
    assert lib.moe_set_test_stall(1) == 0
    assert lib.moe_set_test_stall(0) == 1
    assert lib.moe_set_pdl(0) == 1                                # on by default
    assert lib.moe_set_pdl(1) == 0
    assert lib.moe_set_dispatch_path(moe.DISPATCH_ONE_PASS) == moe.DISPATCH_AUTO   # auto by default
    assert lib.moe_set_dispatch_path(3) == -1
    assert lib.moe_set_dispatch_path(moe.DISPATCH_TWO_PASS) == moe.DISPATCH_ONE_PASS
    assert lib.moe_set_dispatch_path(moe.DISPATCH_AUTO) == moe.DISPATCH_TWO_PASS


def test_rejected_calls_launch_nothing():
    """moe_kernel_launches counts the library's launches; calls refused on the host add none."""
    lib = moe.load()
    before = lib.moe_kernel_launches()
    bad = moe.Shape(T=16, d=100, E=8, k=2, f=128, R=2).c()          # d not a multiple of 128
    assert lib.moe_route(ctypes.byref(bad), FAKE, FAKE, FAKE, FAKE, 1 << 30, None) == moe.MOE_ERR_UNSUPPORTED
    b = moe.moe_layer_buffers_t(*([FAKE] * len(moe.moe_layer_buffers_t._fields_)))
    assert lib.moe_layer(ctypes.byref(bad), ctypes.byref(b), FAKE, 1 << 30, None) == moe.MOE_ERR_UNSUPPORTED
    assert lib.moe_kernel_launches() == before


def test_gathering_gemm_rejects_inputs_past_32_bit_row_offsets():
    """GEMM1 that gathers rows of x keeps byte offsets into x in 32 bits: T*d*2 must fit."""
    lib = moe.load()
    big = moe.Shape(T=(1 << 20) + 8, d=2048, E=8, k=2, f=1024, R=2).c()   # x is 4 GiB + 32 KiB
    assert lib.moe_expert_gate_up_gather(ctypes.byref(big), FAKE, FAKE, FAKE, FAKE, None, FAKE, 1 << 62,
                                         None) == moe.MOE_ERR_UNSUPPORTED
    b = moe.moe_layer_buffers_t(*([FAKE] * len(moe.moe_layer_buffers_t._fields_)))
    b.x_perm = None
    b.w13s = b.w2s = b.y_shared = None
    assert lib.moe_layer(ctypes.byref(big), ctypes.byref(b), FAKE, 1 << 62, None) == moe.MOE_ERR_UNSUPPORTED


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    """No silent fallback: without the CUDA library every entry point raises."""
    monkeypatch.setattr(moe, "_lib", None)
    monkeypatch.setattr(moe, "LIB_PATH", str(tmp_path / "absent" / "libmoe_b200.so"))
    with pytest.raises(RuntimeError, match="not built"):
        moe.load(build_if_missing=False)


def test_binding_refuses_host_buffers_before_the_abi():
    """A host tensor where a device buffer belongs raises ValueError in Python, so no
    host address ever reaches a kernel; a missing workspace is refused the same way."""
    import torch
    cpu_ws = torch.zeros(moe.workspace_bytes(TINY), dtype=torch.uint8)
    for call in (lambda: moe.get_status(cpu_ws), lambda: moe.clear_status(cpu_ws),
                 lambda: moe.moe_route(TINY, None, None, None, cpu_ws),
                 lambda: moe.moe_combine(TINY, None, None, None, None, None, cpu_ws)):
        with pytest.raises(ValueError, match="ws must be a CUDA tensor"):
            call()
    with pytest.raises(ValueError, match="ws must be a CUDA uint8 tensor"):
        moe.moe_expert_down(TINY, None, None, None, None, None, None)
    with pytest.raises(ValueError, match=r"outs\['topk_idx'\] must be a CUDA tensor"):
        moe.moe_layer(TINY, None, None, None, None, None, None, moe.alloc_layer_outputs(TINY, device="cpu"), cpu_ws)
    with pytest.raises(ValueError, match="logits must be a CUDA tensor"):
        moe.moe_route(TINY, torch.zeros((TINY.T, TINY.E)), None, None, cpu_ws)


def test_capacity_for_is_the_exact_ceiling():
    """capacity = ceil(C * T * k / E) in exact arithmetic: checked against integer ceiling
    division for two-decimal factors C = n / 100, and on a factor whose binary value sits
    just above a decimal (0.1 * 3 = 0.30000000000000004) where float arithmetic rounds up."""
    from hypothesis import given, settings, strategies as st

    assert moe.capacity_for(1.0, 4096, 2, 8) == 1024
    assert moe.capacity_for(1.25, 4096, 2, 8) == 1280
    assert moe.capacity_for(0.1 * 3, 10, 1, 3) == 1          # float: 1.0000000000000002 -> 2

    @settings(max_examples=200, deadline=None)
    @given(st.integers(1, 400), st.integers(0, 20000), st.integers(1, 8), st.integers(1, 256))
    def check(n, T, k, E):
        assert moe.capacity_for(n / 100, T, k, E) == -(-(n * T * k) // (100 * E))

    check()


def test_capacity_for_in_the_library_rejects_invalid_factors_and_overflow():
    """moe_capacity_for (the C ABI) takes C as num/den and keeps every product in 128 bits."""
    lib = moe.load()
    assert lib.moe_capacity_for(5, 4, 4096, 2, 8) == 1280
    assert lib.moe_capacity_for(1, 3, 10, 1, 1) == 4                     # ceil(10/3)
    assert lib.moe_capacity_for(1, 1, 0, 2, 8) == 0                      # empty batch
    for args in ((0, 1, 16, 2, 8), (1, 0, 16, 2, 8), (1, 1, -1, 2, 8), (1, 1, 16, 0, 8), (1, 1, 16, 2, 0),
                 (-3, 1, 16, 2, 8)):
        assert lib.moe_capacity_for(*args) == -1, args
    big = (1 << 62)
    assert lib.moe_capacity_for(big, 1, 1 << 30, 8, 1) == -1             # above INT32_MAX
    assert lib.moe_capacity_for(big, big, (1 << 31) - 1, 1, 1) == (1 << 31) - 1
    with pytest.raises(ValueError):
        moe.capacity_for(0.0, 16, 2, 8)


def test_layer_binding_checks_every_output_buffer():
    """moe_layer's binding checks dtype, contiguity and shape of every output (the C ABI cannot
    see tensor sizes), so a short `out` or a missing required buffer never reaches a kernel."""
    import torch
    outs = moe.alloc_layer_outputs(TINY, device="cpu")
    ws = torch.zeros(16, dtype=torch.uint8)
    cases = [("out", torch.empty((TINY.T - 1, TINY.d), dtype=torch.bfloat16), r"outs\['out'\] has shape"),
             ("y_perm", torch.empty((TINY.A, TINY.d), dtype=torch.float32), r"outs\['y_perm'\] must be torch.bfloat16"),
             ("row_src", torch.empty((TINY.A * 2,), dtype=torch.int32)[::2], r"outs\['row_src'\] must be contiguous"),
             ("x_perm", torch.empty((TINY.A + 8, TINY.d), dtype=torch.bfloat16), r"outs\['x_perm'\] has shape"),
             ("imbalance", torch.empty((1,), dtype=torch.float32), r"outs\['imbalance'\] has shape")]
    for name, bad, msg in cases:
        o = dict(outs)
        o[name] = bad
        with pytest.raises(ValueError, match=msg):
            moe.moe_layer(TINY, None, None, None, None, None, None, o, ws)
    o = dict(outs)
    o["out"] = None
    with pytest.raises(ValueError, match=r"outs\['out'\] is required"):
        moe.moe_layer(TINY, None, None, None, None, None, None, o, ws)
    sh = moe.Shape(T=16, d=128, E=8, k=2, f=128, R=2, n_shared=1)
    o = moe.alloc_layer_outputs(sh, device="cpu")
    o["y_shared"] = None
    with pytest.raises(ValueError, match=r"outs\['y_shared'\] is required"):
        moe.moe_layer(sh, None, None, None, None, None, None, o, ws)


def test_static_dispatch_limit_counts_only_the_dispatch_scratch():
    """The 1 MiB array holds what the dispatch kernels use (header, chunk counts, in-chunk ranks):
    the skewed-prefill shape (590,080 bytes) passes the size check, whatever else the full
    workspace holds; T 131072 x top-8 (4 MiB of ranks) does not. Without a GPU the accepted
    shape then fails at its first CUDA call, never as MOE_ERR_UNSUPPORTED."""
    lib = moe.load()
    ok = moe.Shape(T=16384, d=7168, E=256, k=8, f=2048, R=8, n_shared=1)
    assert moe.workspace_bytes(ok) > (1 << 20)
    rc = lib.moe_dispatch_static(ctypes.byref(ok.c()), *([FAKE] * 10), None, None)
    assert rc != moe.MOE_ERR_UNSUPPORTED
    big = moe.Shape(T=131072, d=128, E=256, k=8, f=128, R=8)
    assert lib.moe_dispatch_static(ctypes.byref(big.c()), *([FAKE] * 10), None, None) == moe.MOE_ERR_UNSUPPORTED
