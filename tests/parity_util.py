"""Shared helpers of the GPU parity tests: tolerances and conversions.

Tolerances (floating-point outputs against the fp64 oracle, per tensor):
  rel-L2  ||gpu - ref|| / ||ref||     <= 5e-3
  max-abs max|gpu - ref|              <= 3e-2 * max|ref|
  gates   |gpu - ref|                 <= 2^-20
Integer, index and byte outputs are compared bit for bit.
"""
import numpy as np

REL_L2 = 5e-3
MAX_ABS_FRAC = 3e-2
GATE_TOL = 2.0 ** -20


def bits(t) -> np.ndarray:
    """bf16 torch tensor -> uint16 numpy bit patterns."""
    import torch
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def f64(b: np.ndarray) -> np.ndarray:
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def np_i32(t) -> np.ndarray:
    return t.detach().cpu().numpy().astype(np.int32)


def close(gpu: np.ndarray, ref: np.ndarray, what: str = ""):
    gpu = np.asarray(gpu, np.float64)
    ref = np.asarray(ref, np.float64)
    assert gpu.shape == ref.shape, (what, gpu.shape, ref.shape)
    assert np.all(np.isfinite(gpu)), f"{what}: non-finite values"
    if ref.size == 0:
        return
    err = gpu - ref
    nref = np.linalg.norm(ref)
    rel = np.linalg.norm(err) / max(nref, 1e-300)
    mx = np.max(np.abs(err))
    lim = MAX_ABS_FRAC * np.max(np.abs(ref))
    assert rel <= REL_L2, f"{what}: rel-L2 {rel:.3e} > {REL_L2}"
    assert mx <= lim, f"{what}: max-abs {mx:.3e} > {lim:.3e}"
    return rel, mx
