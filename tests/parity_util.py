"""Shared helpers of the GPU parity tests (tolerances and comparisons)."""
import numpy as np

# Output tolerances.  Absolute bars are the ones stated for the path (2e-2 for bf16
# inputs, 1e-4 for fp32 inputs).  Outputs here are ~1e-3..1e-1 in magnitude, so a
# relative bar per (sequence, head) row is checked too.  Derivation for the CUDA path:
# inputs are read exactly and accumulated in fp32 with fused multiply-adds (one rounding
# per term); the sums run over at most 1024 rank terms and a few thousand rows, so the
# relative error of the reconstructed rows and logits stays near 1e-6 for well-scaled
# data; expf, the split merge and the final division add a few fp32 ulps.  1e-3 (bf16)
# and 2e-5 (fp32) leave an order of magnitude of margin.
TOL = {"bf16": (2e-2, 1e-3), "f32": (1e-4, 2e-5)}


def compare_outputs(got, ref, dtype, mask=None):
    """Assert max-abs and per-row relative error bars; returns (max_abs, max_rel)."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    if mask is not None:
        got, ref = got[mask], ref[mask]
    assert np.all(np.isfinite(got)), "non-finite output"
    abs_tol, rel_tol = TOL[dtype]
    err = np.abs(got - ref)
    max_abs = float(err.max()) if err.size else 0.0
    scale = np.abs(ref).max(axis=-1, keepdims=True)
    rel = (err / np.maximum(scale, 1e-30)).max() if err.size else 0.0
    assert max_abs <= abs_tol, f"max abs error {max_abs:.3e} > {abs_tol}"
    assert rel <= rel_tol, f"max relative error {rel:.3e} > {rel_tol}"
    return max_abs, float(rel)


def bf16_ulp_diff(a_u16: np.ndarray, b_u16: np.ndarray) -> np.ndarray:
    """Distance in bf16 ulps between two bf16 bit arrays (same sign assumed)."""
    a = a_u16.astype(np.int32)
    b = b_u16.astype(np.int32)
    # map sign-magnitude to a monotone integer line
    a = np.where(a & 0x8000, -(a & 0x7FFF), a)
    b = np.where(b & 0x8000, -(b & 0x7FFF), b)
    return np.abs(a - b)
