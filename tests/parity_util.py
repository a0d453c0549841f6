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


def _gamma(n, u):
    return n * u / (1 - n * u)


def certify_near_ties(lm_gpu, lm_ora, q, sel_gpu, sel_ora, s_ora, G, top_k, n_sink, n_recent):
    """Checks that every chunk selected on one side only is a certified near-tie and
    returns the number of units whose selections differ.

    lm_* [B][Hkv][nC][hd] and q [B][Hq][hd] as fp64; s_ora the oracle's scores of lm_ora;
    sel_gpu is the selection made from lm_gpu, sel_ora the oracle's from lm_ora.
    beta_c = max_h sum_d |lm_gpu - lm_ora|[c][d] |q_h[d]|
             + gamma_hd(2^-53) max_h sum_d (|lm_gpu| + |lm_ora|)[c][d] |q_h[d]|
    bounds |s_gpu(c) - s_ora(c)| (the first term the change of the exact sums, the second
    the fp64 rounding of both canonical sums).  The k-th candidate score moves by at most
    beta = max_c beta_c, so a chunk selected on one side only scores within 2 beta of the
    oracle's k-th score, at or below it if only the GPU side took it, at or above it if
    only the oracle did."""
    B, Hkv, nC, hd = lm_ora.shape
    forced = np.zeros(nC, dtype=bool)
    forced[:min(n_sink, nC)] = True
    forced[max(nC - n_recent, 0):] = True
    k_eff = min(top_k, int((~forced).sum()))
    n_diff = 0
    for b in range(B):
        for g in range(Hkv):
            a, o = set(sel_gpu[b, g].tolist()), set(sel_ora[b, g].tolist())
            if a == o:
                continue
            n_diff += 1
            qg = np.abs(q[b, g * G:(g + 1) * G])                       # [G][hd]
            dl = np.abs(lm_gpu[b, g] - lm_ora[b, g])                    # [nC][hd]
            mag = (np.abs(lm_ora[b, g]) + np.abs(lm_gpu[b, g])) @ qg.T
            beta_c = (dl @ qg.T).max(axis=1) + _gamma(hd, 2.0 ** -53) * mag.max(axis=1)
            beta = beta_c.max() * (1 + 1e-9)
            tau = np.sort(s_ora[b, g][~forced])[::-1][k_eff - 1]
            for c in a ^ o:
                sc = s_ora[b, g, c]
                assert abs(sc - tau) <= 2 * beta, (b, g, c, sc, tau, beta)
                assert (sc <= tau) if c in a else (sc >= tau), (b, g, c, sc, tau)
    return n_diff
