"""Oracle of the cross-layer factorization of one window (CLF).

TEST INFRASTRUCTURE ONLY, like the rest of this package.  Plain numpy in fp64, with
LAPACK's SVD (``numpy.linalg.svd``) as the one library step.

xKV page, section 2.2 (cross-layer factorization), steps 1-3: the caches of the W
consecutive layers of a window are concatenated side by side, a rank-r SVD of the
concatenation is taken, and it yields one token basis A shared by the window and one
reconstruction matrix B_l per layer; A·B_l stands in for layer l's cache.

Reading taken where the page leaves a choice open: per sequence b the concatenation is
X_b = [X_0,b | X_1,b | ... | X_{W-1},b] (L rows, W·d_kv columns, layer-major columns),
the truncated SVD X_b ≈ U_r S_r V_r^T is split as A_b = U_r (orthonormal columns) and
B_l,b = (S_r V_r^T)[:, l·d_kv:(l+1)·d_kv].  Only the product A·B_l is unique (A is
fixed up to an r x r rotation, and up to column signs even in exact arithmetic), so
parity compares products, singular values and orthonormality, never A itself.
"""
from __future__ import annotations

import numpy as np


def concatenate_window(X: np.ndarray, b: int) -> np.ndarray:
    """Step 1: X [W][B][L][d_kv] -> the L x W·d_kv concatenation of sequence b."""
    W = X.shape[0]
    return np.concatenate([np.asarray(X[l, b], dtype=np.float64) for l in range(W)], axis=1)


def factorize_window(X, rank: int):
    """Steps 2-3 for every sequence: A [B][L][r] and Bt [W][B][d_kv][r], where
    Bt[l][b] = B_l,b^T (B_l stored column-major, as the decode calls take it).
    Also returns the singular values of each concatenation, s [B][min(L, W·d_kv)]."""
    X = np.asarray(X, dtype=np.float64)
    W, B, L, d = X.shape
    n = W * d
    if not 1 <= rank <= min(L, n):
        raise ValueError("rank must be in [1, min(L, W*d_kv)]")
    A = np.empty((B, L, rank))
    Bt = np.empty((W, B, d, rank))
    S = np.empty((B, min(L, n)))
    for b in range(B):
        Xb = concatenate_window(X, b)
        U, s, Vt = np.linalg.svd(Xb, full_matrices=False)
        A[b] = U[:, :rank]
        SV = s[:rank, None] * Vt[:rank]              # S_r V_r^T, r x W·d_kv
        for l in range(W):
            Bt[l, b] = SV[:, l * d:(l + 1) * d].T
        S[b] = s
    return A, Bt, S


def reconstruct_window(A, Bt) -> np.ndarray:
    """A·B_l for every layer and sequence: [W][B][L][d_kv] in fp64."""
    A = np.asarray(A, dtype=np.float64)
    Bt = np.asarray(Bt, dtype=np.float64)
    W, B = Bt.shape[0], Bt.shape[1]
    out = np.empty((W, B, A.shape[1], Bt.shape[2]))
    for l in range(W):
        for b in range(B):
            out[l, b] = A[b] @ Bt[l, b].T
    return out


def refold_window(A, Bt, tail, rank: int, to_storage=None):
    """Refold a tail of generated, uncompressed rows into the window's factors (the dense
    tail buffer of the decode loop, emptied periodically): per layer the cache the decode
    calls see, [A·B_l ; tail_l] ((L + T) x d_kv, the reconstructed part rounded to the
    storage type by `to_storage` when given), is factored again at rank r exactly as
    factorize_window does.  tail: [W][B][T][d_kv].  Returns factorize_window's triple."""
    P = reconstruct_window(A, Bt)
    if to_storage is not None:
        P = to_storage(P)
    X = np.concatenate([P, np.asarray(tail, dtype=np.float64)], axis=2)
    return factorize_window(X, rank)
