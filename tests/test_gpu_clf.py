"""GPU parity of the cross-layer factorization of a window (xKV page, section 2.2)
against the oracle's truncated SVD.

Only A·B_l, the singular values and the orthonormality of A are unique (A is one
orthonormal basis of the dominant subspace; the oracle's is U_r), so those are compared.

Tolerances, from the arithmetic: the inputs have a drop of 20x in their spectrum right
after rank r, so n_iter = 3 passes leave a convergence error of about 0.05^7 relative,
far below rounding.  fp32: products accumulate in fp32 over at most a few thousand
terms and CholeskyQR2 leaves A orthonormal to ~1e-6, so A·B_l is within ~1e-5 of the
largest entry; the bar is 1e-4.  bf16: A and B_l are stored in bf16 (relative error
2^-9 each), so A·B_l is within ~4e-3 of the largest entry; the bar is 2e-2.
"""
import numpy as np
import pytest
import torch

from cross_layer_compressed_b200 import synth
from parity_util import bf16_ulp_diff

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda")
TOL = {"f32": 1e-4, "bf16": 2e-2}
ORTH_TOL = {"f32": 1e-5, "bf16": 2e-2}


@pytest.fixture(scope="module")
def xkv():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from cross_layer_compressed_b200 import build
    build.build()
    from cross_layer_compressed_b200 import xkv as m
    return m


def _tdt(dtype):
    return torch.float32 if dtype == "f32" else torch.bfloat16


def _run(xkv, X_dev, omega, W, B, L, Hkv, hd, r, n_iter, dtype):
    d = xkv.dims(B, Hkv, Hkv, hd, L, chunk=8, rank_k=0, rank_v=0, dtype=dtype)
    dk = Hkv * hd
    A = torch.empty((B, L, r), dtype=_tdt(dtype), device=DEV)
    Bt = torch.empty((W, B, dk, r), dtype=_tdt(dtype), device=DEV)
    ws = torch.empty(xkv.xkv_factorize_workspace_bytes(d, W, r), dtype=torch.uint8, device=DEV)
    om = torch.from_numpy(omega).to(DEV)
    xkv.xkv_factorize_window(d, W, r, X_dev, om, n_iter, A, Bt, ws)
    torch.cuda.synchronize()
    return A.double().cpu().numpy(), Bt.double().cpu().numpy()


def _inputs(W, B, L, Hkv, hd, n_modes, r, tau, gap, dtype, seed=0):
    X, s = synth.np_window_caches(W, B, L, Hkv * hd, n_modes, r, tau, gap, seed)
    Xs = synth.to_storage(X, dtype)                     # what the GPU reads
    return Xs, Xs.double().numpy(), s                   # and the oracle, exactly


def _check_against_oracle(ora, A, Bt, Xq, r, dtype):
    A_ref, Bt_ref, S = ora.factorize_window(Xq, r)
    P_ref = ora.reconstruct_window(A_ref, Bt_ref)
    P = ora.reconstruct_window(A, Bt)
    scale = np.abs(P_ref).max()
    err = np.abs(P - P_ref).max() / scale
    assert err <= TOL[dtype], f"A·B_l differs from the truncated SVD by {err:.2e} of max"
    W, B = Bt.shape[0], Bt.shape[1]
    for b in range(B):
        gram = A[b].T @ A[b]
        assert np.abs(gram - np.eye(r)).max() <= ORTH_TOL[dtype]
        Bb = np.concatenate([Bt[l, b].T for l in range(W)], axis=1)      # r x n
        sv = np.linalg.svd(Bb, compute_uv=False)
        assert np.abs(sv - S[b, :r]).max() <= 10 * TOL[dtype] * S[b, 0]
    return err


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_factorize_matches_truncated_svd(xkv, ora, dtype):
    """W = 2, two sequences, L = 1000 (ragged against the 128-row tiles), d_kv = 128."""
    W, B, L, Hkv, hd, r = 2, 2, 1000, 2, 64, 32
    Xs, Xq, _ = _inputs(W, B, L, Hkv, hd, 96, r, 16.0, 0.05, dtype)
    A, Bt = _run(xkv, Xs.to(DEV), synth.np_test_matrix(W * Hkv * hd, r, 0), W, B, L, Hkv, hd,
                 r, 3, dtype)
    _check_against_oracle(ora, A, Bt, Xq, r, dtype)


@pytest.mark.parametrize("W,B,L,Hkv,hd,r,n_iter", [(4, 1, 640, 1, 128, 64, 2),
                                                    (3, 3, 777, 1, 64, 48, 3),
                                                    (1, 2, 2048, 4, 128, 128, 2)])
def test_factorize_shapes(xkv, ora, W, B, L, Hkv, hd, r, n_iter):
    Xs, Xq, _ = _inputs(W, B, L, Hkv, hd, r + 40, r, 24.0, 0.05, "f32", seed=W + r)
    A, Bt = _run(xkv, Xs.to(DEV), synth.np_test_matrix(W * Hkv * hd, r, 1), W, B, L, Hkv, hd,
                 r, n_iter, "f32")
    _check_against_oracle(ora, A, Bt, Xq, r, "f32")


def test_factorize_full_rank_reproduces_the_caches(xkv, ora):
    """r = W·d_kv: the factorization is exact, A·B_l = X_l."""
    W, B, L, Hkv, hd = 2, 2, 300, 1, 64
    r = W * Hkv * hd
    rng = np.random.default_rng(4)
    X = rng.standard_normal((W, B, L, Hkv * hd))
    Xs = synth.to_storage(X, "f32")
    A, Bt = _run(xkv, Xs.to(DEV), synth.np_test_matrix(r, r, 2), W, B, L, Hkv, hd, r, 1, "f32")
    P = ora.reconstruct_window(A, Bt)
    assert np.abs(P - Xs.double().numpy()).max() <= 1e-4 * np.abs(X).max()


def test_factorize_rank_deficient_caches(xkv, ora):
    """rank(X) = 20 < r = 32: A·B_l = X_l, and A has 20 orthonormal columns and 12 zero
    columns (the directions the data does not have)."""
    W, B, L, Hkv, hd, r = 2, 1, 512, 1, 64, 32
    Xs, Xq, _ = _inputs(W, B, L, Hkv, hd, 20, r, 8.0, 1.0, "f32", seed=9)
    A, Bt = _run(xkv, Xs.to(DEV), synth.np_test_matrix(W * Hkv * hd, r, 3), W, B, L, Hkv, hd,
                 r, 2, "f32")
    P = ora.reconstruct_window(A, Bt)
    assert np.abs(P - Xq).max() <= 1e-4 * np.abs(Xq).max()
    gram = A[0].T @ A[0]
    diag = np.sort(np.diag(gram))
    assert np.abs(diag[:12]).max() <= 1e-6 and np.abs(diag[12:] - 1.0).max() <= 1e-5
    assert np.abs(gram - np.diag(np.diag(gram))).max() <= 1e-5


def test_factorize_feeds_the_decode_layout(xkv, ora):
    """The factors come out in the layouts the decode calls read (A as Ak_win, B_l^T as
    Bkt_layer): landmarks built from them on the GPU match the oracle's landmarks of the
    same factors to the landmark kernel's own bar (at most 1 bf16 ulp, rarely)."""
    W, B, L, Hkv, hd, r = 2, 2, 1024, 2, 128, 64
    Xs, _, _ = _inputs(W, B, L, Hkv, hd, 96, r, 16.0, 0.05, "bf16", seed=5)
    d = xkv.dims(B, Hkv, Hkv, hd, L, chunk=8, rank_k=r, rank_v=r, dtype="bf16")
    A = torch.empty((B, L, r), dtype=torch.bfloat16, device=DEV)
    Bt = torch.empty((W, B, Hkv * hd, r), dtype=torch.bfloat16, device=DEV)
    ws = torch.empty(xkv.xkv_factorize_workspace_bytes(d, W, r), dtype=torch.uint8, device=DEV)
    om = torch.from_numpy(synth.np_test_matrix(W * Hkv * hd, r, 4)).to(DEV)
    xkv.xkv_factorize_window(d, W, r, Xs.to(DEV), om, 2, A, Bt, ws)
    lm = torch.empty((B, Hkv, L // 8, hd), dtype=torch.bfloat16, device=DEV)
    xkv.xkv_build_landmarks(d, A, Bt[1], lm)
    torch.cuda.synchronize()
    ref = ora.build_landmarks(A.cpu(), Bt[1].cpu(), Hkv, hd, 8)
    got = lm.cpu().view(torch.int16).numpy().view(np.uint16)
    diff = bf16_ulp_diff(got, ref)
    assert diff.max() <= 1 and (diff > 0).mean() < 1e-3


def test_factorize_full_size_properties(xkv):
    """The Llama-3.1-8B-shaped window of the 32K selective workload (W = 4, 8 sequences,
    L = 32768, d_kv = 1024, r = 512, bf16, 2 passes), too large for the oracle's SVD:
    A is orthonormal, sampled entries of B_l equal X_l^T A in fp64, and the singular
    values of the product equal the generator's stated spectrum."""
    W, B, L, Hkv, hd, r = 4, 8, 32768, 8, 128, 512
    dk, n = Hkv * hd, 4 * Hkv * hd
    X, s = synth.torch_window_caches(W, B, L, dk, r + 64, r, 128.0, 0.1, "bf16", seed=0)
    A, Bt = _run(xkv, X, synth.np_test_matrix(n, r, 0), W, B, L, Hkv, hd, r, 2, "bf16")
    rng = np.random.default_rng(0)
    for b in (0, 5):
        Ab = torch.from_numpy(A[b]).to(DEV)
        gram = (Ab.T @ Ab).cpu().numpy()
        assert np.abs(gram - np.eye(r)).max() <= ORTH_TOL["bf16"]
        Bb = np.concatenate([Bt[l, b].T for l in range(W)], axis=1)
        sv = np.linalg.svd(Bb, compute_uv=False)
        assert np.all(np.abs(sv - s[:r]) <= 2e-2 * s[:r] + 2e-3 * s[0])
        for _ in range(16):
            l, j, i = int(rng.integers(W)), int(rng.integers(dk)), int(rng.integers(r))
            col = X[l, b, :, j].double().cpu().numpy()
            want = float(col @ A[b, :, i])
            assert abs(Bt[l, b, j, i] - want) <= 2e-2 * np.linalg.norm(col)
    del X
    torch.cuda.empty_cache()


# ------------------------------------------------------------------------ refold
def _refold(xkv, A, Bt, tail, W, B, L, T, Hkv, hd, r, n_iter, dtype, seed=0):
    d = xkv.dims(B, Hkv, Hkv, hd, L, chunk=8, rank_k=0, rank_v=0, dtype=dtype)
    dk = Hkv * hd
    A2 = torch.empty((B, L + T, r), dtype=_tdt(dtype), device=DEV)
    Bt2 = torch.empty((W, B, dk, r), dtype=_tdt(dtype), device=DEV)
    ws = torch.empty(xkv.xkv_refold_workspace_bytes(d, W, r, T), dtype=torch.uint8, device=DEV)
    om = torch.from_numpy(synth.np_test_matrix(W * dk, r, seed)).to(DEV)
    xkv.xkv_refold_window(d, W, r, A.to(DEV), Bt.to(DEV), tail.to(DEV) if T else None, T, om,
                          n_iter, A2, Bt2, ws)
    torch.cuda.synchronize()
    return A2.double().cpu().numpy(), Bt2.double().cpu().numpy()


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_refold_matches_oracle(xkv, ora, dtype):
    """Caches of L = 512 compressed rows (factors from the oracle, in the storage type)
    plus T = 100 generated rows: the refolded factors' product equals the oracle's
    refactorization of [A·B_l ; tail_l] (reconstruction rounded to the storage type)."""
    W, B, L, T, Hkv, hd, r = 2, 2, 512, 100, 2, 64, 32
    X, _ = synth.np_window_caches(W, B, L + T, Hkv * hd, 96, r, 16.0, 0.05, seed=3)
    A, Bt, _ = ora.factorize_window(X[:, :, :L], r)
    As, Bts = synth.to_storage(A, dtype), synth.to_storage(Bt, dtype)
    tail = synth.to_storage(X[:, :, L:], dtype)
    A2, Bt2 = _refold(xkv, As, Bts, tail, W, B, L, T, Hkv, hd, r, 3, dtype)
    round_to = (lambda P: synth.to_storage(P, dtype).double().numpy())
    Ar, Btr, S = ora.refold_window(As.double().numpy(), Bts.double().numpy(),
                                   tail.double().numpy(), r, to_storage=round_to)
    P_ref = ora.reconstruct_window(Ar, Btr)
    P = ora.reconstruct_window(A2, Bt2)
    assert A2.shape == (B, L + T, r)
    assert np.abs(P - P_ref).max() <= TOL[dtype] * np.abs(P_ref).max()
    for b in range(B):
        assert np.abs(A2[b].T @ A2[b] - np.eye(r)).max() <= ORTH_TOL[dtype]


def test_refold_without_tail_keeps_the_product(xkv, ora):
    """T = 0 (NULL tail): a rank-r product refactored at rank r is unchanged."""
    W, B, L, Hkv, hd, r = 3, 2, 700, 1, 64, 48
    X, _ = synth.np_window_caches(W, B, L, Hkv * hd, 80, r, 24.0, 0.05, seed=4)
    A, Bt, _ = ora.factorize_window(X, r)
    As, Bts = synth.to_storage(A, "f32"), synth.to_storage(Bt, "f32")
    A2, Bt2 = _refold(xkv, As, Bts, None, W, B, L, 0, Hkv, hd, r, 1, "f32")
    P0 = ora.reconstruct_window(As.double().numpy(), Bts.double().numpy())
    P = ora.reconstruct_window(A2, Bt2)
    assert np.abs(P - P0).max() <= 1e-4 * np.abs(P0).max()
