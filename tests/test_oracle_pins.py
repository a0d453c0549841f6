"""Pins for the CPU oracle: checks against facts that do not come from the oracle itself.

Each pin targets a mistake the oracle could plausibly make: a transposed factor, a dropped
rank term, a wrong softmax normalisation, a reversed summation order, a double rounding,
a wrong tie-break, a wrong leader.  Sources: the xKV page (section 2.2 cross-layer
factorization, 2.3 selective reconstruction, section 4 dense reconstruction) and the
Stochastic KV Routing page (inference sharing strategy S, Algorithm 2 load/update skip,
the 32K Qwen3-8B memory figure).
"""
import itertools
import math

import numpy as np
import pytest
import torch

from cross_layer_compressed_b200 import synth


def _f32(x):
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))


def _sdpa64(q, K, V):
    """torch SDPA in fp64 on CPU; q [Hq][hd], K/V [Hkv][T][hd] with GQA by repeat."""
    Hq, hd = q.shape
    Hkv = K.shape[0]
    G = Hq // Hkv
    Kr = torch.as_tensor(K, dtype=torch.float64).repeat_interleave(G, 0)
    Vr = torch.as_tensor(V, dtype=torch.float64).repeat_interleave(G, 0)
    qq = torch.as_tensor(q, dtype=torch.float64)[:, None, :]
    o = torch.nn.functional.scaled_dot_product_attention(qq, Kr, Vr)
    return o[:, 0, :].numpy()


# ------------------------------------------------------------------ rounding helper
@pytest.mark.parametrize("x,bits", [
    (1.0, 0x3F80),
    (1.0 + 2 ** -8, 0x3F80),                 # exact half-way: ties to even (down)
    (1.0 + 3 * 2 ** -8, 0x3F82),             # exact half-way: ties to even (up)
    (1.0 + 2 ** -8 + 2 ** -40, 0x3F81),      # above half-way; an fp32 detour would tie down
    (-(1.0 + 2 ** -8 + 2 ** -40), 0xBF81),
    (3.0e38, 0x7F62),
    (1e39, 0x7F80),                          # overflow to +inf
    (2.0 ** -133, 0x0001),                   # smallest bf16 subnormal
    (0.0, 0x0000),
])
def test_round_bf16_nearest_even_single_step(ora, x, bits):
    assert ora.round_bf16(x) == bits


# ---------------------------------------------------- xKV 2.2: factorization pins
def _window_svd(L, W, d_kv, seed):
    rng = np.random.default_rng(seed)
    X = rng.standard_normal((L, W * d_kv))
    U, s, Vt = np.linalg.svd(X, full_matrices=False)
    A = U * s[None, :]                     # L x r (r = min(L, W*d_kv))
    return X, A, Vt                        # X = A @ Vt


def test_full_rank_factors_reconstruct_the_window(ora):
    """Full-rank SVD factors rebuild each layer's block of the concatenated cache."""
    L, W, d_kv = 48, 3, 8
    X, A, Vt = _window_svd(L, W, d_kv, 1)
    A32 = A.astype(np.float32)
    for layer in range(W):
        Bl = Vt[:, layer * d_kv:(layer + 1) * d_kv]          # r x d_kv
        Bt32 = np.ascontiguousarray(Bl.T.astype(np.float32))  # stored column-major
        rec = ora.reconstruct_rows(_f32(A32), _f32(Bt32), 0, L)
        ref = X[:, layer * d_kv:(layer + 1) * d_kv]
        assert np.max(np.abs(rec - ref)) <= 2e-6 * np.max(np.abs(ref))
        # and exactly the product of the stored factors (library matmul in fp64)
        exact = A32.astype(np.float64) @ Bt32.astype(np.float64).T
        assert np.max(np.abs(rec - exact)) <= 1e-12 * np.max(np.abs(exact))


def test_truncated_rank_drops_exactly_the_tail(ora):
    """Rank-r factors give the best rank-r approximation: the residual's spectral norm is
    the (r+1)-th singular value (Eckart-Young)."""
    L, W, d_kv, r = 40, 2, 8, 5
    X, A, Vt = _window_svd(L, W, d_kv, 2)
    s = np.linalg.svd(X, compute_uv=False)
    A32 = np.ascontiguousarray(A[:, :r].astype(np.float32))
    rec = np.hstack([ora.reconstruct_rows(_f32(A32), _f32(np.ascontiguousarray(
        Vt[:r, l * d_kv:(l + 1) * d_kv].T.astype(np.float32))), 0, L) for l in range(W)])
    resid = np.linalg.norm(X - rec, 2)
    assert abs(resid - s[r]) <= 1e-5 * s[0]


# ---------------------------------------- dense reconstruction = plain attention
def _xkv_case(L, W, Hq, Hkv, hd, seed, chunk=8):
    """W=1 full-rank factors of random K and V caches (fp32 storage)."""
    d_kv = Hkv * hd
    rng = np.random.default_rng(seed)
    XK = rng.standard_normal((L, d_kv)) * 0.5
    XV = rng.standard_normal((L, d_kv))
    out = {}
    for tag, X in (("k", XK), ("v", XV)):
        U, s, Vt = np.linalg.svd(X, full_matrices=False)
        out["A" + tag] = np.ascontiguousarray((U * s).astype(np.float32))[None]
        out["B" + tag + "t"] = np.ascontiguousarray(Vt.T.astype(np.float32))[None]
    q = (rng.standard_normal((1, Hq, hd)) * 0.7).astype(np.float32)
    return XK, XV, out, q


def _khat(out, tag, Hkv, hd):
    A = out["A" + tag][0].astype(np.float64)
    Bt = out["B" + tag + "t"][0].astype(np.float64)
    X = A @ Bt.T                                                  # L x d_kv
    return np.stack([X[:, g * hd:(g + 1) * hd] for g in range(Hkv)])  # Hkv x L x hd


@pytest.mark.parametrize("Hq,Hkv", [(4, 2), (4, 4), (5, 1)])
def test_dense_reconstruction_equals_sdpa(ora, Hq, Hkv):
    L, hd, C = 64, 16, 8
    XK, XV, f, q = _xkv_case(L, 1, Hq, Hkv, hd, 3)
    o = ora.reconstruct_attend(_f32(f["Ak"]), _f32(f["Av"]), _f32(f["Bkt"]), _f32(f["Bvt"]),
                               _f32(q), None, C)
    K, V = _khat(f, "k", Hkv, hd), _khat(f, "v", Hkv, hd)
    ref = _sdpa64(q[0], K, V)
    assert np.max(np.abs(o[0] - ref)) <= 1e-6 * np.max(np.abs(ref))
    # against the uncompressed caches: the factorization is lossless at full rank
    Ko = np.stack([XK[:, g * hd:(g + 1) * hd] for g in range(Hkv)])
    Vo = np.stack([XV[:, g * hd:(g + 1) * hd] for g in range(Hkv)])
    ref0 = _sdpa64(q[0], Ko, Vo)
    assert np.max(np.abs(o[0] - ref0)) <= 1e-5 * np.max(np.abs(ref0))


def test_selecting_every_chunk_equals_dense(ora):
    L, hd, C, Hq, Hkv = 64, 16, 8, 4, 2
    _, _, f, q = _xkv_case(L, 1, Hq, Hkv, hd, 4)
    args = [_f32(f[k]) for k in ("Ak", "Av", "Bkt", "Bvt")] + [_f32(q)]
    dense = ora.reconstruct_attend(*args, None, C)
    sel = np.tile(np.arange(L // C, dtype=np.int32), (1, Hkv, 1))
    assert np.array_equal(ora.reconstruct_attend(*args, sel, C), dense)


def test_selective_equals_sdpa_over_selected_rows(ora):
    L, hd, C, Hq, Hkv = 128, 16, 8, 4, 2
    _, _, f, q = _xkv_case(L, 1, Hq, Hkv, hd, 5)
    sel = np.array([[[0, 3, 7, 15], [1, 2, 9, 14]]], dtype=np.int32)
    o = ora.reconstruct_attend(*[_f32(f[k]) for k in ("Ak", "Av", "Bkt", "Bvt")], _f32(q),
                               sel, C)
    K, V = _khat(f, "k", Hkv, hd), _khat(f, "v", Hkv, hd)
    G = Hq // Hkv
    for g in range(Hkv):
        rows = np.concatenate([np.arange(c * C, (c + 1) * C) for c in sel[0, g]])
        ref = _sdpa64(q[0, g * G:(g + 1) * G], K[g:g + 1, rows], V[g:g + 1, rows])
        assert np.max(np.abs(o[0, g * G:(g + 1) * G] - ref)) <= 1e-6 * np.max(np.abs(ref))


@pytest.mark.parametrize("dense,n_tail", [(False, 5), (True, 3), (False, 0)])
def test_tail_rows_join_the_selected_rows_in_one_softmax(ora, dense, n_tail):
    """Generated tokens kept uncompressed: SDPA over the selected (or all) reconstructed
    rows followed by the tail rows, in fp64."""
    L, hd, C, Hq, Hkv, T_max = 128, 16, 8, 4, 2, 7
    _, _, f, q = _xkv_case(L, 1, Hq, Hkv, hd, 11)
    sel = None if dense else np.array([[[0, 3, 7, 15], [1, 2, 9, 14]]], dtype=np.int32)
    rng = np.random.default_rng(12)
    Kt = (rng.standard_normal((1, Hkv, T_max, hd)) * 0.5).astype(np.float32)
    Vt = rng.standard_normal((1, Hkv, T_max, hd)).astype(np.float32)
    o = ora.reconstruct_attend_tail(*[_f32(f[k]) for k in ("Ak", "Av", "Bkt", "Bvt")],
                                    _f32(q), sel, C, _f32(Kt), _f32(Vt), n_tail)
    K, V = _khat(f, "k", Hkv, hd), _khat(f, "v", Hkv, hd)
    G = Hq // Hkv
    for g in range(Hkv):
        rows = np.arange(L) if dense else \
            np.concatenate([np.arange(c * C, (c + 1) * C) for c in sel[0, g]])
        Kg = np.concatenate([K[g, rows], Kt[0, g, :n_tail]])[None]
        Vg = np.concatenate([V[g, rows], Vt[0, g, :n_tail]])[None]
        ref = _sdpa64(q[0, g * G:(g + 1) * G], Kg, Vg)
        assert np.max(np.abs(o[0, g * G:(g + 1) * G] - ref)) <= 1e-6 * np.max(np.abs(ref))
    if n_tail == 0:       # an empty tail is the plain call, operation for operation
        plain = ora.reconstruct_attend(*[_f32(f[k]) for k in ("Ak", "Av", "Bkt", "Bvt")],
                                       _f32(q), sel, C)
        assert np.array_equal(o, plain)


def test_a_dominant_tail_row_returns_its_value(ora):
    """One tail key aligned with the query and far larger than every other logit: the
    output is that row's value (closed form)."""
    L, hd, C, Hq, Hkv = 64, 16, 8, 2, 1
    _, _, f, q = _xkv_case(L, 1, Hq, Hkv, hd, 13)
    Kt = np.zeros((1, Hkv, 4, hd), dtype=np.float32)
    Vt = np.zeros((1, Hkv, 4, hd), dtype=np.float32)
    Kt[0, 0, 2] = 200.0 * (q[0, 0] + q[0, 1])
    Vt[0, 0, 2] = np.arange(hd)
    o = ora.reconstruct_attend_tail(*[_f32(f[k]) for k in ("Ak", "Av", "Bkt", "Bvt")],
                                    _f32(q), None, C, _f32(Kt), _f32(Vt), 3)
    assert np.allclose(o[0], np.arange(hd)[None], atol=1e-6)


def test_softmax_shift_invariance_through_an_extra_rank_term(ora):
    """Adding u to every key row (a rank-1 term: a ones column in A^K, u in B^K) shifts each
    head's logits by a constant, which softmax ignores.  Catches a dropped rank term or a
    missing normalisation."""
    L, hd, C, Hq, Hkv = 64, 16, 8, 4, 2
    _, _, f, q = _xkv_case(L, 1, Hq, Hkv, hd, 6)
    rng = np.random.default_rng(60)
    u = rng.standard_normal(Hkv * hd).astype(np.float32) * 3
    Ak2 = np.concatenate([f["Ak"], np.ones((1, L, 1), np.float32)], axis=2)
    Bkt2 = np.concatenate([f["Bkt"], u[None, :, None]], axis=2)
    sel = np.array([[[0, 2, 5], [1, 6, 7]]], dtype=np.int32)
    base = ora.reconstruct_attend(_f32(f["Ak"]), _f32(f["Av"]), _f32(f["Bkt"]), _f32(f["Bvt"]),
                                  _f32(q), sel, C)
    shifted = ora.reconstruct_attend(_f32(Ak2), _f32(f["Av"]), _f32(Bkt2), _f32(f["Bvt"]),
                                     _f32(q), sel, C)
    assert np.max(np.abs(base - shifted)) <= 1e-5 * np.max(np.abs(base))
    # ... whereas adding it to only some rows must change the result
    Ak3 = Ak2.copy()
    Ak3[0, :8, -1] = 0.0
    moved = ora.reconstruct_attend(_f32(Ak3), _f32(f["Av"]), _f32(Bkt2), _f32(f["Bvt"]),
                                   _f32(q), sel, C)
    assert np.max(np.abs(base - moved)) > 1e-3 * np.max(np.abs(base))


def test_chunk_permutation_invariance(ora):
    L, hd, C, Hq, Hkv = 64, 16, 8, 4, 2
    _, _, f, q = _xkv_case(L, 1, Hq, Hkv, hd, 7)
    nC = L // C
    perm = np.random.default_rng(70).permutation(nC)       # new chunk i holds old perm[i]
    inv = np.argsort(perm)
    rows = np.concatenate([np.arange(p * C, (p + 1) * C) for p in perm])
    sel = np.array([[[0, 1, 4, 6], [2, 3, 5, 7]]], dtype=np.int32)
    sel_p = np.sort(inv[sel], axis=2).astype(np.int32)
    a = ora.reconstruct_attend(_f32(f["Ak"]), _f32(f["Av"]), _f32(f["Bkt"]), _f32(f["Bvt"]),
                               _f32(q), sel, C)
    b = ora.reconstruct_attend(_f32(np.ascontiguousarray(f["Ak"][:, rows])),
                               _f32(np.ascontiguousarray(f["Av"][:, rows])), _f32(f["Bkt"]),
                               _f32(f["Bvt"]), _f32(q), sel_p, C)
    assert np.max(np.abs(a - b)) <= 1e-6 * np.max(np.abs(a))


def test_zero_query_gives_mean_of_selected_values(ora):
    """q = 0: uniform weights, so out = (mean of the selected A^V rows) B^V_g (closed form)."""
    L, hd, C, Hq, Hkv = 64, 16, 8, 4, 2
    _, _, f, q = _xkv_case(L, 1, Hq, Hkv, hd, 8)
    q0 = np.zeros_like(q)
    sel = np.array([[[1, 5], [0, 7]]], dtype=np.int32)
    o = ora.reconstruct_attend(*[_f32(f[k]) for k in ("Ak", "Av", "Bkt", "Bvt")], _f32(q0),
                               sel, C)
    Av = f["Av"][0].astype(np.float64)
    Bvt = f["Bvt"][0].astype(np.float64)
    G = Hq // Hkv
    for g in range(Hkv):
        rows = np.concatenate([np.arange(c * C, (c + 1) * C) for c in sel[0, g]])
        ref = Av[rows].mean(0) @ Bvt[g * hd:(g + 1) * hd].T
        for h in range(G):
            assert np.max(np.abs(o[0, g * G + h] - ref)) <= 1e-6 * np.max(np.abs(ref))


def test_one_sharp_chunk_dominates(ora):
    """A query aligned with one row's key at large scale puts all weight on that row."""
    L, hd, C, Hq, Hkv = 32, 16, 8, 2, 1
    _, _, f, _ = _xkv_case(L, 1, Hq, Hkv, hd, 9)
    K = _khat(f, "k", Hkv, hd)[0]
    V = _khat(f, "v", Hkv, hd)[0]
    t = 13
    q = np.stack([K[t] * 400.0, K[t] * 400.0])[None].astype(np.float32)
    o = ora.reconstruct_attend(*[_f32(f[k]) for k in ("Ak", "Av", "Bkt", "Bvt")], _f32(q),
                               None, C)
    assert np.max(np.abs(o[0, 0] - V[t])) <= 1e-5 * np.max(np.abs(V[t]))


def test_bf16_inputs_are_widened_exactly(ora):
    """bf16 storage: the oracle must read each value exactly (compare with the same inputs
    widened by torch)."""
    L, hd, C, Hq, Hkv = 32, 16, 8, 4, 2
    _, _, f, q = _xkv_case(L, 1, Hq, Hkv, hd, 10)
    bf = {k: torch.from_numpy(v).to(torch.bfloat16) for k, v in f.items()}
    qb = torch.from_numpy(q).to(torch.bfloat16)
    o = ora.reconstruct_attend(bf["Ak"], bf["Av"], bf["Bkt"], bf["Bvt"], qb, None, C)
    o32 = ora.reconstruct_attend(*[bf[k].float() for k in ("Ak", "Av", "Bkt", "Bvt")],
                                 qb.float(), None, C)
    assert np.array_equal(o, o32)


# ------------------------------------------------------------ landmark scoring pins
def test_score_integer_dot_products_and_group_max(ora):
    """Small integers are exact in bf16 and their dot products are exact in fp64."""
    rng = np.random.default_rng(11)
    B, Hkv, G, nC, hd = 2, 3, 4, 10, 16
    lm = rng.integers(-8, 9, size=(B, Hkv, nC, hd))
    q = rng.integers(-8, 9, size=(B, Hkv * G, hd))
    s = ora.score_landmarks(torch.tensor(lm, dtype=torch.bfloat16),
                            torch.tensor(q, dtype=torch.bfloat16))
    ref = np.einsum("bgcd,bghd->bgch", lm, q.reshape(B, Hkv, G, hd)).max(-1)
    assert np.array_equal(s, ref.astype(np.float64))


def test_score_sums_in_ascending_dimension_order(ora):
    """lm = [2^53, 1, -2^53, 0...], q = 1: ascending order gives (2^53 + 1) - 2^53 = 0 in
    fp64 (2^53 + 1 rounds to 2^53); the exact value, or a descending sum, gives 1."""
    hd = 8
    lm = np.zeros((1, 1, 1, hd))
    lm[0, 0, 0, :3] = [2.0 ** 53, 1.0, -(2.0 ** 53)]
    q = np.ones((1, 1, hd))
    s = ora.score_landmarks(torch.tensor(lm, dtype=torch.bfloat16),
                            torch.tensor(q, dtype=torch.bfloat16))
    assert s[0, 0, 0] == 0.0


def test_score_fp32_products_exact(ora):
    """fp32 x fp32 products have at most 48 significant bits: exact in fp64, so a single
    product is reproduced exactly."""
    rng = np.random.default_rng(12)
    a = rng.standard_normal(5).astype(np.float32)
    b = rng.standard_normal(5).astype(np.float32)
    for x, y in zip(a, b):
        lm = np.zeros((1, 1, 1, 4), np.float32)
        q = np.zeros((1, 1, 4), np.float32)
        lm[0, 0, 0, 2] = x
        q[0, 0, 2] = y
        s = ora.score_landmarks(_f32(lm), _f32(q))
        assert s[0, 0, 0] == float(x) * float(y)


# ------------------------------------------------------------------ selection pins
def _brute_force_select(scores, k, forced):
    """Exhaustive: the unique k-subset of candidates such that every member precedes every
    non-member under (score descending, index ascending)."""
    n = len(scores)
    cand = [c for c in range(n) if c not in forced]
    k = min(k, len(cand))
    hits = []
    for sub in itertools.combinations(cand, k):
        rest = [c for c in cand if c not in sub]
        ok = all((scores[a] > scores[b]) or (scores[a] == scores[b] and a < b)
                 for a in sub for b in rest)
        if ok:
            hits.append(sorted(set(sub) | set(forced)))
    assert len(hits) == 1
    return hits[0]


@pytest.mark.parametrize("seed", range(6))
def test_select_matches_brute_force_with_ties(ora, seed):
    rng = np.random.default_rng(100 + seed)
    n = 12
    scores = rng.integers(-3, 4, size=n).astype(np.float64)   # many exact ties
    for k, sink, recent in [(4, 1, 1), (3, 0, 0), (2, 2, 3), (4, 0, 2), (0, 1, 1)]:
        forced = sorted(set(range(sink)) | set(range(n - recent, n)))
        want = _brute_force_select(scores, k, forced)
        got = ora.select_chunks(scores[None, None, :], k, sink, recent)[0, 0]
        assert list(got) == want


def test_select_k_at_least_candidates_takes_everything(ora):
    s = np.arange(10, dtype=np.float64)[None, None, :]
    assert list(ora.select_chunks(s, 50, 1, 2)[0, 0]) == list(range(10))
    # sink and recent overlapping on a tiny context
    assert list(ora.select_chunks(s[:, :, :3], 1, 2, 2)[0, 0]) == [0, 1, 2]
    assert ora.n_selected(3, 1, 2, 2) == 3


def test_select_orders_negative_zero_below_positive_zero(ora):
    s = np.array([[[5.0, -0.0, 0.0, -1.0]]])
    assert list(ora.select_chunks(s, 2, 0, 0)[0, 0]) == [0, 2]


def test_select_is_per_unit(ora):
    s = np.array([[[1.0, 9.0, 3.0, 2.0], [9.0, 1.0, 2.0, 3.0]],
                  [[0.0, 0.0, 0.0, 0.0], [1.0, 2.0, 3.0, 4.0]]])
    got = ora.select_chunks(s, 1, 0, 1)
    assert got.tolist() == [[[1, 3], [0, 3]], [[0, 3], [2, 3]]]


# --------------------------------------------------------------- landmark pins
def test_landmarks_are_chunk_means_of_reconstructed_keys(ora):
    """Linearity: mean_t(A[t] B) = (mean_t A[t]) B; the oracle rounds once to fp32."""
    w = synth.reduced(synth.TINY_SR_F32, batch=1, ctx_len=64)
    x = synth.np_xkv_layer_inputs(w, 0, 0)
    lm = ora.build_landmarks(x["Ak"], x["Bkt"], w.n_kv_heads, w.head_dim, w.chunk)
    A = x["Ak"][0].double().numpy()
    Bt = x["Bkt"][0].double().numpy()
    abar = A.reshape(-1, w.chunk, A.shape[1]).mean(1)                 # nC x r
    ref = (abar @ Bt.T).reshape(-1, w.n_kv_heads, w.head_dim).transpose(1, 0, 2)
    ulp = np.spacing(np.abs(ref).astype(np.float32))
    assert np.all(np.abs(lm[0].astype(np.float64) - ref) <= ulp)


def test_landmarks_bf16_within_one_ulp_of_exact_mean(ora):
    w = synth.reduced(synth.LLAMA8B_SR_32K, batch=1, ctx_len=64, rank_k=32, rank_v=32,
                      n_kv_heads=2, n_q_heads=4, head_dim=16, n_needles=0)
    x = synth.np_xkv_layer_inputs(w, 0, 0)
    lm = ora.build_landmarks(x["Ak"], x["Bkt"], w.n_kv_heads, w.head_dim, w.chunk)
    got = ora.as_float64(ora.to_torch(lm))
    A = x["Ak"][0].double().numpy()
    Bt = x["Bkt"][0].double().numpy()
    ref = (A.reshape(-1, w.chunk, A.shape[1]).mean(1) @ Bt.T).reshape(
        -1, w.n_kv_heads, w.head_dim).transpose(1, 0, 2)
    half_ulp = np.abs(ref) * 2.0 ** -8                                 # bf16: 8 bits
    assert np.all(np.abs(got[0] - ref) <= half_ulp * 1.0000001)


# --------------------------------------------------------------------- R-CLA pins
def test_leader_map_nearest_previous_leader(ora):
    S = list(range(0, 36, 4))
    lo = ora.leader_map(S, 36)
    assert lo.tolist() == [4 * (l // 4) for l in range(36)]
    lo2 = ora.leader_map([0, 1, 5, 6, 20], 24)
    want = [0, 1, 1, 1, 1, 5, 6] + [6] * 13 + [20] * 4
    assert lo2.tolist() == want
    with pytest.raises(ValueError):
        ora.leader_map([3, 7], 10)                                    # layer 0 has no leader


def _rcla_case(B=2, Hkv=2, G=2, hd=16, L_max=40, length=30, n_lead=3, seed=20):
    rng = np.random.default_rng(seed)
    K = np.zeros((n_lead, B, Hkv, L_max, hd), np.float32)
    V = np.zeros((n_lead, B, Hkv, L_max, hd), np.float32)
    K[..., :length, :] = rng.standard_normal((n_lead, B, Hkv, length, hd))
    V[..., :length, :] = rng.standard_normal((n_lead, B, Hkv, length, hd))
    q = rng.standard_normal((B, Hkv * G, hd)).astype(np.float32)
    kn = rng.standard_normal((B, Hkv, hd)).astype(np.float32)
    vn = rng.standard_normal((B, Hkv, hd)).astype(np.float32)
    return K, V, q, kn, vn


def test_rcla_leader_update_then_attend_equals_sdpa(ora):
    K, V, q, kn, vn = _rcla_case()
    S = [0, 2, 5]
    lo = ora.leader_map(S, 8)
    length = 30
    K0, V0 = K.copy(), V.copy()
    o = ora.rcla_decode_attend(5, lo, K, V, length, _f32(kn), _f32(vn), _f32(q))
    slot = 2
    assert np.array_equal(K[slot, :, :, length], kn) and np.array_equal(V[slot, :, :, length], vn)
    mask = np.ones(K.shape, bool)
    mask[slot, :, :, length] = False
    assert np.array_equal(K[mask], K0[mask])                          # nothing else written
    for b in range(2):
        ref = _sdpa64(q[b], K[slot, b, :, :length + 1], V[slot, b, :, :length + 1])
        assert np.max(np.abs(o[b] - ref)) <= 1e-6 * np.max(np.abs(ref))


def test_rcla_non_leader_reads_leader_cache_and_writes_nothing(ora):
    K, V, q, _, _ = _rcla_case(seed=21)
    lo = ora.leader_map([0, 2, 5], 8)
    K0 = K.copy()
    o = ora.rcla_decode_attend(4, lo, K, V, 31, None, None, _f32(q))  # leader of 4 is 2
    assert np.array_equal(K, K0)
    for b in range(2):
        ref = _sdpa64(q[b], K[1, b, :, :31], V[1, b, :, :31])
        assert np.max(np.abs(o[b] - ref)) <= 1e-6 * np.max(np.abs(ref))
    with pytest.raises(ValueError):                                   # non-leader owns no cache
        ora.rcla_decode_attend(4, lo, K, V, 31, _f32(np.zeros((2, 2, 16))),
                               _f32(np.zeros((2, 2, 16))), _f32(q))


def test_rcla_single_row_returns_that_value(ora):
    """len = 0 with an update: one row, weight 1, so out = v_new (closed form)."""
    K, V, q, kn, vn = _rcla_case(length=0, seed=22)
    lo = ora.leader_map([0], 2)
    o = ora.rcla_decode_attend(0, lo, K, V, 0, _f32(kn), _f32(vn), _f32(q))
    G = 2
    for b in range(2):
        for h in range(4):
            assert np.array_equal(o[b, h], vn[b, h // G])


# ------------------------------------------------------------------ footprint pins
def test_footprint_equals_bytes_of_generated_tensors(ora):
    """xKV 2.2 storage O(L*r + W*r*d): compare the closed form with the bytes of the
    tensors the generator actually builds."""
    w = synth.reduced(synth.LLAMA8B_SR_32K, batch=1, ctx_len=64, rank_k=32, rank_v=48,
                      n_layers=5, window=2, n_kv_heads=2, n_q_heads=4, head_dim=16,
                      n_needles=0)
    total = 0
    for win in range(w.n_windows):
        x = synth.np_xkv_layer_inputs(w, 0, win * w.window)
        total += x["Ak"].nbytes + x["Av"].nbytes
    for layer in range(w.n_layers):
        x = synth.np_xkv_layer_inputs(w, 0, layer)
        total += x["Bkt"].nbytes + x["Bvt"].nbytes
    got = ora.footprint_bytes(w.batch, w.n_kv_heads, w.head_dim, w.ctx_len, w.chunk, w.rank_k,
                              w.rank_v, 1, w.n_layers, w.window, False)
    assert got == total
    lm_bytes = w.n_layers * w.n_chunks * w.d_kv * 2
    assert ora.footprint_bytes(w.batch, w.n_kv_heads, w.head_dim, w.ctx_len, w.chunk, w.rank_k,
                               w.rank_v, 1, w.n_layers, w.window, True) == total + lm_bytes


def test_footprint_is_smaller_than_dense_by_the_page_formula(ora):
    """For W layers of L tokens: W*L*d (dense, per K or V) vs L*r + W*r*d."""
    L, W, r, d = 32768, 4, 512, 1024
    got = ora.footprint_bytes(1, 8, 128, L, 8, r, r, 1, W, W, False)
    assert got == 2 * (L * r + W * r * d) * 2
    assert got < 2 * W * L * d * 2


def test_rcla_cache_bytes_match_the_page(ora):
    """Stochastic KV Routing page: Qwen3-8B at 32K, one cache per 4 layers, 4.6 -> 1.1 GB (4x)."""
    import os
    path = os.path.join(os.path.dirname(__file__), "golden", "rcla_qwen3_8b_32k_kv_bytes.txt")
    g = {}
    for line in open(path):
        if line.strip() and not line.startswith("#"):
            k, v = line.split()
            g[k] = float(v)
    n = int(g["n_layers"])
    leaders = len(range(0, n, int(g["leader_stride"])))
    dense = ora.rcla_cache_bytes(1, int(g["n_kv_heads"]), int(g["head_dim"]), int(g["ctx_len"]),
                                 1, n)
    shared = ora.rcla_cache_bytes(1, int(g["n_kv_heads"]), int(g["head_dim"]), int(g["ctx_len"]),
                                  1, leaders)
    assert dense == n * int(g["ctx_len"]) * 2 * int(g["n_kv_heads"]) * int(g["head_dim"]) * 2
    assert dense / shared == g["ratio"]
    gib = 2.0 ** 30
    # the page prints one decimal without a unit; in GiB both agree to within 3 %
    assert abs(dense / gib - g["dense_gb"]) <= 0.03 * g["dense_gb"]
    assert abs(shared / gib - g["shared_gb"]) <= 0.03 * g["shared_gb"]


# ------------------------------------------------------------ workload sanity
def test_needles_are_selected_by_the_oracle(ora):
    """The planted needle chunks reach the top-k of every (sequence, KV head)."""
    w = synth.reduced(synth.LLAMA8B_SR_32K, batch=2, ctx_len=1024, rank_k=128, rank_v=64,
                      n_kv_heads=2, n_q_heads=8, head_dim=128, top_k=8)
    x = synth.np_xkv_layer_inputs(w, 0, 1)
    lm = ora.to_torch(ora.build_landmarks(x["Ak"], x["Bkt"], w.n_kv_heads, w.head_dim, w.chunk))
    s = ora.score_landmarks(lm, x["q"])
    sel = ora.select_chunks(s, w.top_k, w.n_sink, w.n_recent)
    for b in range(w.batch):
        for g in range(w.n_kv_heads):
            assert set(x["needles"][b].tolist()) <= set(sel[b, g].tolist())


# ------------------------------------------------- cross-layer factorization (CLF)
# xKV page, section 2.2: concatenate the window's caches, rank-r SVD, shared A and per-
# layer B_l.  The pins build caches whose SVD is known by construction.
def _orthonormal(rng, rows, cols):
    q, _ = np.linalg.qr(rng.standard_normal((rows, cols)))
    return q


def _window_from_modes(U, s, V, W, d):
    """X_l = U diag(s) V_l^T, V_l the l-th block of d rows of V: [W][1][L][d]."""
    return np.stack([(U * s) @ V[l * d:(l + 1) * d].T for l in range(W)])[:, None]


def test_clf_tiny_closed_form(ora):
    """One layer, X = [[3, 0], [0, 4], [0, 0]]: singular values (4, 3); the rank-1 part
    is the 4 alone."""
    X = np.array([[3.0, 0.0], [0.0, 4.0], [0.0, 0.0]])[None, None]
    A, Bt, S = ora.factorize_window(X, 1)
    assert np.allclose(S[0], [4.0, 3.0], atol=1e-14)
    prod = ora.reconstruct_window(A, Bt)[0, 0]
    assert np.allclose(prod, [[0.0, 0.0], [0.0, 4.0], [0.0, 0.0]], atol=1e-14)


@pytest.mark.parametrize("W,L,d,m,r", [(2, 40, 8, 12, 5), (4, 64, 6, 20, 9), (3, 30, 4, 12, 12)])
def test_clf_known_spectrum(ora, W, L, d, m, r):
    """Caches built as U diag(s) V^T: the oracle returns s, its rank-r product is the
    first r modes of the construction layer by layer, and the residual energy is the
    sum of the dropped s_i^2 (Eckart-Young)."""
    rng = np.random.default_rng(7)
    U, V = _orthonormal(rng, L, m), _orthonormal(rng, W * d, m)
    s = np.sort(rng.uniform(0.5, 3.0, m))[::-1]
    X = _window_from_modes(U, s, V, W, d)
    A, Bt, S = ora.factorize_window(X, r)
    assert np.allclose(S[0, :m], s, atol=1e-12) and np.allclose(S[0, m:], 0.0, atol=1e-12)
    want = _window_from_modes(U[:, :r], s[:r], V[:, :r], W, d)
    got = ora.reconstruct_window(A, Bt)
    assert np.abs(got - want).max() <= 1e-12 * s[0]
    resid = np.sum((X - got) ** 2)
    assert abs(resid - np.sum(s[r:] ** 2)) <= 1e-12 * np.sum(s ** 2)


def test_clf_full_rank_is_exact(ora):
    """r = min(L, W·d): the factorization reproduces every layer's cache."""
    rng = np.random.default_rng(3)
    X = rng.standard_normal((3, 2, 10, 4))            # L = 10 < W·d = 12
    A, Bt, _ = ora.factorize_window(X, 10)
    assert np.abs(ora.reconstruct_window(A, Bt) - X).max() <= 1e-12 * np.abs(X).max()


def test_clf_basis_and_blocks(ora):
    """A has orthonormal columns; B_l = A^T X_l block by block, so a layer that is
    twice another gets twice its B, and a zero layer gets B_l = 0 -- a transposed or
    misplaced concatenation block fails here."""
    rng = np.random.default_rng(5)
    X0 = rng.standard_normal((1, 2, 50, 6))
    X = np.concatenate([X0, 2.0 * X0, np.zeros_like(X0)], axis=0)      # W = 3
    A, Bt, _ = ora.factorize_window(X, 4)
    for b in range(2):
        assert np.allclose(A[b].T @ A[b], np.eye(4), atol=1e-12)
        for l in range(3):
            assert np.allclose(Bt[l, b], X[l, b].T @ A[b], atol=1e-12)
        assert np.allclose(Bt[1, b], 2.0 * Bt[0, b], atol=1e-12)
        assert np.abs(Bt[2, b]).max() == 0.0


def test_clf_layer_order(ora):
    """Reordering the window's layers reorders the B_l and leaves each A·B_l in place."""
    rng = np.random.default_rng(11)
    X = rng.standard_normal((3, 1, 30, 5))
    r = 6
    P = ora.reconstruct_window(*ora.factorize_window(X, r)[:2])
    perm = [2, 0, 1]
    Pp = ora.reconstruct_window(*ora.factorize_window(X[perm], r)[:2])
    assert np.abs(Pp - P[perm]).max() <= 1e-12 * np.abs(X).max()


def test_clf_rank_bounds(ora):
    X = np.zeros((2, 1, 5, 3))
    for r in (0, 7):
        with pytest.raises(ValueError):
            ora.factorize_window(X, r)


def test_clf_generator_spectrum(ora):
    """The input generator's caches have exactly the spectrum it states."""
    X, s = synth.np_window_caches(2, 2, 120, 16, 40, 8, 6.0, 0.1, seed=0)
    _, _, S = ora.factorize_window(X, 8)
    for b in range(2):
        assert np.allclose(S[b, :40], s, atol=1e-12)
        assert np.allclose(S[b, 40:], 0.0, atol=1e-12)


def test_clf_refold_empty_tail_keeps_the_product(ora):
    """Refolding no rows refactors a rank-r product at rank r: the product is unchanged
    (the rank-r matrix is its own truncated SVD)."""
    rng = np.random.default_rng(21)
    X = rng.standard_normal((2, 2, 60, 5))
    A, Bt, _ = ora.factorize_window(X, 4)
    A2, Bt2, _ = ora.refold_window(A, Bt, np.zeros((2, 2, 0, 5)), 4)
    assert np.abs(ora.reconstruct_window(A2, Bt2) - ora.reconstruct_window(A, Bt)).max() <= 1e-12


def test_clf_refold_tail_in_span_is_exact(ora):
    """Tail rows that are combinations of the basis' rows' directions (each tail row a
    mix of rows of A·B_l with one set of weights across layers) add nothing new: the
    refolded product is [A·B_l ; tail_l] exactly, and the tail rows are rebuilt."""
    rng = np.random.default_rng(22)
    X = rng.standard_normal((3, 1, 40, 4))
    A, Bt, _ = ora.factorize_window(X, 5)
    P = ora.reconstruct_window(A, Bt)                         # rank 5 per sequence
    w = rng.standard_normal((7, 40))
    tail = np.stack([w @ P[l, 0] for l in range(3)])[:, None]  # [3][1][7][4], same rows mixed
    A2, Bt2, _ = ora.refold_window(A, Bt, tail, 5)
    want = np.concatenate([P, tail], axis=2)
    assert np.abs(ora.reconstruct_window(A2, Bt2) - want).max() <= 1e-10 * np.abs(want).max()


def test_clf_refold_is_the_factorization_of_the_extended_cache(ora):
    """A general tail: refolding equals factorizing the extended caches directly (the
    composition the refold is defined by), and the new basis covers L + T rows."""
    rng = np.random.default_rng(23)
    X = rng.standard_normal((2, 2, 30, 6))
    A, Bt, _ = ora.factorize_window(X, 6)
    tail = rng.standard_normal((2, 2, 9, 6))
    A2, Bt2, S2 = ora.refold_window(A, Bt, tail, 6)
    ext = np.concatenate([ora.reconstruct_window(A, Bt), tail], axis=2)
    A3, Bt3, S3 = ora.factorize_window(ext, 6)
    assert A2.shape == (2, 39, 6)
    assert np.allclose(S2, S3, atol=1e-12)
    assert np.abs(ora.reconstruct_window(A2, Bt2) - ora.reconstruct_window(A3, Bt3)).max() <= 1e-12


try:
    from hypothesis import given, settings, strategies as st
except ImportError:  # pragma: no cover - hypothesis is part of the test environment
    given = None

if given is not None:
    @settings(max_examples=30, deadline=None)
    @given(W=st.integers(1, 3), L=st.integers(3, 24), d=st.integers(1, 5),
           frac=st.floats(0.1, 1.0), seed=st.integers(0, 2 ** 31 - 1))
    def test_clf_random_windows_are_optimal_projections(ora, W, L, d, frac, seed):
        """Random windows and ranks: A is orthonormal, B_l = A^T X_l, the product is an
        orthogonal projection (||X||^2 = ||AB||^2 + ||X - AB||^2), and no random rank-r
        orthonormal basis leaves a smaller residual (Eckart-Young optimality checked
        against competitors, not against the SVD's own numbers)."""
        n = W * d
        r = max(1, min(L, n, int(round(frac * min(L, n)))))
        rng = np.random.default_rng(seed)
        X = rng.standard_normal((W, 1, L, d))
        A, Bt, _ = ora.factorize_window(X, r)
        a = A[0]
        assert np.allclose(a.T @ a, np.eye(r), atol=1e-10)
        for l in range(W):
            assert np.allclose(Bt[l, 0], X[l, 0].T @ a, atol=1e-10)
        P = ora.reconstruct_window(A, Bt)
        tot, kept, res = np.sum(X ** 2), np.sum(P ** 2), np.sum((X - P) ** 2)
        assert abs(tot - kept - res) <= 1e-9 * tot
        Xc = ora.concatenate_window(X, 0)
        for _ in range(5):
            q, _ = np.linalg.qr(rng.standard_normal((L, r)))
            other = np.sum((Xc - q @ (q.T @ Xc)) ** 2)
            assert other >= res - 1e-9 * tot


# -------------------------------------- value-range reservation pins (VASE page, 2.A)
def test_value_ranges_with_identity_basis_are_row_ranges(ora):
    """With A^V = I (L = r) the reconstruction is exact and V_hat is B^V_l^T itself, so the
    statistic is numpy's peak-to-peak of each row's head slice, maxed over the chunk."""
    rng = np.random.default_rng(7)
    B, Hkv, hd, C, L = 2, 3, 8, 4, 16
    d_kv = Hkv * hd
    V = rng.standard_normal((B, L, d_kv))
    V[1, 9, 2 * hd + 5] = 40.0                  # one large value: chunk 2 of head 2
    Av = np.stack([np.eye(L)] * B)              # [B][L][r], r = L
    Bvt = np.ascontiguousarray(V.transpose(0, 2, 1))   # [B][d_kv][r]: Bvt[j][i] = V[i][j]
    rho = ora.value_ranges(_f32(Av), _f32(Bvt), Hkv, hd, C)
    Vf = _f32(V).double().numpy()
    want = np.ptp(Vf.reshape(B, L // C, C, Hkv, hd), axis=4).max(axis=2).transpose(0, 2, 1)
    assert np.array_equal(rho, want)
    assert int(np.argmax(rho[1, 2])) == 2 and rho[1, 2, 2] > 40.0


def test_value_ranges_scale_and_shift(ora):
    """Range is translation invariant per row and scales with |alpha| (a sign flip swaps
    max and min); a constant row has range 0."""
    rng = np.random.default_rng(8)
    B, Hkv, hd, C, L, r = 1, 2, 16, 8, 32, 12
    Av = rng.standard_normal((B, L, r))
    Bvt = rng.standard_normal((B, Hkv * hd, r))
    rho = ora.value_ranges(_f32(Av), _f32(Bvt), Hkv, hd, C)
    rho_neg = ora.value_ranges(_f32(-2.0 * Av), _f32(Bvt), Hkv, hd, C)
    assert np.allclose(rho_neg, 2.0 * rho, rtol=1e-12, atol=0)
    const = np.zeros((B, Hkv * hd, r))
    const[:, :, 0] = 1.0                        # every head slice of a row is constant
    assert np.all(ora.value_ranges(_f32(Av), _f32(const), Hkv, hd, C) == 0.0)


def _brute_force_reserve(rho, n_value, forced):
    """Exhaustive: the unique n_res-subset of candidates preceding every other candidate
    under (rho descending, index ascending)."""
    return _brute_force_select(rho, n_value, []) if not forced else \
        [c for c in _brute_force_select(rho, n_value, forced) if c not in forced]


@pytest.mark.parametrize("seed", range(5))
def test_reserve_matches_brute_force_with_ties(ora, seed):
    rng = np.random.default_rng(200 + seed)
    n = 11
    rho = rng.integers(0, 4, size=n).astype(np.float64)       # many exact ties
    for nv, sink, recent in [(3, 1, 1), (0, 1, 2), (2, 0, 0), (20, 1, 1), (4, 2, 3)]:
        forced = sorted(set(range(sink)) | set(range(n - recent, n)))
        want = _brute_force_reserve(rho, nv, forced)
        got = ora.reserve_value_chunks(rho[None, None, :], nv, sink, recent)[0, 0]
        assert list(got) == want
        assert ora.n_reserved(n, nv, sink, recent) == len(want)


@pytest.mark.parametrize("seed", range(5))
def test_select_with_reserved_chunks_matches_brute_force(ora, seed):
    """The reserved chunks join the forced set; the top-k of the others by score follow."""
    rng = np.random.default_rng(300 + seed)
    n = 12
    scores = rng.integers(-2, 3, size=n).astype(np.float64)
    for k, sink, recent, res in [(3, 1, 1, [4, 7]), (2, 0, 0, [0]), (4, 1, 2, []),
                                 (50, 1, 1, [3, 5]), (0, 2, 2, [6])]:
        forced = sorted(set(range(sink)) | set(range(n - recent, n)) | set(res))
        want = _brute_force_select(scores, k, forced)
        resv = np.array(res, dtype=np.int32).reshape(1, 1, -1)
        got = ora.select_chunks_reserved(scores[None, None, :], resv, k, sink, recent)[0, 0]
        assert list(got) == want


def test_select_with_no_reserved_chunks_is_plain_selection(ora):
    rng = np.random.default_rng(9)
    s = rng.standard_normal((2, 3, 200))
    empty = np.zeros((2, 3, 0), dtype=np.int32)
    assert np.array_equal(ora.select_chunks_reserved(s, empty, 17, 1, 4),
                          ora.select_chunks(s, 17, 1, 4))


def test_select_with_reserved_rejects_forced_or_repeated_chunks(ora):
    s = np.zeros((1, 1, 10))
    with pytest.raises(ValueError):
        ora.select_chunks_reserved(s, np.array([[[0, 5]]], dtype=np.int32), 2, 1, 1)   # sink
    with pytest.raises(ValueError):
        ora.select_chunks_reserved(s, np.array([[[5, 5]]], dtype=np.int32), 2, 1, 1)   # repeat


def test_large_range_chunk_is_kept_whatever_its_score(ora):
    """A chunk whose values span a large range is reserved even when its score is the
    lowest of all (the point of the VASE reservation)."""
    rng = np.random.default_rng(10)
    B, Hkv, hd, C, L, r = 1, 1, 16, 8, 128, 16
    Av = rng.standard_normal((B, L, r)) * 0.1
    Av[0, 5 * C + 3] *= 200.0                  # token in chunk 5: a large-range value row
    Bvt = rng.standard_normal((B, Hkv * hd, r))
    rho = ora.value_ranges(_f32(Av), _f32(Bvt), Hkv, hd, C)
    res = ora.reserve_value_chunks(rho, 1, 1, 1)
    assert list(res[0, 0]) == [5]
    scores = np.arange(L // C, dtype=np.float64)[None, None, :].copy()
    scores[0, 0, 5] = -1e9                     # the worst score
    sel = ora.select_chunks_reserved(scores, res, 3, 1, 1)[0, 0]
    assert 5 in sel and list(sel) == [0, 5, 12, 13, 14, 15]
