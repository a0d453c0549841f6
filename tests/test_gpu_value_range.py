"""GPU parity of the value-range-aware selection (after the VASE page, section 2.A: the
tokens whose value vector has the largest range max(v) - min(v) are always kept, applied
to this path's chunks).

* The statistic rho (built once per cache: the largest range of a reconstructed value row
  of each chunk) is computed on the GPU with fp32 accumulation; it must match the
  oracle's fp64 statistic within a bound derived from that accumulation.
* Given identical statistics, the reservation is bit-exact; given identical landmarks,
  queries and reserved chunks, the fused selection is bit-exact.
* From the GPU's own statistic, a reservation may differ from the oracle's only at
  certified near-ties (the measured statistic difference bounds how far a rank can move).
"""
import numpy as np
import pytest
import torch

from cross_layer_compressed_b200 import synth

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda")


@pytest.fixture(scope="module")
def xkv():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from cross_layer_compressed_b200 import build
    build.build()
    from cross_layer_compressed_b200 import xkv as m
    return m


LLAMA_R = synth.reduced(synth.LLAMA8B_SR_32K, batch=2, ctx_len=2048, top_k=24)
QWEN14_R = synth.reduced(synth.QWEN14B_SR_16K, batch=2, ctx_len=1024, top_k=20)
TINY = synth.TINY_SR_F32


def _dev(t):
    return t.to(DEV).contiguous()


def _inputs(w, seed=0, plant=True):
    """One layer's inputs, with one token per sequence made a large-range value row."""
    x = synth.np_xkv_layer_inputs(w, seed=seed, layer=min(1, w.n_layers - 1))
    if plant:
        Av = x["Av"].float()
        for b in range(w.batch):
            t = (37 + 101 * b) % w.ctx_len
            Av[b, t] *= 30.0
        x["Av"] = Av.to(x["Av"].dtype)
    return x


def _gpu_rho(xkv, w, x):
    d = xkv.dims_of(w)
    rho = torch.full((w.batch, w.n_kv_heads, w.n_chunks), float("nan"), device=DEV)
    status = torch.full((1,), 7, dtype=torch.int32, device=DEV)
    xkv.xkv_build_value_ranges(d, _dev(x["Av"]), _dev(x["Bvt"]), rho, status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    return rho.cpu().double().numpy()


def _rho_bound(ora, w, x):
    """|rho_gpu - rho_ora| <= 2 gamma_r(2^-23) max_{t,j} sum_i |A_ti B_ij|: each entry of a
    reconstructed row is an fp32 accumulation of r exact products (the tensor cores may
    truncate rather than round, hence 2^-23), and a range is the difference of two."""
    A = np.abs(ora.as_float64(x["Av"]))                  # [B][L][r]
    Bt = np.abs(ora.as_float64(x["Bvt"]))                # [B][d_kv][r]
    r = A.shape[2]
    gam = r * 2.0 ** -23 / (1 - r * 2.0 ** -23)
    mag = np.matmul(A, Bt.transpose(0, 2, 1)).max(axis=(1, 2))   # [B]
    return 2 * gam * mag * (1 + 1e-6)


@pytest.mark.parametrize("w", [TINY, LLAMA_R, QWEN14_R], ids=lambda w: w.name)
def test_value_ranges_match_oracle(xkv, ora, w):
    x = _inputs(w)
    got = _gpu_rho(xkv, w, x)
    ref = ora.value_ranges(x["Av"], x["Bvt"], w.n_kv_heads, w.head_dim, w.chunk)
    bound = _rho_bound(ora, w, x)
    err = np.abs(got - ref).max(axis=(1, 2))
    assert np.all(err <= bound), (err, bound)
    # the planted large-range token's chunk leads every head of its sequence
    for b in range(w.batch):
        c = ((37 + 101 * b) % w.ctx_len) // w.chunk
        assert np.all(np.argmax(got[b], axis=1) == c)


def _reserve(xkv, w, rho_t, n_value, n_sink, n_recent, nC=None):
    nC = nC or w.n_chunks
    d = xkv.dims(rho_t.shape[0], rho_t.shape[1] * 4, rho_t.shape[1], 128, nC * 8, 8, 16, 16,
                 xkv.XKV_BF16)
    n_res = xkv.xkv_n_reserved(nC, n_value, n_sink, n_recent)
    res = torch.full((rho_t.shape[0], rho_t.shape[1], max(n_res, 1)), -7, dtype=torch.int32,
                     device=DEV)
    got_n = xkv.xkv_reserve_value_chunks(d, rho_t.to(DEV).contiguous(), n_value, n_sink,
                                         n_recent, res)
    torch.cuda.synchronize()
    assert got_n == n_res
    return res.cpu().numpy()[..., :n_res]


@pytest.mark.parametrize("nC,n_value,n_sink,n_recent", [
    (4096, 16, 1, 4), (300, 0, 1, 4), (300, 296, 1, 4), (300, 500, 1, 4), (37, 5, 3, 3),
    (5, 2, 3, 3), (16384, 64, 1, 4), (2048, 1, 0, 0), (777, 100, 0, 9)])
def test_reserve_bit_exact_given_the_statistic(xkv, ora, nC, n_value, n_sink, n_recent):
    """Ties (integer statistics, a unit where every chunk ties), every budget from none to
    more than the candidates, sink and recent windows that overlap."""
    rng = np.random.default_rng(nC + n_value)
    B, Hkv = 2, 3
    rho = rng.integers(0, 40, size=(B, Hkv, nC)).astype(np.float32)
    rho[0, 0] = 3.0
    rho[1, 1] = rng.standard_normal(nC).astype(np.float32) ** 2
    got = _reserve(xkv, None, torch.from_numpy(rho), n_value, n_sink, n_recent, nC=nC)
    ref = ora.reserve_value_chunks(rho.astype(np.float64), n_value, n_sink, n_recent)
    assert np.array_equal(got, ref)


def _fused(xkv, w, lm, q, reserved, n_res, top_k=None):
    d = xkv.dims_of(w)
    top_k = w.top_k if top_k is None else top_k
    base = xkv.xkv_n_selected(w.n_chunks, 0, w.n_sink, w.n_recent)
    rest = w.n_chunks - base - n_res
    n_sel = base + n_res + min(top_k, rest)
    sel = torch.full((w.batch, w.n_kv_heads, n_sel), -7, dtype=torch.int32, device=DEV)
    ws = torch.empty(xkv.xkv_score_select_workspace_bytes(d), dtype=torch.uint8, device=DEV)
    got_n = xkv.xkv_score_select(d, lm, q, top_k, w.n_sink, w.n_recent, sel, ws,
                                 reserved=reserved, n_reserved=n_res)
    torch.cuda.synchronize()
    assert got_n == n_sel
    band = ws[:4 * w.batch * w.n_kv_heads].cpu().view(torch.int32).numpy().view(np.uint32)
    return sel.cpu().numpy(), band.reshape(w.batch, w.n_kv_heads)


@pytest.mark.parametrize("w", [LLAMA_R, QWEN14_R], ids=lambda w: w.name)
def test_fused_selection_with_reserved_chunks_bit_exact(xkv, ora, w):
    x = _inputs(w)
    lm = ora.to_torch(ora.build_landmarks(x["Ak"], x["Bkt"], w.n_kv_heads, w.head_dim, w.chunk))
    rho = ora.value_ranges(x["Av"], x["Bvt"], w.n_kv_heads, w.head_dim, w.chunk)
    for n_value in (1, 7, 40):
        res = ora.reserve_value_chunks(rho, n_value, w.n_sink, w.n_recent)
        ref = ora.select_chunks_reserved(ora.score_landmarks(lm, x["q"]), res, w.top_k, w.n_sink,
                                         w.n_recent)
        got, band = _fused(xkv, w, _dev(lm), _dev(x["q"]), torch.from_numpy(res).to(DEV),
                           res.shape[2])
        assert np.array_equal(got, ref)
        assert np.all(band != 0xFFFFFFFE)


def test_fused_selection_rejects_a_bad_reserved_list(xkv, ora):
    """A reserved chunk inside the sink window, or repeated, fails its unit (-1 entries);
    the other units are unaffected."""
    w = LLAMA_R
    x = _inputs(w, plant=False)
    lm = ora.to_torch(ora.build_landmarks(x["Ak"], x["Bkt"], w.n_kv_heads, w.head_dim, w.chunk))
    rng = np.random.default_rng(3)
    res = np.stack([np.sort(rng.choice(np.arange(1, w.n_chunks - w.n_recent), 4, replace=False))
                    for _ in range(w.batch * w.n_kv_heads)]).reshape(w.batch, w.n_kv_heads, 4)
    res = res.astype(np.int32)
    res[0, 1, 0] = 0                   # the sink chunk
    res[1, 3, 2] = res[1, 3, 1]        # a repeat
    got, band = _fused(xkv, w, _dev(lm), _dev(x["q"]), torch.from_numpy(res).to(DEV), 4)
    assert np.all(got[0, 1] == -1) and band[0, 1] == 0xFFFFFFFE
    assert np.all(got[1, 3] == -1) and band[1, 3] == 0xFFFFFFFE
    ok = np.ones((w.batch, w.n_kv_heads), dtype=bool)
    ok[0, 1] = ok[1, 3] = False
    good = res.copy()
    good[0, 1] = good[0, 0]
    good[1, 3] = good[1, 2]
    ref = ora.select_chunks_reserved(ora.score_landmarks(lm, x["q"]), good, w.top_k, w.n_sink,
                                     w.n_recent)
    assert np.array_equal(got[ok], ref[ok])


@pytest.mark.parametrize("w", [LLAMA_R, QWEN14_R], ids=lambda w: w.name)
def test_value_reserved_pipeline_from_gpu_statistics(xkv, ora, w):
    """The product pipeline: statistic, reservation and fused selection on the GPU.  The
    reservation from the GPU statistic differs from the oracle's only at certified near-
    ties; the selection is bit-exact given the GPU's reserved chunks."""
    x = _inputs(w)
    rho_g = _gpu_rho(xkv, w, x)
    rho_o = ora.value_ranges(x["Av"], x["Bvt"], w.n_kv_heads, w.head_dim, w.chunk)
    beta = np.abs(rho_g - rho_o).max() * (1 + 1e-9) + 1e-300
    n_value = 12
    res_g = _reserve(xkv, w, torch.from_numpy(rho_g.astype(np.float32)), n_value, w.n_sink,
                     w.n_recent)
    res_o = ora.reserve_value_chunks(rho_o, n_value, w.n_sink, w.n_recent)
    assert np.array_equal(res_g, ora.reserve_value_chunks(rho_g, n_value, w.n_sink,
                                                          w.n_recent))
    forced = set(synth.forced_chunks(w.n_chunks, w.n_sink, w.n_recent))
    cand = np.array([c not in forced for c in range(w.n_chunks)])
    n_diff = 0
    for b in range(w.batch):
        for g in range(w.n_kv_heads):
            a, o = set(res_g[b, g].tolist()), set(res_o[b, g].tolist())
            if a == o:
                continue
            n_diff += 1
            tau = np.sort(rho_o[b, g][cand])[::-1][res_o.shape[2] - 1]
            for c in a ^ o:
                assert abs(rho_o[b, g, c] - tau) <= 2 * beta
    print(f"{w.name}: {n_diff} units reserve differently, all certified near-ties")
    lm = torch.empty((w.batch, w.n_kv_heads, w.n_chunks, w.head_dim),
                     dtype=torch.float32 if w.dtype == "f32" else torch.bfloat16, device=DEV)
    xkv.xkv_build_landmarks(xkv.dims_of(w), _dev(x["Ak"]), _dev(x["Bkt"]), lm)
    got, _ = _fused(xkv, w, lm, _dev(x["q"]), torch.from_numpy(res_g).to(DEV), res_g.shape[2])
    ref = ora.select_chunks_reserved(ora.score_landmarks(lm.cpu(), x["q"]), res_g, w.top_k,
                                     w.n_sink, w.n_recent)
    assert np.array_equal(got, ref)
