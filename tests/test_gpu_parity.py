"""GPU parity: every entry point of the CUDA library against the CPU oracle, element by
element, on seeded synthetic inputs at sizes the oracle finishes in seconds (several
tiles, ragged tails), plus edge cases.  Scores and selections must match bit for bit;
attention outputs within the tolerances of parity_util.TOL."""
import dataclasses

import numpy as np
import pytest
import torch

from cross_layer_compressed_b200 import synth
from parity_util import bf16_ulp_diff, compare_outputs

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


# Small workloads (each spans several CTAs and ends on a ragged tile)
TINY = synth.TINY_SR_F32                                                  # as specified
LLAMA_R = synth.reduced(synth.LLAMA8B_SR_32K, batch=2, ctx_len=2048, top_k=24)
QWEN14_R = synth.reduced(synth.QWEN14B_SR_16K, batch=2, ctx_len=1024, top_k=20)
DENSE_R = synth.reduced(synth.LLAMA8B_DENSE_128K, batch=1, ctx_len=1024)
SMALL_HD64 = dataclasses.replace(synth.reduced(synth.LLAMA8B_SR_32K, batch=3, ctx_len=1536,
                                               top_k=11, n_needles=0),
                                 head_dim=64, n_kv_heads=2, n_q_heads=6, rank_k=96, rank_v=80,
                                 name="hd64_g3")
XKV_CASES = [TINY, LLAMA_R, QWEN14_R, SMALL_HD64]


def _dev(t):
    return t.to(DEV).contiguous()


def _host_lm(ora, lm_np):
    return ora.to_torch(lm_np)


def _layer_inputs(w, layer=1):
    return synth.np_xkv_layer_inputs(w, seed=0, layer=min(layer, w.n_layers - 1))


# ------------------------------------------------------------------------ landmarks
@pytest.mark.parametrize("w", XKV_CASES, ids=lambda w: w.name)
def test_landmarks_match_oracle(xkv, ora, w):
    x = _layer_inputs(w)
    ref = ora.build_landmarks(x["Ak"], x["Bkt"], w.n_kv_heads, w.head_dim, w.chunk)
    d = xkv.dims_of(w)
    dt = torch.float32 if w.dtype == "f32" else torch.bfloat16
    lm = torch.empty((w.batch, w.n_kv_heads, w.n_chunks, w.head_dim), dtype=dt, device=DEV)
    xkv.xkv_build_landmarks(d, _dev(x["Ak"]), _dev(x["Bkt"]), lm)
    torch.cuda.synchronize()
    got = lm.cpu()
    if w.dtype == "f32":
        g = got.numpy()
        # fp64 accumulation in a different order, one rounding to fp32: at most 1 ulp
        assert np.all(np.abs(g.astype(np.float64) - ref.astype(np.float64))
                      <= np.spacing(np.abs(ref)))
    else:
        gu = got.view(torch.int16).numpy().view(np.uint16)
        diff = bf16_ulp_diff(gu, ref)
        assert diff.max() <= 1
        assert (diff > 0).mean() < 1e-4


# ------------------------------------------------------------------------- scoring
@pytest.mark.parametrize("w", XKV_CASES, ids=lambda w: w.name)
def test_scores_bit_exact(xkv, ora, w):
    x = _layer_inputs(w)
    lm = _host_lm(ora, ora.build_landmarks(x["Ak"], x["Bkt"], w.n_kv_heads, w.head_dim, w.chunk))
    ref = ora.score_landmarks(lm, x["q"])
    scores = torch.empty((w.batch, w.n_kv_heads, w.n_chunks), dtype=torch.float64, device=DEV)
    xkv.xkv_score_landmarks(xkv.dims_of(w), _dev(lm), _dev(x["q"]), scores)
    torch.cuda.synchronize()
    got = scores.cpu().numpy()
    assert np.array_equal(got.view(np.uint64), ref.view(np.uint64))


def test_scores_bit_exact_heavy_cancellation(xkv, ora):
    """Values whose fp64 sums round differently in any other order (2^53 + 1 - 2^53)."""
    B, Hkv, G, hd, nC = 1, 2, 4, 128, 200
    rng = np.random.default_rng(3)
    lm = rng.integers(-4, 5, size=(B, Hkv, nC, hd)).astype(np.float64)
    lm[..., 0] = 2.0 ** 53
    lm[..., 1] = 1.0
    lm[..., 2] = -(2.0 ** 53)
    q = np.ones((B, Hkv * G, hd))
    q[:, :, 3:] = rng.integers(-3, 4, size=(B, Hkv * G, hd - 3))
    lm_t = torch.tensor(lm, dtype=torch.bfloat16)
    q_t = torch.tensor(q, dtype=torch.bfloat16)
    ref = ora.score_landmarks(lm_t, q_t)
    d = xkv.dims(B, Hkv * G, Hkv, hd, nC * 8, 8, 16, 16, xkv.XKV_BF16)
    scores = torch.empty((B, Hkv, nC), dtype=torch.float64, device=DEV)
    xkv.xkv_score_landmarks(d, _dev(lm_t), _dev(q_t), scores)
    torch.cuda.synchronize()
    assert np.array_equal(scores.cpu().numpy().view(np.uint64), ref.view(np.uint64))


@pytest.mark.parametrize("hd,G,nC", [(64, 1, 37), (64, 8, 100), (128, 2, 33), (128, 8, 65),
                                     (64, 4, 1), (128, 5, 300)])
def test_scores_bit_exact_shapes(xkv, ora, hd, G, nC):
    """Every head size and group size of the bf16 scoring kernels, with row counts that
    end in a partial warp batch."""
    B, Hkv = 2, 3
    rng = np.random.default_rng(hd * 1000 + G * 10 + nC)
    lm_t = torch.tensor(rng.standard_normal((B, Hkv, nC, hd)), dtype=torch.bfloat16)
    q_t = torch.tensor(rng.standard_normal((B, Hkv * G, hd)), dtype=torch.bfloat16)
    ref = ora.score_landmarks(lm_t, q_t)
    d = xkv.dims(B, Hkv * G, Hkv, hd, nC * 8, 8, 16, 16, xkv.XKV_BF16)
    scores = torch.full((B, Hkv, nC), float("nan"), dtype=torch.float64, device=DEV)
    xkv.xkv_score_landmarks(d, _dev(lm_t), _dev(q_t), scores)
    torch.cuda.synchronize()
    assert np.array_equal(scores.cpu().numpy().view(np.uint64), ref.view(np.uint64))


# ------------------------------------------------------------------------ selection
def _run_select(xkv, scores_np, top_k, n_sink, n_recent, chunk=8):
    B, Hkv, nC = scores_np.shape
    d = xkv.dims(B, Hkv, Hkv, 64, nC * chunk, chunk, 16, 16, xkv.XKV_BF16)
    n_sel = xkv.xkv_n_selected(nC, top_k, n_sink, n_recent)
    sel = torch.full((B, Hkv, n_sel), -7, dtype=torch.int32, device=DEV)
    got_n = xkv.xkv_select_chunks(d, torch.from_numpy(scores_np).to(DEV), top_k, n_sink,
                                  n_recent, sel)
    torch.cuda.synchronize()
    assert got_n == n_sel
    return sel.cpu().numpy()


@pytest.mark.parametrize("w", XKV_CASES, ids=lambda w: w.name)
def test_select_bit_exact(xkv, ora, w):
    x = _layer_inputs(w)
    lm = _host_lm(ora, ora.build_landmarks(x["Ak"], x["Bkt"], w.n_kv_heads, w.head_dim, w.chunk))
    s = ora.score_landmarks(lm, x["q"])
    ref = ora.select_chunks(s, w.top_k, w.n_sink, w.n_recent)
    got = _run_select(xkv, s, w.top_k, w.n_sink, w.n_recent, w.chunk)
    assert np.array_equal(got, ref)
    for b, nd in enumerate(x["needles"]):
        for g in range(w.n_kv_heads):
            assert set(nd.tolist()) <= set(got[b, g].tolist())


@pytest.mark.parametrize("nC,top_k,n_sink,n_recent", [
    (4096, 256, 1, 4), (4097 - 1, 0, 1, 4), (1000, 990, 1, 4), (1000, 995, 1, 4),
    (1000, 2000, 1, 4), (37, 5, 3, 3), (5, 2, 3, 3), (16384, 128, 1, 4), (1, 1, 0, 0),
    (2048, 1, 0, 0), (3000, 2999, 0, 0), (777, 100, 0, 9)])
def test_select_edge_cases_with_ties(xkv, ora, nC, top_k, n_sink, n_recent):
    rng = np.random.default_rng(nC + top_k)
    B, Hkv = 2, 3
    s = rng.integers(-20, 21, size=(B, Hkv, nC)).astype(np.float64)   # heavy exact ties
    s[0, 0] = 1.0                                                      # all tied
    s[1, 2, ::2] = -0.0
    s[1, 2, 1::2] = 0.0                                               # signed zeros
    ref = ora.select_chunks(s, top_k, n_sink, n_recent)
    got = _run_select(xkv, s, top_k, n_sink, n_recent)
    assert np.array_equal(got, ref)


def test_select_ranked_bin_with_ties(xkv, ora):
    """Distinct scores except a dozen chunks planted at exactly the k-th value: the radix
    descent stops at a bin of a few keys (ranked directly, ties by index)."""
    rng = np.random.default_rng(21)
    B, Hkv, nC, k = 2, 3, 4096, 256
    s = rng.standard_normal((B, Hkv, nC))
    for b in range(B):
        for g in range(Hkv):
            v = np.sort(s[b, g, 1:nC - 4])[::-1][k - 6]
            idx = rng.choice(np.arange(1, nC - 4), 12, replace=False)
            s[b, g, idx] = v
    ref = ora.select_chunks(s, k, 1, 4)
    assert np.array_equal(_run_select(xkv, s, k, 1, 4), ref)


def test_select_distinct_scores_extremes(xkv, ora):
    rng = np.random.default_rng(9)
    s = rng.standard_normal((1, 2, 3000)) * 1e300
    s[0, 1, :10] = [1e-320, -1e-320, 5e-324, -5e-324, 1e308, -1e308, 0, -0.0,
                    1, -1]
    ref = ora.select_chunks(s, 77, 2, 2)
    assert np.array_equal(_run_select(xkv, s, 77, 2, 2), ref)


def test_select_nan_scores_mark_the_unit_failed(xkv, ora):
    """A NaN score (how a failed scoring launch shows) makes its unit select -1
    everywhere; the other units are selected as usual."""
    rng = np.random.default_rng(4)
    s = rng.standard_normal((2, 3, 500))
    s[1, 2, 123] = np.nan
    got = _run_select(xkv, s, 20, 1, 4)
    assert np.all(got[1, 2] == -1)
    good = np.ones((2, 3), dtype=bool)
    good[1, 2] = False
    ref = ora.select_chunks(np.where(np.isnan(s), 0.0, s), 20, 1, 4)
    assert np.array_equal(got[good], ref[good])


# ------------------------------------------------------------ reconstruct + attend
def _attend(xkv, w, x, sel, dense=False):
    d = xkv.dims_of(w)
    n_sel = 0 if dense else sel.shape[2]
    mode = xkv.XKV_MODE_DENSE if dense else xkv.XKV_MODE_SELECTIVE
    ws = torch.empty(max(1, xkv.xkv_workspace_bytes(d, n_sel, mode)), dtype=torch.uint8,
                     device=DEV)
    out = torch.full((w.batch, w.n_q_heads, w.head_dim), float("nan"), device=DEV)
    sel_d = None if dense else torch.from_numpy(sel).to(DEV)
    xkv.xkv_reconstruct_attend(d, _dev(x["Ak"]), _dev(x["Av"]), _dev(x["Bkt"]), _dev(x["Bvt"]),
                               _dev(x["q"]), sel_d, n_sel, out, ws)
    torch.cuda.synchronize()
    return out.cpu().numpy()


@pytest.mark.parametrize("w", XKV_CASES, ids=lambda w: w.name)
def test_reconstruct_attend_selective(xkv, ora, w):
    x = _layer_inputs(w)
    lm = _host_lm(ora, ora.build_landmarks(x["Ak"], x["Bkt"], w.n_kv_heads, w.head_dim, w.chunk))
    sel = ora.select_chunks(ora.score_landmarks(lm, x["q"]), w.top_k, w.n_sink, w.n_recent)
    ref = ora.reconstruct_attend(x["Ak"], x["Av"], x["Bkt"], x["Bvt"], x["q"], sel, w.chunk)
    got = _attend(xkv, w, x, sel)
    compare_outputs(got, ref, w.dtype)


@pytest.mark.parametrize("G", [1, 2, 6, 7, 8, 16])
def test_reconstruct_attend_group_sizes(xkv, ora, G):
    """The tensor-core kernel for group sizes on both sides of its role split: eight
    producer warps up to 6 query heads per KV head, four above (the larger epilogue needs
    the registers)."""
    w = dataclasses.replace(synth.reduced(synth.LLAMA8B_SR_32K, batch=2, ctx_len=2048, top_k=24),
                            n_kv_heads=2, n_q_heads=2 * G, name=f"sr_g{G}")
    x = _layer_inputs(w)
    lm = _host_lm(ora, ora.build_landmarks(x["Ak"], x["Bkt"], w.n_kv_heads, w.head_dim, w.chunk))
    sel = ora.select_chunks(ora.score_landmarks(lm, x["q"]), w.top_k, w.n_sink, w.n_recent)
    ref = ora.reconstruct_attend(x["Ak"], x["Av"], x["Bkt"], x["Bvt"], x["q"], sel, w.chunk)
    compare_outputs(_attend(xkv, w, x, sel), ref, w.dtype)


@pytest.mark.parametrize("w", [LLAMA_R, QWEN14_R], ids=lambda w: w.name)
def test_reconstruct_attend_cuda_core_path_bf16(xkv, ora, w, monkeypatch):
    """The CUDA-core kernel on bf16 shapes the tensor-core kernel normally takes."""
    monkeypatch.setenv("XKV_FORCE_SIMT", "1")
    x = _layer_inputs(w)
    lm = _host_lm(ora, ora.build_landmarks(x["Ak"], x["Bkt"], w.n_kv_heads, w.head_dim, w.chunk))
    sel = ora.select_chunks(ora.score_landmarks(lm, x["q"]), w.top_k, w.n_sink, w.n_recent)
    ref = ora.reconstruct_attend(x["Ak"], x["Av"], x["Bkt"], x["Bvt"], x["q"], sel, w.chunk)
    compare_outputs(_attend(xkv, w, x, sel), ref, w.dtype)


@pytest.mark.parametrize("force_simt", [False, True], ids=["tensor_core", "cuda_core"])
def test_reconstruct_attend_invalid_selection_fails_loudly(xkv, ora, monkeypatch, force_simt):
    """A chunk index outside [0, nC) fails the call on the device: every output is NaN
    and the workspace status word holds the INVALID_ARG bit; the next call is clean."""
    if force_simt:
        monkeypatch.setenv("XKV_FORCE_SIMT", "1")
    w = LLAMA_R
    x = _layer_inputs(w)
    lm = _host_lm(ora, ora.build_landmarks(x["Ak"], x["Bkt"], w.n_kv_heads, w.head_dim, w.chunk))
    sel = ora.select_chunks(ora.score_landmarks(lm, x["q"]), w.top_k, w.n_sink, w.n_recent)
    d = xkv.dims_of(w)
    ws = torch.empty(xkv.xkv_workspace_bytes(d, sel.shape[2], xkv.XKV_MODE_SELECTIVE),
                     dtype=torch.uint8, device=DEV)
    out = torch.zeros((w.batch, w.n_q_heads, w.head_dim), device=DEV)
    args = [_dev(x["Ak"]), _dev(x["Av"]), _dev(x["Bkt"]), _dev(x["Bvt"]), _dev(x["q"])]
    for bad in (-1, w.n_chunks):
        sel_bad = sel.copy()
        sel_bad[1, 0, 3] = bad
        xkv.xkv_reconstruct_attend(d, *args, torch.from_numpy(sel_bad).to(DEV), sel.shape[2],
                                   out, ws)
        torch.cuda.synchronize()
        assert torch.isnan(out).all()
        status = int(ws[:4].cpu().view(torch.int32).item())
        assert status & (1 << xkv.XKV_ERR_INVALID_ARG)
    xkv.xkv_reconstruct_attend(d, *args, torch.from_numpy(sel).to(DEV), sel.shape[2], out, ws)
    torch.cuda.synchronize()
    assert int(ws[:4].cpu().view(torch.int32).item()) == 0
    ref = ora.reconstruct_attend(x["Ak"], x["Av"], x["Bkt"], x["Bvt"], x["q"], sel, w.chunk)
    compare_outputs(out.cpu().numpy(), ref, w.dtype)


@pytest.mark.parametrize("w", [DENSE_R, TINY], ids=lambda w: w.name)
def test_reconstruct_attend_dense(xkv, ora, w):
    x = _layer_inputs(w)
    ref = ora.reconstruct_attend(x["Ak"], x["Av"], x["Bkt"], x["Bvt"], x["q"], None, w.chunk)
    got = _attend(xkv, w, x, None, dense=True)
    compare_outputs(got, ref, w.dtype)


@pytest.mark.parametrize("n_sel", [1, 3, 17, 128])
def test_reconstruct_attend_selection_sizes(xkv, ora, n_sel):
    """One chunk (8 rows, a single partial tile) up to every chunk."""
    w = dataclasses.replace(LLAMA_R, ctx_len=1024, batch=1)
    x = _layer_inputs(w)
    rng = np.random.default_rng(n_sel)
    sel = np.stack([np.sort(rng.choice(w.n_chunks, n_sel, replace=False))
                    for _ in range(w.n_kv_heads)])[None].astype(np.int32)
    ref = ora.reconstruct_attend(x["Ak"], x["Av"], x["Bkt"], x["Bvt"], x["q"], sel, w.chunk)
    compare_outputs(_attend(xkv, w, x, sel), ref, w.dtype)


def test_pipeline_end_to_end_tiny(xkv, ora):
    """The whole decode step of the tiny fp32 workload on the GPU (landmarks built on the
    GPU too) against the oracle's pipeline."""
    w = TINY
    d = xkv.dims_of(w)
    for layer in range(w.n_layers):
        x = _layer_inputs(w, layer)
        lm_ref = ora.build_landmarks(x["Ak"], x["Bkt"], w.n_kv_heads, w.head_dim, w.chunk)
        s_ref = ora.score_landmarks(ora.to_torch(lm_ref), x["q"])
        sel_ref = ora.select_chunks(s_ref, w.top_k, w.n_sink, w.n_recent)
        o_ref = ora.reconstruct_attend(x["Ak"], x["Av"], x["Bkt"], x["Bvt"], x["q"], sel_ref,
                                       w.chunk)
        lm = torch.empty((w.batch, w.n_kv_heads, w.n_chunks, w.head_dim), device=DEV)
        xkv.xkv_build_landmarks(d, _dev(x["Ak"]), _dev(x["Bkt"]), lm)
        sc = torch.empty((w.batch, w.n_kv_heads, w.n_chunks), dtype=torch.float64, device=DEV)
        xkv.xkv_score_landmarks(d, lm, _dev(x["q"]), sc)
        sel = torch.empty((w.batch, w.n_kv_heads, w.n_sel), dtype=torch.int32, device=DEV)
        xkv.xkv_select_chunks(d, sc, w.top_k, w.n_sink, w.n_recent, sel)
        ws = torch.empty(xkv.xkv_workspace_bytes(d, w.n_sel, 0), dtype=torch.uint8, device=DEV)
        out = torch.empty((w.batch, w.n_q_heads, w.head_dim), device=DEV)
        xkv.xkv_reconstruct_attend(d, _dev(x["Ak"]), _dev(x["Av"]), _dev(x["Bkt"]),
                                   _dev(x["Bvt"]), _dev(x["q"]), sel, w.n_sel, out, ws)
        torch.cuda.synchronize()
        assert np.array_equal(lm.cpu().numpy(), lm_ref)
        assert np.array_equal(sc.cpu().numpy().view(np.uint64), s_ref.view(np.uint64))
        assert np.array_equal(sel.cpu().numpy(), sel_ref)
        compare_outputs(out.cpu().numpy(), o_ref, w.dtype)


@pytest.mark.parametrize("plain_order", [False, True], ids=["chained", "plain_order"])
def test_device_chain_back_to_back(xkv, ora, monkeypatch, plain_order):
    """Score, select and attend of two bf16 layers issued back to back on one stream with
    no host synchronisation in between, the kernels chained by programmatic dependent
    launch (or, with XKV_NO_PDL, in plain stream order): scores and selections equal the
    oracle's bit for bit and the outputs agree within tolerance."""
    if plain_order:
        monkeypatch.setenv("XKV_NO_PDL", "1")
    w = LLAMA_R
    d = xkv.dims_of(w)
    refs, devs = [], []
    for layer in range(2):
        x = _layer_inputs(w, layer)
        lm_np = ora.build_landmarks(x["Ak"], x["Bkt"], w.n_kv_heads, w.head_dim, w.chunk)
        s_ref = ora.score_landmarks(_host_lm(ora, lm_np), x["q"])
        sel_ref = ora.select_chunks(s_ref, w.top_k, w.n_sink, w.n_recent)
        o_ref = ora.reconstruct_attend(x["Ak"], x["Av"], x["Bkt"], x["Bvt"], x["q"], sel_ref,
                                       w.chunk)
        refs.append((s_ref, sel_ref, o_ref))
        devs.append(dict(lm=_dev(_host_lm(ora, lm_np)), q=_dev(x["q"]), Ak=_dev(x["Ak"]),
                         Av=_dev(x["Av"]), Bkt=_dev(x["Bkt"]), Bvt=_dev(x["Bvt"])))
    torch.cuda.synchronize()
    ws = torch.empty(xkv.xkv_workspace_bytes(d, w.n_sel, 0), dtype=torch.uint8, device=DEV)
    got = []
    for t in devs:
        sc = torch.empty((w.batch, w.n_kv_heads, w.n_chunks), dtype=torch.float64, device=DEV)
        sel = torch.empty((w.batch, w.n_kv_heads, w.n_sel), dtype=torch.int32, device=DEV)
        out = torch.empty((w.batch, w.n_q_heads, w.head_dim), device=DEV)
        xkv.xkv_score_landmarks(d, t["lm"], t["q"], sc)
        xkv.xkv_select_chunks(d, sc, w.top_k, w.n_sink, w.n_recent, sel)
        xkv.xkv_reconstruct_attend(d, t["Ak"], t["Av"], t["Bkt"], t["Bvt"], t["q"], sel,
                                   w.n_sel, out, ws)
        got.append((sc, sel, out))
    torch.cuda.synchronize()
    for (sc, sel, out), (s_ref, sel_ref, o_ref) in zip(got, refs):
        assert np.array_equal(sc.cpu().numpy().view(np.uint64), s_ref.view(np.uint64))
        assert np.array_equal(sel.cpu().numpy(), sel_ref)
        compare_outputs(out.cpu().numpy(), o_ref, w.dtype)
    assert int(ws[:4].cpu().view(torch.int32).item()) == 0


# ------------------------------------------------------------- generated-token tail
@pytest.mark.parametrize("w,dense,n_tail", [(LLAMA_R, False, 37), (LLAMA_R, False, 1),
                                            (LLAMA_R, False, 0), (TINY, False, 5),
                                            (DENSE_R, True, 17), (QWEN14_R, False, 300)],
                         ids=lambda v: getattr(v, "name", str(v)))
def test_reconstruct_attend_with_tail(xkv, ora, w, dense, n_tail):
    """Selected (or all) reconstructed rows plus an uncompressed tail in one softmax."""
    x = _layer_inputs(w)
    T_max = max(n_tail, 1) + 3
    rng = np.random.default_rng(n_tail + 7)
    dt = torch.float32 if w.dtype == "f32" else torch.bfloat16
    Kt = torch.tensor(rng.standard_normal((w.batch, w.n_kv_heads, T_max, w.head_dim)) * 0.3,
                      dtype=dt)
    Vt = torch.tensor(rng.standard_normal((w.batch, w.n_kv_heads, T_max, w.head_dim)), dtype=dt)
    sel = None
    if not dense:
        lm = _host_lm(ora, ora.build_landmarks(x["Ak"], x["Bkt"], w.n_kv_heads, w.head_dim,
                                               w.chunk))
        sel = ora.select_chunks(ora.score_landmarks(lm, x["q"]), w.top_k, w.n_sink, w.n_recent)
    ref = ora.reconstruct_attend_tail(x["Ak"], x["Av"], x["Bkt"], x["Bvt"], x["q"], sel,
                                      w.chunk, Kt, Vt, n_tail)
    d = xkv.dims_of(w)
    n_sel = 0 if sel is None else sel.shape[2]
    ws = torch.empty(xkv.xkv_tail_workspace_bytes(d, n_sel, T_max), dtype=torch.uint8,
                     device=DEV)
    out = torch.full((w.batch, w.n_q_heads, w.head_dim), float("nan"), device=DEV)
    xkv.xkv_reconstruct_attend_tail(d, _dev(x["Ak"]), _dev(x["Av"]), _dev(x["Bkt"]),
                                    _dev(x["Bvt"]), _dev(x["q"]),
                                    None if sel is None else torch.from_numpy(sel).to(DEV),
                                    n_sel, _dev(Kt), _dev(Vt), T_max, n_tail, out, ws)
    torch.cuda.synchronize()
    compare_outputs(out.cpu().numpy(), ref, w.dtype)


# ------------------------------------------------------- reassociated (rank space)
def _reassoc(xkv, w, x, sel):
    d = xkv.dims_of(w)
    n_sel = 0 if sel is None else sel.shape[2]
    ws = torch.empty(xkv.xkv_workspace_bytes(d, n_sel, xkv.XKV_MODE_REASSOC), dtype=torch.uint8,
                     device=DEV)
    out = torch.full((w.batch, w.n_q_heads, w.head_dim), float("nan"), device=DEV)
    xkv.xkv_reassociated_attend(d, _dev(x["Ak"]), _dev(x["Av"]), _dev(x["Bkt"]), _dev(x["Bvt"]),
                                _dev(x["q"]), None if sel is None else torch.from_numpy(sel).to(DEV),
                                n_sel, out, ws)
    torch.cuda.synchronize()
    return out.cpu().numpy(), ws


@pytest.mark.parametrize("w", [LLAMA_R, QWEN14_R], ids=lambda w: w.name)
def test_reassociated_attend_selective(xkv, ora, w):
    """Rank-space attention equals the oracle's explicit reconstruct-then-attend."""
    x = _layer_inputs(w)
    lm = _host_lm(ora, ora.build_landmarks(x["Ak"], x["Bkt"], w.n_kv_heads, w.head_dim, w.chunk))
    sel = ora.select_chunks(ora.score_landmarks(lm, x["q"]), w.top_k, w.n_sink, w.n_recent)
    ref = ora.reconstruct_attend(x["Ak"], x["Av"], x["Bkt"], x["Bvt"], x["q"], sel, w.chunk)
    compare_outputs(_reassoc(xkv, w, x, sel)[0], ref, w.dtype)


def test_reassociated_attend_dense(xkv, ora):
    w = DENSE_R
    x = _layer_inputs(w)
    ref = ora.reconstruct_attend(x["Ak"], x["Av"], x["Bkt"], x["Bvt"], x["q"], None, w.chunk)
    compare_outputs(_reassoc(xkv, w, x, None)[0], ref, w.dtype)


# Dense mode runs the head-batched kernel (one pass over A for all heads of a sequence,
# spans of 128-token tiles): ragged last tiles, several spans per sequence and several
# tiles per span, batches whose spans do not fill the GPU evenly, 8 / 16 / 24 / 32 heads
# and smaller ranks.
DENSE_CASES = [
    synth.reduced(synth.LLAMA8B_DENSE_128K, batch=1, ctx_len=1000, name="dense_ragged"),
    synth.reduced(synth.LLAMA8B_DENSE_128K, batch=3, ctx_len=2056, name="dense_b3"),
    synth.reduced(synth.LLAMA8B_DENSE_128K, batch=1, ctx_len=40960, name="dense_40k_spans"),
    dataclasses.replace(synth.reduced(synth.LLAMA8B_DENSE_128K, batch=2, ctx_len=1536),
                        n_q_heads=16, n_kv_heads=8, name="dense_hq16_g2"),
    dataclasses.replace(synth.reduced(synth.LLAMA8B_DENSE_128K, batch=2, ctx_len=1152),
                        n_q_heads=8, n_kv_heads=8, rank_k=256, rank_v=384, name="dense_hq8_g1"),
    dataclasses.replace(synth.reduced(synth.LLAMA8B_DENSE_128K, batch=1, ctx_len=2048),
                        n_q_heads=24, n_kv_heads=6, rank_k=384, rank_v=640, name="dense_hq24"),
    # 32 or more spans per sequence: the merge and the projection run as one kernel
    # (slices of 32 and of 128 rank columns, one and four heads per group)
    dataclasses.replace(synth.reduced(synth.LLAMA8B_DENSE_128K, batch=1, ctx_len=8192),
                        n_q_heads=8, n_kv_heads=8, rank_k=256, rank_v=384,
                        name="dense_hq8_many_spans"),
    synth.reduced(synth.LLAMA8B_DENSE_128K, batch=2, ctx_len=16384, name="dense_b2_many_spans"),
]


def test_reassociated_attend_dense_more_items_than_sms(xkv, ora):
    """160 sequences of 4 tiles: one span per sequence, so 160 items on at most 148 CTAs
    and some CTAs take a second item (the next item's Q~, the accumulator hand-back and
    the buffer parities carried across items)."""
    w = dataclasses.replace(synth.reduced(synth.LLAMA8B_DENSE_128K, batch=160, ctx_len=512),
                            rank_k=256, rank_v=384, name="dense_b160")
    x = _layer_inputs(w)
    units = [(b, g) for b in (0, 11, 12, 147, 148, 159) for g in (0, w.n_kv_heads - 1)]
    ref = ora.reconstruct_attend(x["Ak"], x["Av"], x["Bkt"], x["Bvt"], x["q"], None, w.chunk,
                                 units=units)
    got = _reassoc(xkv, w, x, None)[0]
    G = w.n_q_heads // w.n_kv_heads
    for b, g in units:
        compare_outputs(got[b, g * G:(g + 1) * G], ref[b, g * G:(g + 1) * G], w.dtype)


@pytest.mark.parametrize("w", DENSE_CASES, ids=lambda w: w.name)
def test_reassociated_attend_dense_all_heads(xkv, ora, w):
    x = _layer_inputs(w)
    units = None if w.ctx_len <= 4096 else [(0, 0), (w.batch - 1, w.n_kv_heads - 1)]
    ref = ora.reconstruct_attend(x["Ak"], x["Av"], x["Bkt"], x["Bvt"], x["q"], None, w.chunk,
                                 units=units)
    got = _reassoc(xkv, w, x, None)[0]
    G = w.n_q_heads // w.n_kv_heads
    for b, g in units or [(b, g) for b in range(w.batch) for g in range(w.n_kv_heads)]:
        compare_outputs(got[b, g * G:(g + 1) * G], ref[b, g * G:(g + 1) * G], w.dtype)


@pytest.mark.parametrize("n_sel", [1, 3, 17, 33, 128])
def test_reassociated_selection_sizes(xkv, ora, n_sel):
    """Items of one chunk, odd 8-row group counts (padded MMA steps), several splits."""
    w = LLAMA_R
    x = _layer_inputs(w)
    rng = np.random.default_rng(n_sel)
    sel = np.sort(np.stack([np.stack([rng.choice(w.n_chunks, n_sel, replace=False)
                                      for _ in range(w.n_kv_heads)]) for _ in range(w.batch)]),
                  axis=2).astype(np.int32)
    ref = ora.reconstruct_attend(x["Ak"], x["Av"], x["Bkt"], x["Bvt"], x["q"], sel, w.chunk)
    compare_outputs(_reassoc(xkv, w, x, sel)[0], ref, w.dtype)


def test_reassociated_invalid_selection_and_shapes(xkv, ora):
    w = LLAMA_R
    x = _layer_inputs(w)
    sel = np.tile(np.arange(10, dtype=np.int32), (w.batch, w.n_kv_heads, 1))
    sel[0, 1, 4] = w.n_chunks                       # out of range: NaN outputs, status bit
    out, ws = _reassoc(xkv, w, x, sel)
    assert np.isnan(out).all()
    assert int(ws[:4].cpu().view(torch.int32).item()) & (1 << xkv.XKV_ERR_INVALID_ARG)
    # fp32 is outside the rank-space kernel: refused before any launch
    d = xkv.dims_of(TINY)
    assert xkv.xkv_workspace_bytes(d, 0, xkv.XKV_MODE_REASSOC) == 0
    dummy = torch.zeros(64, dtype=torch.float32, device=DEV)
    with pytest.raises(xkv.XkvError) as e:
        xkv.xkv_reassociated_attend(d, dummy, dummy, dummy, dummy, dummy, None, 0, dummy,
                                    torch.zeros(1 << 20, dtype=torch.uint8, device=DEV))
    assert e.value.status == xkv.XKV_ERR_UNSUPPORTED


# ----------------------------------------------------------------------------- R-CLA
RCLA_R = synth.reduced(synth.QWEN3_8B_RCLA_32K, batch=2, ctx_len=1500, n_layers=8,
                       extra_rows=8)


@pytest.mark.parametrize("w", [RCLA_R, dataclasses.replace(RCLA_R, dtype="f32", head_dim=64,
                                                            n_q_heads=10, n_kv_heads=2,
                                                            name="rcla_f32_g5")],
                         ids=lambda w: w.name)
def test_rcla_decode_step_matches_oracle(xkv, ora, w):
    """One decode step over all layers: leaders append their new row, then every layer
    attends its leader's cache; outputs and the caches after the step must agree."""
    length = w.ctx_len
    x = synth.np_rcla_inputs(w, seed=0, len_rows=length)
    S = synth.leader_set(w)
    lo = ora.leader_map(S, w.n_layers)
    K_ref = ora.as_float64(x["K_lead"]).astype(np.float32) if w.dtype == "f32" else \
        x["K_lead"].view(torch.int16).numpy().view(np.uint16).copy()
    V_ref = ora.as_float64(x["V_lead"]).astype(np.float32) if w.dtype == "f32" else \
        x["V_lead"].view(torch.int16).numpy().view(np.uint16).copy()
    K = _dev(x["K_lead"])
    V = _dev(x["V_lead"])
    d = xkv.dims(w.batch, w.n_q_heads, w.n_kv_heads, w.head_dim, w.L_max, dtype=w.dtype)
    ws = torch.empty(xkv.xkv_workspace_bytes(d, 0, xkv.XKV_MODE_RCLA), dtype=torch.uint8,
                     device=DEV)
    for layer in range(w.n_layers):
        leader = lo[layer] == layer
        slot = S.index(lo[layer])
        kn = x["k_new"][slot] if leader else None
        vn = x["v_new"][slot] if leader else None
        n = length if leader else length + 1
        ref = ora.rcla_decode_attend(layer, lo, K_ref, V_ref, n, kn, vn, x["q"][layer])
        out = torch.empty((w.batch, w.n_q_heads, w.head_dim), device=DEV)
        xkv.rcla_decode_attend(d, layer, lo, K, V, w.L_max, n,
                               _dev(kn) if leader else None, _dev(vn) if leader else None,
                               _dev(x["q"][layer]), out, ws)
        torch.cuda.synchronize()
        compare_outputs(out.cpu().numpy(), ref, w.dtype)
    if w.dtype == "f32":
        assert np.array_equal(K.cpu().numpy(), K_ref) and np.array_equal(V.cpu().numpy(), V_ref)
    else:
        assert np.array_equal(K.cpu().view(torch.int16).numpy().view(np.uint16), K_ref)
        assert np.array_equal(V.cpu().view(torch.int16).numpy().view(np.uint16), V_ref)


@pytest.mark.parametrize("length", [0, 1, 127, 128, 129, 4095])
def test_rcla_lengths(xkv, ora, length):
    """From a single (new) row up to several tiles and splits, ragged tails."""
    w = synth.reduced(synth.QWEN3_8B_RCLA_32K, batch=1, ctx_len=max(length, 1), n_layers=2,
                      extra_rows=1, outlier_frac=0.0)
    x = synth.np_rcla_inputs(w, seed=length, len_rows=length)
    lo = ora.leader_map([0], 2)
    K_ref = x["K_lead"].view(torch.int16).numpy().view(np.uint16).copy()
    V_ref = x["V_lead"].view(torch.int16).numpy().view(np.uint16).copy()
    ref = ora.rcla_decode_attend(0, lo, K_ref, V_ref, length, x["k_new"][0], x["v_new"][0],
                                 x["q"][0])
    d = xkv.dims(w.batch, w.n_q_heads, w.n_kv_heads, w.head_dim, w.L_max, dtype=w.dtype)
    ws = torch.empty(xkv.xkv_workspace_bytes(d, 0, xkv.XKV_MODE_RCLA), dtype=torch.uint8,
                     device=DEV)
    out = torch.empty((w.batch, w.n_q_heads, w.head_dim), device=DEV)
    K, V = _dev(x["K_lead"]), _dev(x["V_lead"])
    xkv.rcla_decode_attend(d, 0, lo, K, V, w.L_max, length, _dev(x["k_new"][0]),
                           _dev(x["v_new"][0]), _dev(x["q"][0]), out, ws)
    torch.cuda.synchronize()
    compare_outputs(out.cpu().numpy(), ref, w.dtype)
    assert np.array_equal(K.cpu().view(torch.int16).numpy().view(np.uint16), K_ref)


@pytest.mark.parametrize("G,length", [(1, 700), (2, 1300), (5, 2100), (8, 900), (4, 5000)])
def test_rcla_group_sizes(xkv, ora, G, length):
    """Every group size of the bf16 kernels; a leader appends, then a follower attends."""
    w = dataclasses.replace(
        synth.reduced(synth.QWEN3_8B_RCLA_32K, batch=2, ctx_len=length, n_layers=2,
                      extra_rows=2, outlier_frac=0.01),
        n_kv_heads=2, n_q_heads=2 * G, name=f"rcla_g{G}")
    x = synth.np_rcla_inputs(w, seed=G, len_rows=length)
    lo = ora.leader_map([0], 2)
    K_ref = x["K_lead"].view(torch.int16).numpy().view(np.uint16).copy()
    V_ref = x["V_lead"].view(torch.int16).numpy().view(np.uint16).copy()
    d = xkv.dims(w.batch, w.n_q_heads, w.n_kv_heads, w.head_dim, w.L_max, dtype=w.dtype)
    ws = torch.empty(xkv.xkv_workspace_bytes(d, 0, xkv.XKV_MODE_RCLA), dtype=torch.uint8,
                     device=DEV)
    K, V = _dev(x["K_lead"]), _dev(x["V_lead"])
    for layer in (0, 1):
        leader = layer == 0
        n = length if leader else length + 1
        kn = x["k_new"][0] if leader else None
        vn = x["v_new"][0] if leader else None
        ref = ora.rcla_decode_attend(layer, lo, K_ref, V_ref, n, kn, vn, x["q"][layer])
        out = torch.empty((w.batch, w.n_q_heads, w.head_dim), device=DEV)
        xkv.rcla_decode_attend(d, layer, lo, K, V, w.L_max, n, _dev(kn) if leader else None,
                               _dev(vn) if leader else None, _dev(x["q"][layer]), out, ws)
        torch.cuda.synchronize()
        compare_outputs(out.cpu().numpy(), ref, w.dtype)
    assert np.array_equal(K.cpu().view(torch.int16).numpy().view(np.uint16), K_ref)
    assert np.array_equal(V.cpu().view(torch.int16).numpy().view(np.uint16), V_ref)


@pytest.mark.parametrize("switch", ["XKV_NO_TC", "XKV_FORCE_SIMT"])
@pytest.mark.parametrize("G,length", [(4, 5000), (5, 2100)])
def test_rcla_other_kernels_bf16(xkv, ora, monkeypatch, switch, G, length):
    """The TMA + CUDA-core kernel (XKV_NO_TC) and the plain CUDA-core kernel
    (XKV_FORCE_SIMT) on bf16 caches the tensor-core kernel normally takes."""
    monkeypatch.setenv(switch, "1")
    test_rcla_group_sizes(xkv, ora, G, length)


def test_rcla_outlier_values_are_attended(xkv, ora):
    """Rows whose V is 20x larger (1% of tokens) dominate nothing by themselves but must be
    carried exactly: compare against the oracle with the outliers present."""
    w = synth.reduced(synth.QWEN3_8B_RCLA_32K, batch=2, ctx_len=3000, n_layers=1,
                      extra_rows=0)
    x = synth.np_rcla_inputs(w, seed=5, len_rows=3000)
    lo = [0]
    K_ref = x["K_lead"].view(torch.int16).numpy().view(np.uint16).copy()
    V_ref = x["V_lead"].view(torch.int16).numpy().view(np.uint16).copy()
    ref = ora.rcla_decode_attend(0, lo, K_ref, V_ref, 3000, None, None, x["q"][0])
    d = xkv.dims(w.batch, w.n_q_heads, w.n_kv_heads, w.head_dim, w.L_max, dtype=w.dtype)
    ws = torch.empty(xkv.xkv_workspace_bytes(d, 0, xkv.XKV_MODE_RCLA), dtype=torch.uint8,
                     device=DEV)
    out = torch.empty((w.batch, w.n_q_heads, w.head_dim), device=DEV)
    xkv.rcla_decode_attend(d, 0, lo, _dev(x["K_lead"]), _dev(x["V_lead"]), w.L_max, 3000,
                           None, None, _dev(x["q"][0]), out, ws)
    torch.cuda.synchronize()
    compare_outputs(out.cpu().numpy(), ref, w.dtype)


def test_unsupported_device_paths_fail_loudly(xkv):
    """Argument errors surface as exceptions from the binding (no silent fallback)."""
    d = xkv.dims(1, 4, 2, 64, 64, 8, 16, 16, xkv.XKV_BF16)
    with pytest.raises(xkv.XkvError):
        xkv.xkv_score_landmarks(d, None, None, None)


# ------------------------------------------------------------ repeat-run determinism
def test_repeat_runs_are_bit_identical(xkv, ora):
    """With no race checker on this pool, repeat runs stand in for one: every stage of
    the decode path (scores, selection, explicit and rank-space attention, R-CLA with its
    cache update) has a fixed reduction order and no atomics on data, so five runs on the
    same inputs must agree bit for bit.  A race in the selection, the split merge or a
    shared-memory ring shows up as a difference."""
    w = QWEN14_R
    d = xkv.dims_of(w)
    x = _layer_inputs(w)
    lm = _dev(_host_lm(ora, ora.build_landmarks(x["Ak"], x["Bkt"], w.n_kv_heads, w.head_dim,
                                                w.chunk)))
    g = {k: _dev(x[k]) for k in ("Ak", "Av", "Bkt", "Bvt", "q")}
    runs = []
    for _ in range(5):
        sc = torch.empty((w.batch, w.n_kv_heads, w.n_chunks), dtype=torch.float64, device=DEV)
        sel = torch.empty((w.batch, w.n_kv_heads, w.n_sel), dtype=torch.int32, device=DEV)
        xkv.xkv_score_landmarks(d, lm, g["q"], sc)
        xkv.xkv_select_chunks(d, sc, w.top_k, w.n_sink, w.n_recent, sel)
        outs = []
        for fn, mode in ((xkv.xkv_reconstruct_attend, xkv.XKV_MODE_SELECTIVE),
                         (xkv.xkv_reassociated_attend, xkv.XKV_MODE_REASSOC)):
            ws = torch.empty(xkv.xkv_workspace_bytes(d, w.n_sel, mode), dtype=torch.uint8,
                             device=DEV)
            out = torch.empty((w.batch, w.n_q_heads, w.head_dim), device=DEV)
            fn(d, g["Ak"], g["Av"], g["Bkt"], g["Bvt"], g["q"], sel, w.n_sel, out, ws)
            outs.append(out)
        torch.cuda.synchronize()
        runs.append([t.cpu().numpy().copy() for t in (sc, sel, *outs)])
    for r in runs[1:]:
        for a, b in zip(runs[0], r):
            assert np.array_equal(a.view(np.uint8), b.view(np.uint8))

    wr = RCLA_R
    xr = synth.np_rcla_inputs(wr, seed=0, len_rows=wr.ctx_len)
    dr = xkv.dims(wr.batch, wr.n_q_heads, wr.n_kv_heads, wr.head_dim, wr.L_max, dtype=wr.dtype)
    wsr = torch.empty(xkv.xkv_workspace_bytes(dr, 0, xkv.XKV_MODE_RCLA), dtype=torch.uint8,
                      device=DEV)
    lo = [0] * wr.n_layers
    res = []
    for _ in range(3):
        K, V = _dev(xr["K_lead"]), _dev(xr["V_lead"])
        o = torch.empty((wr.batch, wr.n_q_heads, wr.head_dim), device=DEV)
        xkv.rcla_decode_attend(dr, 0, lo, K, V, wr.L_max, wr.ctx_len, _dev(xr["k_new"][0]),
                               _dev(xr["v_new"][0]), _dev(xr["q"][0]), o, wsr)
        torch.cuda.synchronize()
        res.append((o.cpu().numpy().copy(), K.cpu().view(torch.int16).numpy().copy()))
    for o, k in res[1:]:
        assert np.array_equal(o.view(np.uint8), res[0][0].view(np.uint8))
        assert np.array_equal(k, res[0][1])
