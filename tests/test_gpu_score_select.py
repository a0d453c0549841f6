"""GPU parity of the fused scoring + selection call (xkv_score_select) and of selections
made from landmarks built on the GPU.

* Given identical landmarks and queries, xkv_score_select must select exactly what the
  oracle selects from its canonical fp64 scores (bit for bit), whatever path a unit takes
  (fp32 pass + fp64 band, or fp64 throughout).
* Landmarks built on the GPU may differ from the oracle's by one bf16 ulp in rare
  elements, so a selection made from them may differ from the oracle's selection from
  its own landmarks -- but only at certified near-ties: a chunk selected on one side only
  must score within 2 beta of the k-th candidate score, beta bounding how far any score
  can move between the two landmark sets (the bound is derived in
  parity_util.certify_near_ties)."""
import dataclasses

import numpy as np
import pytest
import torch

from cross_layer_compressed_b200 import synth
from parity_util import certify_near_ties as certify

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda")
EXACT_PATH = 0xFFFFFFFF


@pytest.fixture(scope="module")
def xkv():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from cross_layer_compressed_b200 import build
    build.build()
    from cross_layer_compressed_b200 import xkv as m
    return m


TINY = synth.TINY_SR_F32
LLAMA_R = synth.reduced(synth.LLAMA8B_SR_32K, batch=2, ctx_len=2048, top_k=24)
LLAMA_R8 = synth.reduced(synth.LLAMA8B_SR_32K, batch=2, ctx_len=32768, top_k=256)
QWEN14_R = synth.reduced(synth.QWEN14B_SR_16K, batch=2, ctx_len=1024, top_k=20)
SMALL_HD64 = dataclasses.replace(synth.reduced(synth.LLAMA8B_SR_32K, batch=3, ctx_len=1536,
                                               top_k=11, n_needles=0),
                                 head_dim=64, n_kv_heads=2, n_q_heads=6, rank_k=96, rank_v=80,
                                 name="hd64_g3")
CASES = [TINY, LLAMA_R, QWEN14_R, SMALL_HD64]


def _dev(t):
    return t.to(DEV).contiguous()


def _fused(xkv, lm, q, B, Hq, Hkv, hd, nC, top_k, n_sink, n_recent, dtype, chunk=8):
    """Runs xkv_score_select on device tensors; returns (sel, band sizes) on the host."""
    d = xkv.dims(B, Hq, Hkv, hd, nC * chunk, chunk, 16, 16, dtype)
    n_sel = xkv.xkv_n_selected(nC, top_k, n_sink, n_recent)
    sel = torch.full((B, Hkv, max(n_sel, 1)), -7, dtype=torch.int32, device=DEV)
    ws = torch.empty(xkv.xkv_score_select_workspace_bytes(d), dtype=torch.uint8, device=DEV)
    got_n = xkv.xkv_score_select(d, lm, q, top_k, n_sink, n_recent, sel, ws)
    torch.cuda.synchronize()
    assert got_n == n_sel
    band = ws[:4 * B * Hkv].cpu().view(torch.int32).numpy().view(np.uint32).reshape(B, Hkv)
    return sel.cpu().numpy()[..., :n_sel], band


def _bf16(a):
    return torch.tensor(a, dtype=torch.float32).to(torch.bfloat16)


# ------------------------------------------------------- identical inputs: bit-exact
@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_fused_selection_bit_exact(xkv, ora, w):
    x = synth.np_xkv_layer_inputs(w, seed=0, layer=min(1, w.n_layers - 1))
    lm = ora.to_torch(ora.build_landmarks(x["Ak"], x["Bkt"], w.n_kv_heads, w.head_dim, w.chunk))
    ref = ora.select_chunks(ora.score_landmarks(lm, x["q"]), w.top_k, w.n_sink, w.n_recent)
    got, band = _fused(xkv, _dev(lm), _dev(x["q"]), w.batch, w.n_q_heads, w.n_kv_heads,
                       w.head_dim, w.n_chunks, w.top_k, w.n_sink, w.n_recent,
                       xkv.XKV_F32 if w.dtype == "f32" else xkv.XKV_BF16, w.chunk)
    assert np.array_equal(got, ref)
    # these score distributions are resolved by the fp32 pass plus a narrow band
    assert np.all(band != EXACT_PATH) and band.max() <= 64, band


@pytest.mark.parametrize("hd,G,nC,top_k,n_sink,n_recent", [
    (64, 1, 37, 5, 1, 1), (64, 8, 100, 9, 2, 3), (128, 2, 33, 4, 1, 4), (128, 8, 65, 64, 0, 0),
    (64, 4, 1, 1, 0, 0), (128, 5, 300, 20, 1, 4), (128, 3, 4096, 256, 1, 4),
    (128, 4, 16384, 128, 1, 4), (128, 16, 777, 100, 0, 9), (64, 6, 2048, 0, 1, 4),
    (128, 7, 1000, 995, 1, 4), (128, 4, 5, 2, 3, 3), (128, 4, 4097 - 1, 4000, 1, 4),
    (128, 4, 3000, 2999, 0, 0)])
def test_fused_selection_shapes_and_budgets(xkv, ora, hd, G, nC, top_k, n_sink, n_recent):
    """Every group size and head size, budgets from 0 to every candidate, sink and recent
    windows that overlap, row counts that end inside a CTA's slice."""
    B, Hkv = 2, 3
    rng = np.random.default_rng(hd * 100003 + G * 1009 + nC)
    lm = _bf16(rng.standard_normal((B, Hkv, nC, hd)))
    q = _bf16(rng.standard_normal((B, Hkv * G, hd)))
    ref = ora.select_chunks(ora.score_landmarks(lm, q), top_k, n_sink, n_recent)
    got, _ = _fused(xkv, _dev(lm), _dev(q), B, Hkv * G, Hkv, hd, nC, top_k, n_sink, n_recent,
                    xkv.XKV_BF16)
    assert np.array_equal(got, ref)


def test_fused_selection_heavy_ties_take_the_exact_path(xkv, ora):
    """Small integers: many chunks share one exact score, the band is the whole candidate
    set, and the unit is scored in fp64 throughout; ties still go to the lower index."""
    B, Hkv, G, hd, nC = 2, 2, 4, 128, 3000
    rng = np.random.default_rng(11)
    lm = _bf16(rng.integers(-2, 3, size=(B, Hkv, nC, hd)))
    lm[0, 0] = 1.0                                            # every chunk tied
    q = _bf16(rng.integers(-1, 2, size=(B, Hkv * G, hd)))
    ref = ora.select_chunks(ora.score_landmarks(lm, q), 200, 1, 4)
    got, band = _fused(xkv, _dev(lm), _dev(q), B, Hkv * G, Hkv, hd, nC, 200, 1, 4,
                       xkv.XKV_BF16)
    assert np.array_equal(got, ref)
    assert band[0, 0] == EXACT_PATH


def test_fused_selection_resolves_near_ties_in_fp64(xkv, ora):
    """Scores that fp32 cannot tell apart: 2^20 + {0.5 - 2^-9, 0.5, 0.5 + 2^-8} all round to
    2^20 + 0.5 in fp32.  100 chunks score clearly higher, the rest clearly lower, and the
    k-th score falls among the 60 near-tied chunks: they form the band, the fp64 rescore
    orders them (ties by index) exactly as the oracle does."""
    B, Hkv, G, hd, nC = 2, 3, 4, 128, 2048
    rng = np.random.default_rng(5)
    lm = np.zeros((B, Hkv, nC, hd))
    q = np.zeros((B, Hkv * G, hd))
    q[..., 0] = 1.0
    q[..., 7] = 1.0
    for b in range(B):
        for g in range(Hkv):
            perm = 1 + rng.permutation(nC - 5)                  # never sink or recent
            hi_c, mid_c = perm[:100], perm[100:160]
            lm[b, g, :, 0] = 2.0 ** 20 - 2.0 ** 15
            lm[b, g, hi_c, 0] = 2.0 ** 20 + 2.0 ** 14
            lm[b, g, mid_c, 0] = 2.0 ** 20
            lm[b, g, mid_c, 7] = rng.choice([0.5, 0.5 + 2.0 ** -8, 0.5 - 2.0 ** -9], size=60)
    lmt, qt = _bf16(lm), _bf16(q)
    assert np.array_equal(_as_f64(lmt), lm) and np.array_equal(_as_f64(qt), q)   # exact in bf16
    ref = ora.select_chunks(ora.score_landmarks(lmt, qt), 130, 1, 4)
    got, band = _fused(xkv, _dev(lmt), _dev(qt), B, Hkv * G, Hkv, hd, nC, 130, 1, 4,
                       xkv.XKV_BF16)
    assert np.array_equal(got, ref)
    assert np.all(band == 60), band     # exactly the near-tied chunks were rescored


def test_fused_selection_nan_marks_the_unit(xkv, ora):
    """A NaN landmark (outside the contract) sends its unit to the fp64 path and makes
    its entries -1, as xkv_select_chunks does for NaN scores; other units are exact."""
    B, Hkv, G, hd, nC = 2, 3, 4, 128, 500
    rng = np.random.default_rng(4)
    lm = rng.standard_normal((B, Hkv, nC, hd))
    lm[1, 2, 123, 5] = np.nan
    lmt, qt = _bf16(lm), _bf16(rng.standard_normal((B, Hkv * G, hd)))
    got, band = _fused(xkv, _dev(lmt), _dev(qt), B, Hkv * G, Hkv, hd, nC, 20, 1, 4,
                       xkv.XKV_BF16)
    assert np.all(got[1, 2] == -1) and band[1, 2] == EXACT_PATH
    good = np.ones((B, Hkv), dtype=bool)
    good[1, 2] = False
    s = ora.score_landmarks(lmt, qt)
    ref = ora.select_chunks(np.where(np.isnan(s), 0.0, s), 20, 1, 4)
    assert np.array_equal(got[good], ref[good])


def test_fused_selection_matches_the_two_call_path(xkv):
    """At the benchmark's shape (32K tokens, 4096 chunks, G = 4) on GPU-built landmarks:
    the fused call and score + select give the same selection for every unit."""
    w = LLAMA_R8
    d = xkv.dims_of(w)
    c = synth.torch_xkv_layer(w, seed=0, layer=3, device=DEV)
    q = synth.torch_layer_queries(w, 0, 3, c, device=DEV)
    lm = torch.empty((w.batch, w.n_kv_heads, w.n_chunks, w.head_dim), dtype=torch.bfloat16,
                     device=DEV)
    xkv.xkv_build_landmarks(d, c["Ak"], c["Bkt"], lm)
    scores = torch.empty((w.batch, w.n_kv_heads, w.n_chunks), dtype=torch.float64, device=DEV)
    sel2 = torch.empty((w.batch, w.n_kv_heads, w.n_sel), dtype=torch.int32, device=DEV)
    xkv.xkv_score_landmarks(d, lm, q, scores)
    xkv.xkv_select_chunks(d, scores, w.top_k, w.n_sink, w.n_recent, sel2)
    got, band = _fused(xkv, lm, q, w.batch, w.n_q_heads, w.n_kv_heads, w.head_dim, w.n_chunks,
                       w.top_k, w.n_sink, w.n_recent, xkv.XKV_BF16)
    assert np.array_equal(got, sel2.cpu().numpy())
    assert np.all(band != EXACT_PATH)


# ------------------------------------------- GPU-built landmarks: certified near-ties
def _as_f64(x):
    import oracle
    return oracle.as_float64(x)


@pytest.mark.parametrize("w", [LLAMA_R, QWEN14_R, SMALL_HD64], ids=lambda w: w.name)
def test_gpu_landmarks_select_within_certified_near_ties(xkv, ora, w):
    """The product pipeline end to end: landmarks built, scored and selected on the GPU
    (both the fused call and score + select) against the oracle's landmarks, scores and
    selection; and, on the GPU's own landmarks, bit-exact against the oracle."""
    x = synth.np_xkv_layer_inputs(w, seed=0, layer=min(1, w.n_layers - 1))
    d = xkv.dims_of(w)
    lm = torch.empty((w.batch, w.n_kv_heads, w.n_chunks, w.head_dim), dtype=torch.bfloat16,
                     device=DEV)
    xkv.xkv_build_landmarks(d, _dev(x["Ak"]), _dev(x["Bkt"]), lm)
    qd = _dev(x["q"])
    scores = torch.empty((w.batch, w.n_kv_heads, w.n_chunks), dtype=torch.float64, device=DEV)
    sel2 = torch.empty((w.batch, w.n_kv_heads, w.n_sel), dtype=torch.int32, device=DEV)
    xkv.xkv_score_landmarks(d, lm, qd, scores)
    xkv.xkv_select_chunks(d, scores, w.top_k, w.n_sink, w.n_recent, sel2)
    fused, _ = _fused(xkv, lm, qd, w.batch, w.n_q_heads, w.n_kv_heads, w.head_dim, w.n_chunks,
                      w.top_k, w.n_sink, w.n_recent, xkv.XKV_BF16)
    lm_g = lm.cpu()
    lm_o = ora.to_torch(ora.build_landmarks(x["Ak"], x["Bkt"], w.n_kv_heads, w.head_dim,
                                            w.chunk))
    # on the GPU's landmarks the selection is the oracle's, bit for bit
    s_g = ora.score_landmarks(lm_g, x["q"])
    assert np.array_equal(scores.cpu().numpy().view(np.uint64), s_g.view(np.uint64))
    ref_g = ora.select_chunks(s_g, w.top_k, w.n_sink, w.n_recent)
    assert np.array_equal(sel2.cpu().numpy(), ref_g)
    assert np.array_equal(fused, ref_g)
    # against the oracle's own landmarks: equal, or different only at certified near-ties
    s_o = ora.score_landmarks(lm_o, x["q"])
    ref_o = ora.select_chunks(s_o, w.top_k, w.n_sink, w.n_recent)
    n_diff = certify(_as_f64(lm_g), _as_f64(lm_o), _as_f64(x["q"]), fused, ref_o, s_o,
                     w.group, w.top_k, w.n_sink, w.n_recent)
    print(f"{w.name}: {n_diff} of {w.batch * w.n_kv_heads} units differ, all certified "
          "near-ties")
