"""The device-side timeout paths, exercised without faulting anything: a test-only variable
sets the poll limit of one kernel's pipeline waits to 0, so that they give up at once (a
single poll can succeed: mbarrier try_wait may suspend until the data lands); every other
wait (and the drain of the copies and MMAs in flight) keeps its full bound.

* The tensor-core attention kernels (explicit, rank-space selective, rank-space dense)
  must report XKV_ERR_TIMEOUT in the status word and NaN outputs, and the next call, with
  the normal limit, must be clean.
* The R-CLA kernels (tensor-core, and TMA + CUDA-core) poison the partials of the items
  they gave up on, so the outputs are NaN; the next call must match the oracle.
* The factorization's tcgen05 products report XKV_ERR_TIMEOUT in the workspace status
  word and leave NaN factors; the next call must match the oracle's truncated SVD.
* The fused selection's key pass must send the units it covers to the exact fp64 path:
  the selection stays the oracle's, and the next call takes the fp32 path again."""
import dataclasses

import numpy as np
import pytest
import torch

from cross_layer_compressed_b200 import synth
from parity_util import compare_outputs

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


def test_attention_wait_timeout_is_reported_then_the_next_call_is_clean(xkv, ora, monkeypatch):
    w = synth.reduced(synth.LLAMA8B_SR_32K, batch=2, ctx_len=4096, top_k=60, n_needles=0)
    x = synth.np_xkv_layer_inputs(w, seed=5, layer=0)
    g = {k: x[k].to(DEV) for k in ("Ak", "Av", "Bkt", "Bvt", "q")}
    rng = np.random.default_rng(5)
    sel = np.stack([np.sort(rng.choice(w.n_chunks, w.n_sel, replace=False))
                    for _ in range(w.batch * w.n_kv_heads)]).reshape(
        w.batch, w.n_kv_heads, w.n_sel).astype(np.int32)
    sel_d = torch.from_numpy(sel).to(DEV)
    d = xkv.dims_of(w)
    ws = torch.zeros(xkv.xkv_workspace_bytes(d, w.n_sel, xkv.XKV_MODE_SELECTIVE),
                     dtype=torch.uint8, device=DEV)
    out = torch.empty((w.batch, w.n_q_heads, w.head_dim), device=DEV)

    def call():
        xkv.xkv_reconstruct_attend(d, g["Ak"], g["Av"], g["Bkt"], g["Bvt"], g["q"], sel_d,
                                   w.n_sel, out, ws)
        torch.cuda.synchronize()
        return int(ws[:4].cpu().view(torch.int32).item()), out.cpu().numpy()

    monkeypatch.setenv("XKV_TEST_MMA_SPIN", "0")
    status, o = call()
    assert status & (1 << xkv.XKV_ERR_TIMEOUT), status
    assert np.all(np.isnan(o))
    monkeypatch.delenv("XKV_TEST_MMA_SPIN")
    status, o = call()
    assert status == 0
    ref = ora.reconstruct_attend(x["Ak"], x["Av"], x["Bkt"], x["Bvt"], x["q"], sel, w.chunk,
                                 units=[(0, 1), (1, 6)])
    for b, gg in ((0, 1), (1, 6)):
        G = w.group
        compare_outputs(o[b, gg * G:(gg + 1) * G], ref[b, gg * G:(gg + 1) * G], w.dtype)


def test_selection_key_pass_timeout_falls_back_to_the_exact_path(xkv, ora, monkeypatch):
    w = synth.reduced(synth.LLAMA8B_SR_32K, batch=2, ctx_len=8192, top_k=64)
    x = synth.np_xkv_layer_inputs(w, seed=3, layer=1)
    lm = ora.to_torch(ora.build_landmarks(x["Ak"], x["Bkt"], w.n_kv_heads, w.head_dim, w.chunk))
    ref = ora.select_chunks(ora.score_landmarks(lm, x["q"]), w.top_k, w.n_sink, w.n_recent)
    d = xkv.dims_of(w)
    lm_d, q_d = lm.to(DEV), x["q"].to(DEV)
    ws = torch.zeros(xkv.xkv_score_select_workspace_bytes(d), dtype=torch.uint8, device=DEV)
    sel = torch.full((w.batch, w.n_kv_heads, w.n_sel), -7, dtype=torch.int32, device=DEV)

    def call():
        xkv.xkv_score_select(d, lm_d, q_d, w.top_k, w.n_sink, w.n_recent, sel, ws)
        torch.cuda.synchronize()
        band = ws[:4 * w.batch * w.n_kv_heads].cpu().view(torch.int32).numpy().view(np.uint32)
        return sel.cpu().numpy(), band

    monkeypatch.setenv("XKV_TEST_SS_SPIN", "0")
    got, band = call()
    assert np.all(band == 0xFFFFFFFF), band          # every unit on the exact path
    assert np.array_equal(got, ref)
    monkeypatch.delenv("XKV_TEST_SS_SPIN")
    got, band = call()
    assert np.all(band != 0xFFFFFFFF), band
    assert np.array_equal(got, ref)


def _rank_space_timeout_then_clean(xkv, ora, monkeypatch, w, sel, units):
    x = synth.np_xkv_layer_inputs(w, seed=7, layer=0)
    g = {k: x[k].to(DEV) for k in ("Ak", "Av", "Bkt", "Bvt", "q")}
    d = xkv.dims_of(w)
    n_sel = 0 if sel is None else sel.shape[2]
    sel_d = None if sel is None else torch.from_numpy(sel).to(DEV)
    ws = torch.zeros(xkv.xkv_workspace_bytes(d, n_sel, xkv.XKV_MODE_REASSOC), dtype=torch.uint8,
                     device=DEV)
    out = torch.empty((w.batch, w.n_q_heads, w.head_dim), device=DEV)

    def call():
        xkv.xkv_reassociated_attend(d, g["Ak"], g["Av"], g["Bkt"], g["Bvt"], g["q"], sel_d, n_sel,
                                    out, ws)
        torch.cuda.synchronize()
        return int(ws[:4].cpu().view(torch.int32).item()), out.cpu().numpy()

    monkeypatch.setenv("XKV_TEST_MMA_SPIN", "0")
    status, o = call()
    assert status & (1 << xkv.XKV_ERR_TIMEOUT), status
    assert np.all(np.isnan(o))
    monkeypatch.delenv("XKV_TEST_MMA_SPIN")
    status, o = call()
    assert status == 0
    ref = ora.reconstruct_attend(x["Ak"], x["Av"], x["Bkt"], x["Bvt"], x["q"], sel, w.chunk,
                                 units=units)
    G = w.group
    for b, gg in units:
        compare_outputs(o[b, gg * G:(gg + 1) * G], ref[b, gg * G:(gg + 1) * G], w.dtype)


def test_rank_space_selective_wait_timeout_is_reported_then_the_next_call_is_clean(
        xkv, ora, monkeypatch):
    """Selective rank-space kernel: the split merge and projection kernels see the status
    word and write NaN."""
    w = synth.reduced(synth.LLAMA8B_SR_32K, batch=2, ctx_len=4096, top_k=60, n_needles=0)
    rng = np.random.default_rng(11)
    sel = np.stack([np.sort(rng.choice(w.n_chunks, w.n_sel, replace=False))
                    for _ in range(w.batch * w.n_kv_heads)]).reshape(
        w.batch, w.n_kv_heads, w.n_sel).astype(np.int32)
    _rank_space_timeout_then_clean(xkv, ora, monkeypatch, w, sel, [(0, 2), (1, 7)])


def test_rank_space_dense_wait_timeout_is_reported_then_the_next_call_is_clean(
        xkv, ora, monkeypatch):
    """Head-batched dense kernel with 64 spans per sequence, so the merge + projection
    kernel is the one that turns the status word into NaN outputs."""
    w = dataclasses.replace(synth.reduced(synth.LLAMA8B_DENSE_128K, batch=1, ctx_len=8192),
                            n_q_heads=8, n_kv_heads=8, rank_k=256, rank_v=384, name="dense_g1")
    _rank_space_timeout_then_clean(xkv, ora, monkeypatch, w, None, [(0, 0), (0, 5)])


@pytest.mark.parametrize("switch", [None, "XKV_NO_TC"], ids=["tensor_core", "tma"])
def test_rcla_wait_timeout_gives_nan_then_the_next_call_is_clean(xkv, ora, monkeypatch, switch):
    """A follower layer (no append, so both calls attend the same rows) over 20000 rows,
    many items: every CTA gives up on its first item and poisons the items it owed."""
    if switch:
        monkeypatch.setenv(switch, "1")
    length = 20000
    w = dataclasses.replace(
        synth.reduced(synth.QWEN3_8B_RCLA_32K, batch=1, ctx_len=length, n_layers=2,
                      extra_rows=2, outlier_frac=0.0),
        n_kv_heads=2, n_q_heads=8, name="rcla_timeout")
    x = synth.np_rcla_inputs(w, seed=9, len_rows=length)
    lo = ora.leader_map([0], 2)
    K_ref = x["K_lead"].view(torch.int16).numpy().view(np.uint16).copy()
    V_ref = x["V_lead"].view(torch.int16).numpy().view(np.uint16).copy()
    ref = ora.rcla_decode_attend(1, lo, K_ref, V_ref, length, None, None, x["q"][1])
    d = xkv.dims(w.batch, w.n_q_heads, w.n_kv_heads, w.head_dim, w.L_max, dtype=w.dtype)
    ws = torch.empty(xkv.xkv_workspace_bytes(d, 0, xkv.XKV_MODE_RCLA), dtype=torch.uint8,
                     device=DEV)
    K, V, q = x["K_lead"].to(DEV), x["V_lead"].to(DEV), x["q"][1].to(DEV)
    out = torch.empty((w.batch, w.n_q_heads, w.head_dim), device=DEV)

    def call():
        xkv.rcla_decode_attend(d, 1, lo, K, V, w.L_max, length, None, None, q, out, ws)
        torch.cuda.synchronize()
        return out.cpu().numpy()

    monkeypatch.setenv("XKV_TEST_MMA_SPIN", "0")
    assert np.all(np.isnan(call()))
    monkeypatch.delenv("XKV_TEST_MMA_SPIN")
    compare_outputs(call(), ref, w.dtype)


def test_factorization_product_timeout_is_reported_then_the_next_call_is_clean(
        xkv, ora, monkeypatch):
    W, B, L, Hkv, hd, r = 2, 2, 1000, 2, 64, 32
    X, s = synth.np_window_caches(W, B, L, Hkv * hd, 96, r, 16.0, 0.05, 0)
    Xs = synth.to_storage(X, "bf16")
    d = xkv.dims(B, Hkv, Hkv, hd, L, chunk=8, rank_k=0, rank_v=0, dtype="bf16")
    A = torch.empty((B, L, r), dtype=torch.bfloat16, device=DEV)
    Bt = torch.empty((W, B, Hkv * hd, r), dtype=torch.bfloat16, device=DEV)
    ws = torch.empty(xkv.xkv_factorize_workspace_bytes(d, W, r), dtype=torch.uint8, device=DEV)
    om = torch.from_numpy(synth.np_test_matrix(W * Hkv * hd, r, 0)).to(DEV)
    Xd = Xs.to(DEV)

    def call():
        xkv.xkv_factorize_window(d, W, r, Xd, om, 3, A, Bt, ws)
        torch.cuda.synchronize()
        return (int(ws[:4].cpu().view(torch.int32).item()), A.double().cpu().numpy(),
                Bt.double().cpu().numpy())

    monkeypatch.setenv("XKV_TEST_MMA_SPIN", "0")
    status, A0, Bt0 = call()
    assert status & (1 << xkv.XKV_ERR_TIMEOUT), status
    assert np.all(np.isnan(A0)) and np.all(np.isnan(Bt0))
    monkeypatch.delenv("XKV_TEST_MMA_SPIN")
    status, A1, Bt1 = call()
    assert status == 0
    A_ref, Bt_ref, _ = ora.factorize_window(Xs.double().numpy(), r)
    P_ref = ora.reconstruct_window(A_ref, Bt_ref)
    err = np.abs(ora.reconstruct_window(A1, Bt1) - P_ref).max() / np.abs(P_ref).max()
    assert err <= 2e-2, err
