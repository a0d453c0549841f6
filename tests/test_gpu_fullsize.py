"""GPU parity at the workloads' full sizes, in the launch configuration the benchmark
times: the whole layer (every sequence and head) runs on the GPU; the CPU oracle
recomputes sampled (sequence, KV head) units one by one, and properties that hold at any
size are checked everywhere.  Inputs come from the seeded device generator."""
import numpy as np
import pytest
import torch

from cross_layer_compressed_b200 import synth
from parity_util import bf16_ulp_diff, certify_near_ties, compare_outputs

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


def _u16(t):
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def _xkv_layer_check(xkv, ora, w, layer, units, dense=False, reassociated=False):
    d = xkv.dims_of(w)
    c = synth.torch_xkv_layer(w, seed=0, layer=layer, device=DEV)
    q = synth.torch_layer_queries(w, 0, layer, c, device=DEV)
    out = torch.empty((w.batch, w.n_q_heads, w.head_dim), device=DEV)
    hd, G = w.head_dim, w.group
    if dense:
        mode = xkv.XKV_MODE_REASSOC if reassociated else xkv.XKV_MODE_DENSE
        attend = xkv.xkv_reassociated_attend if reassociated else xkv.xkv_reconstruct_attend
        ws = torch.empty(xkv.xkv_workspace_bytes(d, 0, mode), dtype=torch.uint8, device=DEV)
        attend(d, c["Ak"], c["Av"], c["Bkt"], c["Bvt"], q, None, 0, out, ws)
        torch.cuda.synchronize()
        for b, g in units:
            ref = ora.reconstruct_attend(c["Ak"][b:b + 1].cpu(), c["Av"][b:b + 1].cpu(),
                                         c["Bkt"][b:b + 1].cpu(), c["Bvt"][b:b + 1].cpu(),
                                         q[b:b + 1].cpu(), None, w.chunk, units=[(0, g)])
            compare_outputs(out[b, g * G:(g + 1) * G].cpu().numpy(), ref[0, g * G:(g + 1) * G],
                            w.dtype)
        return
    lm = torch.empty((w.batch, w.n_kv_heads, w.n_chunks, hd), dtype=torch.bfloat16, device=DEV)
    xkv.xkv_build_landmarks(d, c["Ak"], c["Bkt"], lm)
    # the product pipeline on the GPU's own landmarks: the fused selection of every unit,
    # which must equal the two-call path (score, select) bit for bit
    sel_f = torch.empty((w.batch, w.n_kv_heads, w.n_sel), dtype=torch.int32, device=DEV)
    wss = torch.empty(xkv.xkv_score_select_workspace_bytes(d), dtype=torch.uint8, device=DEV)
    xkv.xkv_score_select(d, lm, q, w.top_k, w.n_sink, w.n_recent, sel_f, wss)
    sc2 = torch.empty((w.batch, w.n_kv_heads, w.n_chunks), dtype=torch.float64, device=DEV)
    sel2 = torch.empty_like(sel_f)
    xkv.xkv_score_landmarks(d, lm, q, sc2)
    xkv.xkv_select_chunks(d, sc2, w.top_k, w.n_sink, w.n_recent, sel2)
    torch.cuda.synchronize()
    sel_f_h = sel_f.cpu().numpy()
    assert np.array_equal(sel_f_h, sel2.cpu().numpy())
    band = wss[:4 * w.batch * w.n_kv_heads].cpu().view(torch.int32).numpy().view(np.uint32)
    assert np.all(band != 0xFFFFFFFF), "a unit left the fp32 + band path"
    host = {}
    n_diff = 0
    for b, g in units:
        Ak = c["Ak"][b:b + 1].cpu()
        Bkt_g = c["Bkt"][b:b + 1, g * hd:(g + 1) * hd].contiguous().cpu()
        lm_ref = ora.build_landmarks(Ak, Bkt_g, 1, hd, w.chunk)          # oracle landmarks
        diff = bf16_ulp_diff(_u16(lm[b, g]), lm_ref[0, 0])
        assert diff.max() <= 1 and (diff > 0).mean() < 1e-4
        # GPU landmarks against the oracle's: equal selections or certified near-ties
        qg = q[b:b + 1, g * G:(g + 1) * G].cpu()
        s_ref = ora.score_landmarks(ora.to_torch(lm_ref), qg)
        sel_o = ora.select_chunks(s_ref, w.top_k, w.n_sink, w.n_recent)
        n_diff += certify_near_ties(ora.as_float64(lm[b:b + 1, g:g + 1].cpu()),
                                    ora.as_float64(ora.to_torch(lm_ref)), ora.as_float64(qg),
                                    sel_f_h[b:b + 1, g:g + 1], sel_o, s_ref, G, w.top_k,
                                    w.n_sink, w.n_recent)
        lm[b, g] = ora.to_torch(lm_ref)[0, 0].to(DEV)                   # score what the oracle scores
        host[(b, g)] = (Ak, Bkt_g, lm_ref)
    print(f"{w.name}: {n_diff} of {len(units)} sampled units select differently from GPU "
          "landmarks, all certified near-ties")
    scores = torch.empty((w.batch, w.n_kv_heads, w.n_chunks), dtype=torch.float64, device=DEV)
    sel = torch.empty((w.batch, w.n_kv_heads, w.n_sel), dtype=torch.int32, device=DEV)
    mode = xkv.XKV_MODE_REASSOC if reassociated else xkv.XKV_MODE_SELECTIVE
    attend = xkv.xkv_reassociated_attend if reassociated else xkv.xkv_reconstruct_attend
    ws = torch.empty(xkv.xkv_workspace_bytes(d, w.n_sel, mode), dtype=torch.uint8, device=DEV)
    xkv.xkv_score_landmarks(d, lm, q, scores)
    xkv.xkv_select_chunks(d, scores, w.top_k, w.n_sink, w.n_recent, sel)
    attend(d, c["Ak"], c["Av"], c["Bkt"], c["Bvt"], q, sel, w.n_sel, out, ws)
    torch.cuda.synchronize()
    sel_h = sel.cpu().numpy()
    # properties of every unit: ascending, in range, forced chunks present, needles kept
    assert np.all(np.diff(sel_h, axis=2) > 0)
    assert sel_h.min() >= 0 and sel_h.max() < w.n_chunks
    forced = synth.forced_chunks(w.n_chunks, w.n_sink, w.n_recent)
    assert all(set(forced) <= set(row.tolist()) for row in sel_h.reshape(-1, w.n_sel))
    sc_h = scores.cpu().numpy()
    missing = []
    for b, nd in enumerate(synth.torch_needle_chunks(w, 0)):
        for g in range(w.n_kv_heads):
            for n in set(nd.tolist()) - set(sel_h[b, g].tolist()):
                rank = int((sc_h[b, g] > sc_h[b, g, n]).sum())
                missing.append((b, g, n, rank))
    assert not missing, f"needle chunks not selected (b, g, chunk, score rank): {missing[:8]}"
    # sampled units against the oracle
    for (b, g), (Ak, Bkt_g, lm_ref) in host.items():
        qg = q[b:b + 1, g * G:(g + 1) * G].cpu()
        s_ref = ora.score_landmarks(ora.to_torch(lm_ref), qg)
        got_s = scores[b, g].cpu().numpy()
        assert np.array_equal(got_s.view(np.uint64), s_ref[0, 0].view(np.uint64))
        sel_ref = ora.select_chunks(s_ref, w.top_k, w.n_sink, w.n_recent)
        assert np.array_equal(sel_h[b, g], sel_ref[0, 0])
        ref = ora.reconstruct_attend(c["Ak"][b:b + 1].cpu(), c["Av"][b:b + 1].cpu(),
                                     c["Bkt"][b:b + 1].cpu(), c["Bvt"][b:b + 1].cpu(),
                                     q[b:b + 1].cpu(), sel_h[b:b + 1], w.chunk, units=[(0, g)])
        compare_outputs(out[b, g * G:(g + 1) * G].cpu().numpy(), ref[0, g * G:(g + 1) * G],
                        w.dtype)


def test_llama8b_selective_32k_full_layer(xkv, ora):
    w = synth.LLAMA8B_SR_32K
    _xkv_layer_check(xkv, ora, w, layer=5, units=[(3, 5), (7, 0)])
    torch.cuda.empty_cache()


def test_qwen14b_selective_16k_full_layer(xkv, ora):
    w = synth.QWEN14B_SR_16K
    _xkv_layer_check(xkv, ora, w, layer=9, units=[(0, 7), (63, 2)])
    torch.cuda.empty_cache()


def test_llama8b_selective_32k_full_layer_reassociated(xkv, ora):
    """The rank-space entry point on the same full-size layer and sampled units."""
    w = synth.LLAMA8B_SR_32K
    _xkv_layer_check(xkv, ora, w, layer=5, units=[(3, 5), (7, 0)], reassociated=True)
    torch.cuda.empty_cache()


def test_qwen14b_selective_16k_full_layer_reassociated(xkv, ora):
    w = synth.QWEN14B_SR_16K
    _xkv_layer_check(xkv, ora, w, layer=9, units=[(0, 7), (63, 2)], reassociated=True)
    torch.cuda.empty_cache()


def test_llama8b_dense_128k_full_layer(xkv, ora):
    w = synth.LLAMA8B_DENSE_128K
    _xkv_layer_check(xkv, ora, w, layer=2, units=[(0, 3)], dense=True)
    torch.cuda.empty_cache()


def test_llama8b_dense_128k_full_layer_reassociated(xkv, ora):
    """The head-batched rank-space kernel on the full 128K window: 147 spans of 7 tiles."""
    w = synth.LLAMA8B_DENSE_128K
    _xkv_layer_check(xkv, ora, w, layer=2, units=[(0, 0), (0, 6)], dense=True,
                     reassociated=True)
    torch.cuda.empty_cache()


def test_qwen3_rcla_32k_full_step(xkv, ora):
    """One decode step of all 36 layers (9 leaders append, every layer attends) at full
    size; sampled units of a leader, its follower and the last layer against the oracle."""
    w = synth.QWEN3_8B_RCLA_32K
    c = synth.torch_rcla_cache(w, seed=0, device=DEV)
    q = synth.torch_queries(w, 0, None, device=DEV)[0]                   # [N][B][Hq][hd]
    S = synth.leader_set(w)
    lo = [max(s for s in S if s <= l) for l in range(w.n_layers)]
    length = w.ctx_len
    samples = {4: (5, 2), 5: (5, 2), 35: (11, 7)}                       # layer -> (b, g)
    G = w.group
    before = {}
    for layer, (b, g) in samples.items():
        slot = S.index(lo[layer])
        before[layer] = (_u16(c["K_lead"][slot:slot + 1, b:b + 1, g:g + 1]).copy(),
                         _u16(c["V_lead"][slot:slot + 1, b:b + 1, g:g + 1]).copy())
    d = xkv.dims(w.batch, w.n_q_heads, w.n_kv_heads, w.head_dim, w.L_max, dtype=w.dtype)
    ws = torch.empty(xkv.xkv_workspace_bytes(d, 0, xkv.XKV_MODE_RCLA), dtype=torch.uint8,
                     device=DEV)
    outs = torch.empty((w.n_layers, w.batch, w.n_q_heads, w.head_dim), device=DEV)
    for layer in range(w.n_layers):
        leader = lo[layer] == layer
        si = S.index(lo[layer])
        xkv.rcla_decode_attend(d, layer, lo, c["K_lead"], c["V_lead"], w.L_max,
                               length if leader else length + 1,
                               c["k_new"][0, si] if leader else None,
                               c["v_new"][0, si] if leader else None, q[layer], outs[layer], ws)
    torch.cuda.synchronize()
    for layer, (b, g) in samples.items():
        slot = S.index(lo[layer])
        K0, V0 = before[layer]
        kn = c["k_new"][0, slot, b:b + 1, g:g + 1].cpu()
        vn = c["v_new"][0, slot, b:b + 1, g:g + 1].cpu()
        qg = q[layer, b:b + 1, g * G:(g + 1) * G].cpu()
        if lo[layer] == layer:       # the leader appends, then attends len + 1 rows
            ref = ora.rcla_decode_attend(0, [0], K0, V0, length, kn, vn, qg)
            assert np.array_equal(_u16(c["K_lead"][slot, b, g, length]), _u16(kn[0, 0]))
        else:                        # a follower sees its leader's appended row
            K0[0, 0, 0, length] = _u16(kn[0, 0])
            V0[0, 0, 0, length] = _u16(vn[0, 0])
            ref = ora.rcla_decode_attend(1, [0, 0], K0, V0, length + 1, None, None, qg)
        compare_outputs(outs[layer, b, g * G:(g + 1) * G].cpu().numpy(), ref[0], w.dtype)
    del c
    torch.cuda.empty_cache()
