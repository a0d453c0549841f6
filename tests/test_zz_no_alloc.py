"""The allocation-free reconstruct+attend entry point, for callers that cannot call
cudaMalloc (engine plugin hooks with no workspace, HBM reserved by a serving engine's KV
pool, paths that may not synchronise the device).  It must give the same results as the
workspace entry point, call after call, although every call reuses one fixed scratch
array inside the library.  This file is collected last on purpose."""
import numpy as np
import pytest
import torch

from cross_layer_compressed_b200 import synth
from parity_util import compare_outputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def xkv():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from cross_layer_compressed_b200 import build
    build.build()
    from cross_layer_compressed_b200 import xkv as m
    return m


def _inputs(w, seed, dev):
    x = synth.np_xkv_layer_inputs(w, seed=seed, layer=0)
    g = {k: x[k].to(dev) for k in ("Ak", "Av", "Bkt", "Bvt", "q")}
    rng = np.random.default_rng(seed)
    sel = np.stack([np.sort(rng.choice(w.n_chunks, w.n_sel, replace=False))
                    for _ in range(w.batch * w.n_kv_heads)]).reshape(
        w.batch, w.n_kv_heads, w.n_sel).astype(np.int32)
    g["sel"] = torch.from_numpy(sel).to(dev)
    return g


@pytest.mark.parametrize("w", [
    synth.reduced(synth.LLAMA8B_SR_32K, batch=2, ctx_len=4096, top_k=40, n_needles=0),
    synth.reduced(synth.TINY_SR_F32, ctx_len=2048, top_k=30)], ids=lambda w: w.name)
def test_noalloc_matches_workspace_entry_point_twice(xkv, w):
    dev = torch.device("cuda:0")
    d = xkv.dims_of(w)
    for seed in (1, 2):                      # two calls in a row, different inputs
        g = _inputs(w, seed, dev)
        ws = torch.empty(xkv.xkv_workspace_bytes(d, w.n_sel, xkv.XKV_MODE_SELECTIVE),
                         dtype=torch.uint8, device=dev)
        ref = torch.empty((w.batch, w.n_q_heads, w.head_dim), device=dev)
        xkv.xkv_reconstruct_attend(d, g["Ak"], g["Av"], g["Bkt"], g["Bvt"], g["q"], g["sel"],
                                   w.n_sel, ref, ws)
        out = torch.full_like(ref, float("nan"))
        xkv.xkv_reconstruct_attend_noalloc(d, g["Ak"], g["Av"], g["Bkt"], g["Bvt"], g["q"],
                                           g["sel"], w.n_sel, out)
        torch.cuda.synchronize()
        compare_outputs(out.cpu().numpy(), ref.cpu().numpy(), w.dtype)


def test_noalloc_dense_and_size_limit(xkv):
    dev = torch.device("cuda:0")
    w = synth.reduced(synth.LLAMA8B_DENSE_128K, batch=1, ctx_len=2048)
    d = xkv.dims_of(w)
    g = _inputs(dataclass_with_sel(w), 3, dev)
    ws = torch.empty(xkv.xkv_workspace_bytes(d, 0, xkv.XKV_MODE_DENSE), dtype=torch.uint8,
                     device=dev)
    ref = torch.empty((w.batch, w.n_q_heads, w.head_dim), device=dev)
    xkv.xkv_reconstruct_attend(d, g["Ak"], g["Av"], g["Bkt"], g["Bvt"], g["q"], None, 0, ref, ws)
    out = torch.empty_like(ref)
    xkv.xkv_reconstruct_attend_noalloc(d, g["Ak"], g["Av"], g["Bkt"], g["Bvt"], g["q"], None, 0,
                                       out)
    torch.cuda.synchronize()
    compare_outputs(out.cpu().numpy(), ref.cpu().numpy(), w.dtype)
    # a call whose scratch would exceed the fixed array is refused before any launch
    big = xkv.dims(64, 512, 32, 128, 1 << 20, 8, 512, 768, xkv.XKV_BF16)
    st = xkv.xkv_reconstruct_attend_noalloc(big, g["Ak"], g["Av"], g["Bkt"], g["Bvt"], g["q"],
                                            None, 0, out, check=False)
    assert st == xkv.XKV_ERR_UNSUPPORTED
    assert "scratch" in xkv.last_error()


def dataclass_with_sel(w):
    import dataclasses
    return dataclasses.replace(w, top_k=8, n_sink=1, n_recent=1)
