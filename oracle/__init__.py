"""CPU oracle for decode attention over a cross-layer-compressed KV cache.

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the benchmark's
CPU-baseline leg may use it; the library itself never does.  The arithmetic lives in
``xkv_oracle.c`` (plain scalar C, fp64); this module compiles it with gcc and passes
buffers to it.  Inputs are torch CPU tensors (fp32 or bf16) or numpy arrays.  The
cross-layer factorization of a window (``clf.py``) is numpy fp64 around LAPACK's SVD.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "xkv_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None

F32, BF16 = 0, 1

from .clf import (concatenate_window, factorize_window, reconstruct_window,  # noqa: E402,F401
                  refold_window)


def build(force: bool = False) -> str:
    """Compile the oracle (no fused multiply-add contraction, no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math",
                               "-fPIC", "-shared", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def lib():
    global _lib
    if _lib is None:
        L = ctypes.CDLL(build())
        i32, i64, vp, dp = ctypes.c_int, ctypes.c_int64, ctypes.c_void_p, ctypes.c_double
        L.oracle_round_bf16.argtypes = [dp]
        L.oracle_round_bf16.restype = ctypes.c_uint16
        L.oracle_reconstruct_rows.argtypes = [i32, i32, i32, vp, vp, i64, i64, vp]
        L.oracle_build_landmarks.argtypes = [i32, i32, i32, i64, i32, i32, i32, vp, vp, vp]
        L.oracle_score_landmarks.argtypes = [i32, i32, i32, i32, i64, i32, vp, vp, vp]
        L.oracle_n_selected.argtypes = [i64, i32, i32, i32]
        L.oracle_n_selected.restype = i64
        L.oracle_select_chunks.argtypes = [i32, i32, i64, vp, i32, i32, i32, vp, vp]
        L.oracle_value_ranges.argtypes = [i32, i32, i32, i64, i32, i32, i32, vp, vp, vp]
        L.oracle_n_reserved.argtypes = [i64, i32, i32, i32]
        L.oracle_n_reserved.restype = i64
        L.oracle_reserve_value_chunks.argtypes = [i32, i32, i64, vp, i32, i32, i32, vp, vp]
        L.oracle_select_chunks_reserved.argtypes = [i32, i32, i64, vp, vp, i32, i32, i32, i32,
                                                    vp, vp]
        L.oracle_attend_unit.argtypes = [i32, i32, i32, i32, i32, i32, i64, i32, i32, i32,
                                         i32, vp, vp, vp, vp, vp, vp, i64, vp]
        L.oracle_reconstruct_attend.argtypes = [i32, i32, i32, i32, i64, i32, i32, i32, i32,
                                                vp, vp, vp, vp, vp, vp, i64, vp]
        L.oracle_attend_unit_tail.argtypes = [i32, i32, i32, i32, i32, i32, i64, i32, i32,
                                              i32, i32, vp, vp, vp, vp, vp, vp, i64, vp, vp,
                                              i64, i64, vp]
        L.oracle_leader_map.argtypes = [vp, i32, i32, vp]
        L.oracle_rcla_decode_attend.argtypes = [i32, i32, i32, i32, i32, i32, vp, i32, vp, vp,
                                                i64, i64, vp, vp, vp, vp]
        L.oracle_footprint_bytes.argtypes = [i32, i32, i32, i64, i32, i32, i32, i32, i32, i32,
                                             i32]
        L.oracle_footprint_bytes.restype = i64
        L.oracle_rcla_cache_bytes.argtypes = [i32, i32, i32, i64, i32, i32]
        L.oracle_rcla_cache_bytes.restype = i64
        _lib = L
    return _lib


# ------------------------------------------------------------------ buffer helpers
def _buf(x):
    """(numpy array owning host memory, storage dtype code) for a torch or numpy input."""
    try:
        import torch
        if isinstance(x, torch.Tensor):
            x = x.detach().cpu().contiguous()
            if x.dtype == torch.bfloat16:
                return x.view(torch.int16).numpy().view(np.uint16), BF16
            if x.dtype == torch.float32:
                return x.numpy(), F32
            raise TypeError(f"unsupported dtype {x.dtype}")
    except ImportError:
        pass
    x = np.ascontiguousarray(x)
    if x.dtype == np.uint16:
        return x, BF16
    if x.dtype == np.float32:
        return x, F32
    raise TypeError(f"unsupported dtype {x.dtype}")


def _p(a: np.ndarray):
    return ctypes.c_void_p(a.ctypes.data) if a is not None else None


def _check(rc, what):
    if rc != 0:
        raise ValueError(f"oracle {what} rejected its arguments (rc={rc})")


def _bf16_to_np_f32(u16: np.ndarray) -> np.ndarray:
    return (u16.astype(np.uint32) << 16).view(np.float32)


def as_float64(x) -> np.ndarray:
    """Exact widening of a storage-dtype tensor to fp64 (for tests)."""
    a, dt = _buf(x)
    return (_bf16_to_np_f32(a) if dt == BF16 else a).astype(np.float64)


# ------------------------------------------------------------------------ the calls
def round_bf16(x: float) -> int:
    return int(lib().oracle_round_bf16(float(x)))


def reconstruct_rows(A, Bt, t0: int, n: int) -> np.ndarray:
    """fp64 rows [t0, t0+n) of A * B (A one sequence's L x r basis, Bt = B^T, d_kv x r)."""
    a, dt = _buf(A)
    bt, dt2 = _buf(Bt)
    assert dt == dt2
    d_kv, r = bt.shape
    out = np.empty((n, d_kv), dtype=np.float64)
    _check(lib().oracle_reconstruct_rows(d_kv, r, dt, _p(a), _p(bt), t0, n, _p(out)),
           "reconstruct_rows")
    return out


def build_landmarks(Ak, Bkt, n_kv_heads: int, head_dim: int, chunk: int):
    """lm [B][Hkv][nC][hd] in the storage dtype (returned as a numpy array of that dtype)."""
    a, dt = _buf(Ak)
    bt, _ = _buf(Bkt)
    B, L, rk = a.shape
    nC = L // chunk
    lm = np.empty((B, n_kv_heads, nC, head_dim), dtype=np.float32 if dt == F32 else np.uint16)
    _check(lib().oracle_build_landmarks(B, n_kv_heads, head_dim, L, chunk, rk, dt, _p(a), _p(bt),
                                        _p(lm)), "build_landmarks")
    return lm


def to_torch(x: np.ndarray):
    """numpy storage array (float32 or uint16 bf16 bits) -> torch CPU tensor."""
    import torch
    if x.dtype == np.uint16:
        return torch.from_numpy(x.view(np.int16).copy()).view(torch.bfloat16)
    return torch.from_numpy(x.copy())


def score_landmarks(lm, q) -> np.ndarray:
    l, dt = _buf(lm)
    qq, dt2 = _buf(q)
    assert dt == dt2
    B, Hkv, nC, hd = l.shape
    Hq = qq.shape[1]
    s = np.empty((B, Hkv, nC), dtype=np.float64)
    _check(lib().oracle_score_landmarks(B, Hq, Hkv, hd, nC, dt, _p(l), _p(qq), _p(s)),
           "score_landmarks")
    return s


def n_selected(n_chunks: int, top_k: int, n_sink: int, n_recent: int) -> int:
    return int(lib().oracle_n_selected(n_chunks, top_k, n_sink, n_recent))


def select_chunks(scores: np.ndarray, top_k: int, n_sink: int, n_recent: int) -> np.ndarray:
    s = np.ascontiguousarray(scores, dtype=np.float64)
    B, Hkv, nC = s.shape
    n_sel = n_selected(nC, top_k, n_sink, n_recent)
    sel = np.empty((B, Hkv, max(n_sel, 0)), dtype=np.int32)
    ns = ctypes.c_int64(0)
    _check(lib().oracle_select_chunks(B, Hkv, nC, _p(s), top_k, n_sink, n_recent, _p(sel),
                                      ctypes.byref(ns)), "select_chunks")
    return sel


def value_ranges(Av, Bvt, n_kv_heads: int, head_dim: int, chunk: int) -> np.ndarray:
    """rho [B][Hkv][nC] fp64: per chunk, the largest max - min of a reconstructed value row
    (one KV head's slice) among the chunk's rows."""
    a, dt = _buf(Av)
    bt, dt2 = _buf(Bvt)
    assert dt == dt2
    B, L, rv = a.shape
    rho = np.empty((B, n_kv_heads, L // chunk), dtype=np.float64)
    _check(lib().oracle_value_ranges(B, n_kv_heads, head_dim, L, chunk, rv, dt, _p(a), _p(bt),
                                     _p(rho)), "value_ranges")
    return rho


def n_reserved(n_chunks: int, n_value: int, n_sink: int, n_recent: int) -> int:
    return int(lib().oracle_n_reserved(n_chunks, n_value, n_sink, n_recent))


def reserve_value_chunks(rho: np.ndarray, n_value: int, n_sink: int, n_recent: int):
    """reserved [B][Hkv][n_res] int32: the n_res candidates of largest rho, ascending."""
    r = np.ascontiguousarray(rho, dtype=np.float64)
    B, Hkv, nC = r.shape
    n_res = n_reserved(nC, n_value, n_sink, n_recent)
    out = np.empty((B, Hkv, max(n_res, 0)), dtype=np.int32)
    _check(lib().oracle_reserve_value_chunks(B, Hkv, nC, _p(r), n_value, n_sink, n_recent,
                                             _p(out), None), "reserve_value_chunks")
    return out


def select_chunks_reserved(scores: np.ndarray, reserved: np.ndarray, top_k: int, n_sink: int,
                           n_recent: int) -> np.ndarray:
    """Selection whose forced chunks also include reserved [B][Hkv][n_res]."""
    s = np.ascontiguousarray(scores, dtype=np.float64)
    B, Hkv, nC = s.shape
    res = np.ascontiguousarray(reserved, dtype=np.int32)
    n_res = res.shape[2]
    rest = nC - n_selected(nC, 0, n_sink, n_recent) - n_res
    n_sel = n_selected(nC, 0, n_sink, n_recent) + n_res + min(top_k, rest)
    sel = np.empty((B, Hkv, n_sel), dtype=np.int32)
    _check(lib().oracle_select_chunks_reserved(B, Hkv, nC, _p(s), _p(res) if n_res else None,
                                               n_res, top_k, n_sink, n_recent, _p(sel), None),
           "select_chunks_reserved")
    return sel


def reconstruct_attend(Ak, Av, Bkt, Bvt, q, sel, chunk: int, units=None) -> np.ndarray:
    """out [B][Hq][hd] fp32.  sel [B][Hkv][n_sel] int32 or None (dense).  `units`, if
    given, is a list of (b, g) pairs to compute; other outputs are left as NaN."""
    ak, dt = _buf(Ak)
    av, _ = _buf(Av)
    bk, _ = _buf(Bkt)
    bv, _ = _buf(Bvt)
    qq, _ = _buf(q)
    B, L, rk = ak.shape
    rv = av.shape[2]
    d_kv = bk.shape[1]
    _, Hq, hd = qq.shape
    Hkv = d_kv // hd
    out = np.full((B, Hq, hd), np.nan, dtype=np.float32)
    if sel is not None:
        sel = np.ascontiguousarray(sel, dtype=np.int32)
        n_sel = sel.shape[2]
    else:
        n_sel = 0
    if units is None:
        _check(lib().oracle_reconstruct_attend(B, Hq, Hkv, hd, L, chunk, rk, rv, dt, _p(ak), _p(av),
                                               _p(bk), _p(bv), _p(qq),
                                               _p(sel) if sel is not None else None, n_sel,
                                               _p(out)), "reconstruct_attend")
    else:
        for b, g in units:
            sp = None
            if sel is not None:
                sp = ctypes.c_void_p(sel.ctypes.data + ((b * Hkv + g) * n_sel) * 4)
            _check(lib().oracle_attend_unit(b, g, B, Hq, Hkv, hd, L, chunk, rk, rv, dt, _p(ak),
                                            _p(av), _p(bk), _p(bv), _p(qq), sp, n_sel, _p(out)),
                   "attend_unit")
    return out


def reconstruct_attend_tail(Ak, Av, Bkt, Bvt, q, sel, chunk: int, K_tail, V_tail,
                            n_tail: int, units=None) -> np.ndarray:
    """out [B][Hq][hd] fp32: attention over the reconstructed selected rows (all rows when
    sel is None) followed by the first n_tail rows of K_tail / V_tail [B][Hkv][T_max][hd]
    (storage type of the factors).  `units` as for reconstruct_attend."""
    ak, dt = _buf(Ak)
    av, _ = _buf(Av)
    bk, _ = _buf(Bkt)
    bv, _ = _buf(Bvt)
    qq, _ = _buf(q)
    kt, _ = _buf(K_tail)
    vt, _ = _buf(V_tail)
    B, L, rk = ak.shape
    rv = av.shape[2]
    d_kv = bk.shape[1]
    _, Hq, hd = qq.shape
    Hkv = d_kv // hd
    T_max = kt.shape[2]
    out = np.full((B, Hq, hd), np.nan, dtype=np.float32)
    n_sel = 0
    if sel is not None:
        sel = np.ascontiguousarray(sel, dtype=np.int32)
        n_sel = sel.shape[2]
    for b, g in (units if units is not None else [(b, g) for b in range(B) for g in range(Hkv)]):
        sp = None
        if sel is not None:
            sp = ctypes.c_void_p(sel.ctypes.data + ((b * Hkv + g) * n_sel) * 4)
        _check(lib().oracle_attend_unit_tail(b, g, B, Hq, Hkv, hd, L, chunk, rk, rv, dt,
                                             _p(ak), _p(av), _p(bk), _p(bv), _p(qq), sp,
                                             n_sel, _p(kt), _p(vt), T_max, int(n_tail),
                                             _p(out)), "attend_unit_tail")
    return out


def leader_map(S, n_layers: int) -> np.ndarray:
    s = np.ascontiguousarray(S, dtype=np.int32)
    out = np.empty(n_layers, dtype=np.int32)
    _check(lib().oracle_leader_map(_p(s), len(s), n_layers, _p(out)), "leader_map")
    return out


def rcla_decode_attend(layer: int, leader_of, K_lead: np.ndarray, V_lead: np.ndarray,
                       length: int, k_new, v_new, q) -> np.ndarray:
    """R-CLA decode attention of one layer.  K_lead / V_lead are numpy storage arrays
    [n_lead][B][Hkv][L_max][hd] and are UPDATED in place when the layer is a leader
    given a new row.  Returns out [B][Hq][hd] fp32."""
    lo = np.ascontiguousarray(leader_of, dtype=np.int32)
    qq, dt = _buf(q)
    assert K_lead.flags.c_contiguous and V_lead.flags.c_contiguous
    kn = _buf(k_new)[0] if k_new is not None else None
    vn = _buf(v_new)[0] if v_new is not None else None
    _, B, Hkv, L_max, hd = K_lead.shape
    Hq = qq.shape[1]
    out = np.empty((B, Hq, hd), dtype=np.float32)
    _check(lib().oracle_rcla_decode_attend(B, Hq, Hkv, hd, dt, layer, _p(lo), len(lo),
                                           _p(K_lead), _p(V_lead), L_max, length,
                                           _p(kn) if kn is not None else None,
                                           _p(vn) if vn is not None else None, _p(qq), _p(out)),
           "rcla_decode_attend")
    return out


def footprint_bytes(batch, n_kv_heads, head_dim, ctx_len, chunk, rank_k, rank_v, dtype,
                    n_layers, window, with_landmarks) -> int:
    return int(lib().oracle_footprint_bytes(batch, n_kv_heads, head_dim, ctx_len, chunk,
                                            rank_k, rank_v, dtype, n_layers, window,
                                            int(with_landmarks)))


def rcla_cache_bytes(batch, n_kv_heads, head_dim, ctx_len, dtype, n_leaders) -> int:
    return int(lib().oracle_rcla_cache_bytes(batch, n_kv_heads, head_dim, ctx_len, dtype,
                                             n_leaders))
