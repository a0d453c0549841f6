"""Thin Python binding of the C ABI in include/xkv.h (ctypes; argument marshalling only).

Every function has the name of the C entry point it calls.  Tensor arguments are torch
CUDA tensors (or raw device addresses as ints); every step of the computation runs in
the library's CUDA kernels.  Importing this module raises if the library is not built:
there is no CPU fallback.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libxkv.so")

XKV_OK, XKV_ERR_INVALID_ARG, XKV_ERR_UNSUPPORTED, XKV_ERR_CUDA, XKV_ERR_TIMEOUT, \
    XKV_ERR_INTERNAL = range(6)
XKV_F32, XKV_BF16 = 0, 1
XKV_MODE_SELECTIVE, XKV_MODE_DENSE, XKV_MODE_RCLA, XKV_MODE_REASSOC = 0, 1, 2, 3

STATUS_NAMES = {0: "XKV_OK", 1: "XKV_ERR_INVALID_ARG", 2: "XKV_ERR_UNSUPPORTED",
                3: "XKV_ERR_CUDA", 4: "XKV_ERR_TIMEOUT", 5: "XKV_ERR_INTERNAL"}


class XkvError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {message}")
        self.status = status


class xkv_dims(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int32), ("n_q_heads", ctypes.c_int32),
                ("n_kv_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("ctx_len", ctypes.c_int64), ("chunk", ctypes.c_int32),
                ("rank_k", ctypes.c_int32), ("rank_v", ctypes.c_int32),
                ("dtype", ctypes.c_int32)]


if not os.path.exists(LIB_PATH):
    raise ImportError(f"CUDA library not built ({LIB_PATH} missing); run "
                      "`python -m cross_layer_compressed_b200.build` or __graft_entry__.build()")

_lib = ctypes.CDLL(LIB_PATH)
_vp, _i32, _i64, _sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
_D = ctypes.POINTER(xkv_dims)
_sigs = {
    "xkv_build_landmarks": ([_D, _vp, _vp, _vp, _vp], ctypes.c_int),
    "xkv_score_landmarks": ([_D, _vp, _vp, _vp, _vp], ctypes.c_int),
    "xkv_select_chunks": ([_D, _vp, _i32, _i32, _i32, _vp, ctypes.POINTER(_i32), _vp],
                          ctypes.c_int),
    "xkv_score_select": ([_D, _vp, _vp, _i32, _i32, _i32, _vp, _i32, _vp, ctypes.POINTER(_i32),
                          _vp, _sz, _vp], ctypes.c_int),
    "xkv_score_select_workspace_bytes": ([_D], _sz),
    "xkv_build_value_ranges": ([_D, _vp, _vp, _vp, _vp, _vp], ctypes.c_int),
    "xkv_reserve_value_chunks": ([_D, _vp, _i32, _i32, _i32, _vp, ctypes.POINTER(_i32), _vp],
                                 ctypes.c_int),
    "xkv_n_reserved": ([_i64, _i32, _i32, _i32], _i64),
    "xkv_reconstruct_attend": ([_D, _vp, _vp, _vp, _vp, _vp, _vp, _i32, _vp, _vp, _sz, _vp],
                               ctypes.c_int),
    "rcla_decode_attend": ([_D, _i32, _vp, _i32, _vp, _vp, _i64, _i64, _vp, _vp, _vp, _vp, _vp,
                            _sz, _vp], ctypes.c_int),
    "xkv_reconstruct_attend_tail": ([_D, _vp, _vp, _vp, _vp, _vp, _vp, _i32, _vp, _vp, _i64,
                                     _i64, _vp, _vp, _sz, _vp], ctypes.c_int),
    "xkv_tail_workspace_bytes": ([_D, _i32, _i64], _sz),
    "xkv_reassociated_attend": ([_D, _vp, _vp, _vp, _vp, _vp, _vp, _i32, _vp, _vp, _sz, _vp],
                                ctypes.c_int),
    "xkv_reconstruct_attend_noalloc": ([_D, _vp, _vp, _vp, _vp, _vp, _vp, _i32, _vp, _vp],
                                       ctypes.c_int),
    "xkv_workspace_bytes": ([_D, _i32, _i32], _sz),
    "xkv_factorize_window": ([_D, _i32, _i32, _vp, _vp, _i32, _vp, _vp, _vp, _sz, _vp],
                             ctypes.c_int),
    "xkv_factorize_workspace_bytes": ([_D, _i32, _i32], _sz),
    "xkv_refold_window": ([_D, _i32, _i32, _vp, _vp, _vp, _i64, _vp, _i32, _vp, _vp, _vp, _sz,
                           _vp], ctypes.c_int),
    "xkv_refold_workspace_bytes": ([_D, _i32, _i32, _i64], _sz),
    "xkv_n_selected": ([_i64, _i32, _i32, _i32], _i64),
    "xkv_footprint_bytes": ([_D, _i32, _i32, _i32], _i64),
    "rcla_cache_bytes": ([_D, _i32, _i64], _i64),
    "xkv_last_error": ([], ctypes.c_char_p),
}
for _name, (_args, _ret) in _sigs.items():
    _f = getattr(_lib, _name)
    _f.argtypes, _f.restype = _args, _ret


def dims(batch, n_q_heads, n_kv_heads, head_dim, ctx_len, chunk=8, rank_k=0, rank_v=0,
         dtype=XKV_BF16) -> xkv_dims:
    if isinstance(dtype, str):
        dtype = XKV_F32 if dtype == "f32" else XKV_BF16
    return xkv_dims(batch, n_q_heads, n_kv_heads, head_dim, ctx_len, chunk, rank_k, rank_v,
                    dtype)


def dims_of(w, **over) -> xkv_dims:
    """xkv_dims of a synth.Workload (fields can be overridden)."""
    kw = dict(batch=w.batch, n_q_heads=w.n_q_heads, n_kv_heads=w.n_kv_heads,
              head_dim=w.head_dim, ctx_len=w.ctx_len, chunk=w.chunk, rank_k=w.rank_k,
              rank_v=w.rank_v, dtype=w.dtype)
    kw.update(over)
    return dims(**kw)


def _ptr(x):
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _stream(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream if torch.cuda.is_available() else None
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(status: int):
    if status != XKV_OK:
        raise XkvError(status, (_lib.xkv_last_error() or b"").decode())


def last_error() -> str:
    return (_lib.xkv_last_error() or b"").decode()


# --------------------------------------------------------------------- entry points
def xkv_build_landmarks(d: xkv_dims, Ak_win, Bkt_layer, lm_layer, stream=None, check=True):
    st = _lib.xkv_build_landmarks(ctypes.byref(d), _ptr(Ak_win), _ptr(Bkt_layer),
                                  _ptr(lm_layer), _stream(stream))
    if check:
        _check(st)
    return st


def xkv_score_landmarks(d: xkv_dims, lm_layer, q, scores, stream=None, check=True):
    st = _lib.xkv_score_landmarks(ctypes.byref(d), _ptr(lm_layer), _ptr(q), _ptr(scores),
                                  _stream(stream))
    if check:
        _check(st)
    return st


def xkv_select_chunks(d: xkv_dims, scores, top_k, n_sink, n_recent, sel, stream=None,
                      check=True):
    """Returns n_sel (or the status when check=False)."""
    n = _i32(0)
    st = _lib.xkv_select_chunks(ctypes.byref(d), _ptr(scores), top_k, n_sink, n_recent,
                                _ptr(sel), ctypes.byref(n), _stream(stream))
    if check:
        _check(st)
        return n.value
    return st


def xkv_score_select(d: xkv_dims, lm_layer, q, top_k, n_sink, n_recent, sel, ws,
                     ws_bytes=None, stream=None, check=True, reserved=None, n_reserved=0):
    """Returns n_sel (or the status when check=False)."""
    if ws_bytes is None:
        ws_bytes = ws.numel() * ws.element_size()
    n = _i32(0)
    st = _lib.xkv_score_select(ctypes.byref(d), _ptr(lm_layer), _ptr(q), int(top_k),
                               int(n_sink), int(n_recent), _ptr(reserved), int(n_reserved),
                               _ptr(sel), ctypes.byref(n), _ptr(ws), int(ws_bytes),
                               _stream(stream))
    if check:
        _check(st)
        return n.value
    return st


def xkv_score_select_workspace_bytes(d: xkv_dims) -> int:
    return int(_lib.xkv_score_select_workspace_bytes(ctypes.byref(d)))


def xkv_build_value_ranges(d: xkv_dims, Av_win, Bvt_layer, rho_layer, status=None, stream=None,
                           check=True):
    st = _lib.xkv_build_value_ranges(ctypes.byref(d), _ptr(Av_win), _ptr(Bvt_layer),
                                     _ptr(rho_layer), _ptr(status), _stream(stream))
    if check:
        _check(st)
    return st


def xkv_reserve_value_chunks(d: xkv_dims, rho_layer, n_value, n_sink, n_recent, reserved,
                             stream=None, check=True):
    """Returns n_res (or the status when check=False)."""
    n = _i32(0)
    st = _lib.xkv_reserve_value_chunks(ctypes.byref(d), _ptr(rho_layer), int(n_value),
                                       int(n_sink), int(n_recent), _ptr(reserved),
                                       ctypes.byref(n), _stream(stream))
    if check:
        _check(st)
        return n.value
    return st


def xkv_n_reserved(n_chunks, n_value, n_sink, n_recent) -> int:
    return int(_lib.xkv_n_reserved(int(n_chunks), int(n_value), int(n_sink), int(n_recent)))


def xkv_reconstruct_attend(d: xkv_dims, Ak_win, Av_win, Bkt_layer, Bvt_layer, q, sel, n_sel,
                           out, ws, ws_bytes=None, stream=None, check=True):
    if ws_bytes is None:
        ws_bytes = ws.numel() * ws.element_size()
    st = _lib.xkv_reconstruct_attend(ctypes.byref(d), _ptr(Ak_win), _ptr(Av_win),
                                     _ptr(Bkt_layer), _ptr(Bvt_layer), _ptr(q), _ptr(sel),
                                     int(n_sel), _ptr(out), _ptr(ws), int(ws_bytes),
                                     _stream(stream))
    if check:
        _check(st)
    return st


def xkv_reconstruct_attend_tail(d: xkv_dims, Ak_win, Av_win, Bkt_layer, Bvt_layer, q, sel,
                                n_sel, K_tail, V_tail, T_max, n_tail, out, ws, ws_bytes=None,
                                stream=None, check=True):
    if ws_bytes is None:
        ws_bytes = ws.numel() * ws.element_size()
    st = _lib.xkv_reconstruct_attend_tail(ctypes.byref(d), _ptr(Ak_win), _ptr(Av_win),
                                          _ptr(Bkt_layer), _ptr(Bvt_layer), _ptr(q), _ptr(sel),
                                          int(n_sel), _ptr(K_tail), _ptr(V_tail), int(T_max),
                                          int(n_tail), _ptr(out), _ptr(ws), int(ws_bytes),
                                          _stream(stream))
    if check:
        _check(st)
    return st


def xkv_tail_workspace_bytes(d: xkv_dims, n_sel, T_max) -> int:
    return int(_lib.xkv_tail_workspace_bytes(ctypes.byref(d), int(n_sel), int(T_max)))


def xkv_reassociated_attend(d: xkv_dims, Ak_win, Av_win, Bkt_layer, Bvt_layer, q, sel, n_sel,
                            out, ws, ws_bytes=None, stream=None, check=True):
    if ws_bytes is None:
        ws_bytes = ws.numel() * ws.element_size()
    st = _lib.xkv_reassociated_attend(ctypes.byref(d), _ptr(Ak_win), _ptr(Av_win),
                                      _ptr(Bkt_layer), _ptr(Bvt_layer), _ptr(q), _ptr(sel),
                                      int(n_sel), _ptr(out), _ptr(ws), int(ws_bytes),
                                      _stream(stream))
    if check:
        _check(st)
    return st


def xkv_reconstruct_attend_noalloc(d: xkv_dims, Ak_win, Av_win, Bkt_layer, Bvt_layer, q, sel,
                                   n_sel, out, stream=None, check=True):
    """xkv_reconstruct_attend with the library's fixed scratch array instead of a
    workspace, for callers that cannot allocate device memory (see include/xkv.h)."""
    st = _lib.xkv_reconstruct_attend_noalloc(ctypes.byref(d), _ptr(Ak_win), _ptr(Av_win),
                                             _ptr(Bkt_layer), _ptr(Bvt_layer), _ptr(q),
                                             _ptr(sel), int(n_sel), _ptr(out), _stream(stream))
    if check:
        _check(st)
    return st


def rcla_decode_attend(d: xkv_dims, layer, leader_of, K_lead, V_lead, L_max, length, k_new,
                       v_new, q, out, ws, ws_bytes=None, stream=None, check=True):
    lo = (_i32 * len(leader_of))(*[int(x) for x in leader_of])
    if ws_bytes is None:
        ws_bytes = ws.numel() * ws.element_size()
    st = _lib.rcla_decode_attend(ctypes.byref(d), int(layer), lo, len(leader_of), _ptr(K_lead),
                                 _ptr(V_lead), int(L_max), int(length), _ptr(k_new),
                                 _ptr(v_new), _ptr(q), _ptr(out), _ptr(ws), int(ws_bytes),
                                 _stream(stream))
    if check:
        _check(st)
    return st


def xkv_factorize_window(d: xkv_dims, window, rank, X, omega, n_iter, A_out, Bt_out, ws,
                         ws_bytes=None, stream=None, check=True):
    if ws_bytes is None:
        ws_bytes = ws.numel() * ws.element_size()
    st = _lib.xkv_factorize_window(ctypes.byref(d), int(window), int(rank), _ptr(X), _ptr(omega),
                                   int(n_iter), _ptr(A_out), _ptr(Bt_out), _ptr(ws),
                                   int(ws_bytes), _stream(stream))
    if check:
        _check(st)
    return st


def xkv_factorize_workspace_bytes(d: xkv_dims, window, rank) -> int:
    return int(_lib.xkv_factorize_workspace_bytes(ctypes.byref(d), int(window), int(rank)))


def xkv_refold_window(d: xkv_dims, window, rank, A_win, Bt_win, tail, n_tail, omega, n_iter,
                      A_out, Bt_out, ws, ws_bytes=None, stream=None, check=True):
    if ws_bytes is None:
        ws_bytes = ws.numel() * ws.element_size()
    st = _lib.xkv_refold_window(ctypes.byref(d), int(window), int(rank), _ptr(A_win),
                                _ptr(Bt_win), _ptr(tail) if tail is not None else None,
                                int(n_tail), _ptr(omega), int(n_iter), _ptr(A_out),
                                _ptr(Bt_out), _ptr(ws), int(ws_bytes), _stream(stream))
    if check:
        _check(st)
    return st


def xkv_refold_workspace_bytes(d: xkv_dims, window, rank, n_tail) -> int:
    return int(_lib.xkv_refold_workspace_bytes(ctypes.byref(d), int(window), int(rank),
                                               int(n_tail)))


def xkv_workspace_bytes(d: xkv_dims, n_sel: int, mode: int) -> int:
    return int(_lib.xkv_workspace_bytes(ctypes.byref(d), int(n_sel), int(mode)))


def xkv_n_selected(n_chunks, top_k, n_sink, n_recent) -> int:
    return int(_lib.xkv_n_selected(int(n_chunks), int(top_k), int(n_sink), int(n_recent)))


def xkv_footprint_bytes(d: xkv_dims, n_layers, window, with_landmarks) -> int:
    return int(_lib.xkv_footprint_bytes(ctypes.byref(d), int(n_layers), int(window),
                                        int(with_landmarks)))


def rcla_cache_bytes(d: xkv_dims, n_leaders, L_max) -> int:
    return int(_lib.rcla_cache_bytes(ctypes.byref(d), int(n_leaders), int(L_max)))


def xkv_last_error() -> str:
    return last_error()
