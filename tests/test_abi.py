"""Host side of the C ABI (no GPU needed): the library loads, exports every entry point
include/xkv.h declares, rejects bad arguments before touching CUDA, propagates injected
faults, and its size helpers agree with the oracle's closed forms."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def xkv():
    from cross_layer_compressed_b200 import build
    build.build()
    from cross_layer_compressed_b200 import xkv as m
    return m


def _declared_functions():
    src = open(os.path.join(ROOT, "include", "xkv.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\s*\*?\s*([a-z_][a-z0-9_]*)\s*\(",
                       src, flags=re.M)
    return sorted(set(names))


def test_library_exports_every_declared_symbol(xkv):
    names = _declared_functions()
    assert {"xkv_score_landmarks", "xkv_select_chunks", "xkv_reconstruct_attend",
            "rcla_decode_attend", "xkv_build_landmarks"} <= set(names)
    lib = ctypes.CDLL(xkv.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n


def test_library_is_built_for_sm100a_only():
    """The in-tree build targets sm_100a (checked from the build flags, not the binary)."""
    from cross_layer_compressed_b200 import build
    assert "arch=compute_100a,code=sm_100a" in build.FLAGS


FAKE = 0x10000  # aligned, never dereferenced on the host


def _d(xkv, **kw):
    base = dict(batch=2, n_q_heads=8, n_kv_heads=2, head_dim=128, ctx_len=1024, chunk=8,
                rank_k=64, rank_v=64, dtype=xkv.XKV_BF16)
    base.update(kw)
    return xkv.dims(**base)


@pytest.mark.parametrize("kw,status", [
    (dict(n_q_heads=6, n_kv_heads=4), 1),          # Hq % Hkv
    (dict(head_dim=96), 2),                         # unsupported head_dim
    (dict(chunk=12), 1),                            # chunk not a multiple of 8
    (dict(ctx_len=1004), 1),                        # L % C
    (dict(rank_k=40), 1),                           # rank not a multiple of 16
    (dict(rank_v=2048), 2),                         # rank above 1024
    (dict(batch=0), 1),
    (dict(dtype=7), 1),
    (dict(n_q_heads=34, n_kv_heads=2), 2),          # G > 16
])
def test_bad_dims_rejected_without_launch(xkv, kw, status):
    d = _d(xkv, **kw)
    st = xkv.xkv_score_landmarks(d, FAKE, FAKE, FAKE, stream=0, check=False)
    assert st == status
    assert xkv.last_error()


def test_null_and_misaligned_pointers_rejected(xkv):
    d = _d(xkv)
    assert xkv.xkv_score_landmarks(d, 0, FAKE, FAKE, stream=0, check=False) == 1
    assert xkv.xkv_score_landmarks(d, FAKE + 8, FAKE, FAKE, stream=0, check=False) == 1
    assert "aligned" in xkv.last_error()
    assert xkv.xkv_build_landmarks(d, FAKE, FAKE + 2, FAKE, stream=0, check=False) == 1
    assert xkv.xkv_select_chunks(d, FAKE, -1, 1, 1, FAKE, stream=0, check=False) == 1
    ws = xkv.xkv_workspace_bytes(d, 10, xkv.XKV_MODE_SELECTIVE)
    assert xkv.xkv_reconstruct_attend(d, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 0, FAKE, FAKE, ws,
                                      stream=0, check=False) == 1      # n_sel = 0
    assert xkv.xkv_reconstruct_attend(d, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 129, FAKE, FAKE,
                                      ws, stream=0, check=False) == 1  # n_sel > nC


def test_workspace_too_small_rejected(xkv):
    d = _d(xkv)
    ws = xkv.xkv_workspace_bytes(d, 20, xkv.XKV_MODE_SELECTIVE)
    assert ws > 0
    st = xkv.xkv_reconstruct_attend(d, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 20, FAKE, FAKE,
                                    ws - 4, stream=0, check=False)
    assert st == 1 and "workspace" in xkv.last_error()


def test_workspace_bound_covers_every_smaller_call(xkv):
    """A workspace sized for the largest row count fits every smaller call (the split
    count used by a call never exceeds the bound)."""
    for G, Hkv, B in [(4, 8, 8), (5, 8, 1), (1, 2, 3), (16, 1, 1)]:
        d = _d(xkv, n_q_heads=G * Hkv, n_kv_heads=Hkv, batch=B, ctx_len=4096)
        big = xkv.xkv_workspace_bytes(d, 512, xkv.XKV_MODE_SELECTIVE)
        for n in range(1, 513, 7):
            assert xkv.xkv_workspace_bytes(d, n, xkv.XKV_MODE_SELECTIVE) <= big
        dr = _d(xkv, n_q_heads=G * Hkv, n_kv_heads=Hkv, batch=B, ctx_len=40000)
        big_r = xkv.xkv_workspace_bytes(dr, 0, xkv.XKV_MODE_RCLA)
        for L in list(range(1, 40000, 997)) + [40000]:
            dd = _d(xkv, n_q_heads=G * Hkv, n_kv_heads=Hkv, batch=B, ctx_len=L)
            assert xkv.xkv_workspace_bytes(dd, 0, xkv.XKV_MODE_RCLA) <= big_r


def test_tail_call_arguments_rejected_without_launch(xkv):
    """xkv_reconstruct_attend_tail: the tail's bounds, pointers and workspace are checked
    before any CUDA call, and its workspace adds room for the tail's splits."""
    d = _d(xkv)
    base = xkv.xkv_workspace_bytes(d, 10, xkv.XKV_MODE_SELECTIVE)
    ws = xkv.xkv_tail_workspace_bytes(d, 10, 64)
    assert ws > base and xkv.xkv_tail_workspace_bytes(d, 10, 0) == 0
    assert xkv.xkv_tail_workspace_bytes(d, 10, 128) >= ws   # bound grows with T_max
    args = (FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 10)

    def call(Kt, Vt, T_max, n_tail, wsb=ws):
        return xkv.xkv_reconstruct_attend_tail(d, *args, Kt, Vt, T_max, n_tail, FAKE, FAKE,
                                               wsb, stream=0, check=False)
    assert call(FAKE, FAKE, 64, 65) == 1                    # n_tail > T_max
    assert call(FAKE, FAKE, 0, 0) == 1                      # T_max must be positive
    assert call(FAKE, FAKE, 64, -1) == 1
    assert call(0, FAKE, 64, 3) == 1                        # tail pointer missing
    assert call(FAKE + 4, FAKE, 64, 3) == 1                 # misaligned
    assert call(FAKE, FAKE, 64, 3, ws - 4) == 1             # workspace too small
    assert "workspace" in xkv.last_error()


def test_rcla_leader_rules(xkv):
    d = _d(xkv)
    ws = xkv.xkv_workspace_bytes(_d(xkv, ctx_len=64), 0, xkv.XKV_MODE_RCLA)
    lo = [0, 0, 2, 2]

    def call(layer, leader_of, length=10, kn=None, vn=None, L_max=64):
        return xkv.rcla_decode_attend(d, layer, leader_of, FAKE, FAKE, L_max, length, kn, vn,
                                      FAKE, FAKE, FAKE, ws, stream=0, check=False)
    assert call(1, lo, kn=FAKE, vn=FAKE) == 1            # non-leader with a new row
    assert "not a leader" in xkv.last_error()
    assert call(2, lo, kn=FAKE) == 1                     # k_new without v_new
    assert call(0, [1, 1, 2, 2]) == 1                    # layer 0 not a leader
    assert call(3, [0, 0, 3, 2]) == 1                    # leader_of[2] = 3 > 2
    assert call(3, [0, 0, 1, 1]) == 1                    # 1 is not a leader
    assert call(4, lo) == 1                              # layer out of range
    assert call(2, lo, length=64, kn=FAKE, vn=FAKE) == 1  # no room for the new row
    assert call(0, lo, length=0) == 1                    # nothing to attend


def test_fault_injection_propagates_before_any_launch(xkv, monkeypatch):
    """XKV_FAULT makes a valid call return the injected status on the host (no GPU)."""
    d = _d(xkv)
    monkeypatch.setenv("XKV_FAULT", "xkv_score_landmarks:3")
    assert xkv.xkv_score_landmarks(d, FAKE, FAKE, FAKE, stream=0, check=False) == 3
    assert "injected" in xkv.last_error()
    with pytest.raises(xkv.XkvError) as ei:
        xkv.xkv_score_landmarks(d, FAKE, FAKE, FAKE, stream=0)
    assert ei.value.status == xkv.XKV_ERR_CUDA
    monkeypatch.setenv("XKV_FAULT", "rcla_decode_attend:4")
    ws = xkv.xkv_workspace_bytes(_d(xkv, ctx_len=64), 0, xkv.XKV_MODE_RCLA)
    assert xkv.rcla_decode_attend(d, 1, [0, 0], FAKE, FAKE, 64, 10, None, None, FAKE, FAKE,
                                  FAKE, ws, stream=0, check=False) == 4
    # other entry points are unaffected (they fail later, on the device check)
    monkeypatch.setenv("XKV_FAULT", "xkv_select_chunks:5")
    assert xkv.xkv_score_landmarks(d, FAKE, 0, FAKE, stream=0, check=False) == 1


def test_size_helpers_match_oracle(xkv, ora):
    for (B, Hkv, hd, L, C, rk, rv, dt, N, W, lm) in [
            (8, 8, 128, 32768, 8, 512, 768, 1, 32, 4, 1), (1, 2, 64, 1024, 8, 64, 64, 0, 2, 2, 0),
            (64, 8, 128, 16384, 8, 512, 768, 1, 48, 4, 1), (3, 2, 64, 96, 16, 32, 48, 1, 5, 2, 1)]:
        d = xkv.dims(B, Hkv * 4, Hkv, hd, L, C, rk, rv, dt)
        assert xkv.xkv_footprint_bytes(d, N, W, lm) == ora.footprint_bytes(
            B, Hkv, hd, L, C, rk, rv, dt, N, W, lm)
    for nC, k, s, r in [(4096, 256, 1, 4), (10, 50, 1, 2), (3, 1, 2, 2), (128, 16, 1, 1),
                        (7, 0, 0, 0), (5, 2, 9, 0), (5, 2, 0, 9)]:
        assert xkv.xkv_n_selected(nC, k, s, r) == ora.n_selected(nC, k, s, r)
    d = xkv.dims(16, 32, 8, 128, 32832, dtype=1)
    assert xkv.rcla_cache_bytes(d, 9, 32832) == ora.rcla_cache_bytes(16, 8, 128, 32832, 1, 9)


def test_plain_c_program_links_and_calls_the_host_entry_points(xkv, tmp_path):
    """The boundary is a C ABI: a C99 program that includes include/xkv.h and links the
    library calls the host-only entry points (no device needed) and gets the same
    answers as the Python binding."""
    import shutil
    import subprocess
    if shutil.which("gcc") is None:
        pytest.skip("no C compiler")
    src = tmp_path / "abi.c"
    src.write_text(r'''
#include <stdio.h>
#include "xkv.h"
int main(void) {
    xkv_dims d = {8, 32, 8, 128, 32768, 8, 512, 768, XKV_BF16};
    long long nsel = (long long)xkv_n_selected(4096, 256, 1, 4);
    long long fp = (long long)xkv_footprint_bytes(&d, 32, 4, 1);
    unsigned long long ws = (unsigned long long)xkv_workspace_bytes(&d, 261, XKV_MODE_SELECTIVE);
    xkv_dims bad = d;
    bad.head_dim = 96;
    xkv_status st = xkv_score_landmarks(&bad, (void *)0, (void *)0, (double *)0, (void *)0);
    unsigned long long fws = (unsigned long long)xkv_factorize_workspace_bytes(&d, 4, 512);
    unsigned long long rws = (unsigned long long)xkv_refold_workspace_bytes(&d, 4, 512, 256);
    printf("%lld %lld %llu %d %s %llu %llu\n", nsel, fp, ws, (int)st,
           xkv_last_error()[0] ? "msg" : "none", fws, rws);
    return 0;
}
''')
    lib_dir = os.path.dirname(xkv.LIB_PATH)
    exe = tmp_path / "abi"
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", str(src), "-I",
                    os.path.join(ROOT, "include"), "-L", lib_dir, "-lxkv",
                    f"-Wl,-rpath,{lib_dir}", "-o", str(exe)], check=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout.split()
    d = xkv.dims(8, 32, 8, 128, 32768, 8, 512, 768, xkv.XKV_BF16)
    assert int(out[0]) == xkv.xkv_n_selected(4096, 256, 1, 4) == 261
    assert int(out[1]) == xkv.xkv_footprint_bytes(d, 32, 4, 1)
    assert int(out[2]) == xkv.xkv_workspace_bytes(d, 261, xkv.XKV_MODE_SELECTIVE)
    assert int(out[3]) == xkv.XKV_ERR_UNSUPPORTED and out[4] == "msg"
    assert int(out[5]) == xkv.xkv_factorize_workspace_bytes(d, 4, 512) > 0
    assert int(out[6]) == xkv.xkv_refold_workspace_bytes(d, 4, 512, 256) > int(out[5])


# ------------------------------------------------------- cross-layer factorization
def _fd(xkv, **kw):
    base = dict(batch=2, n_q_heads=2, n_kv_heads=2, head_dim=64, ctx_len=1000, chunk=8,
                rank_k=0, rank_v=0, dtype=xkv.XKV_BF16)
    base.update(kw)
    return xkv.dims(**base)


@pytest.mark.parametrize("kw,window,rank,n_iter,status", [
    ({}, 0, 32, 1, 1),                              # window < 1
    ({}, 2, 40, 1, 1),                              # rank not a multiple of 16
    ({}, 2, 0, 1, 1),
    ({}, 2, 2048, 1, 2),                            # rank above 1024
    (dict(ctx_len=16), 2, 32, 1, 1),                # rank above L
    (dict(n_kv_heads=1), 1, 80, 1, 1),              # rank above W * d_kv = 64
    ({}, 2, 32, -1, 1),                             # n_iter out of range
    ({}, 2, 32, 17, 1),
    (dict(head_dim=96), 2, 32, 1, 2),
    (dict(dtype=5), 2, 32, 1, 1),
    (dict(batch=0), 2, 32, 1, 1),
])
def test_factorize_bad_arguments_rejected_without_launch(xkv, kw, window, rank, n_iter, status):
    d = _fd(xkv, **kw)
    st = xkv.xkv_factorize_window(d, window, rank, FAKE, FAKE, n_iter, FAKE, FAKE, FAKE,
                                  1 << 40, stream=0, check=False)
    assert st == status
    assert xkv.last_error()


def test_factorize_pointer_and_workspace_checks(xkv):
    d = _fd(xkv)
    need = xkv.xkv_factorize_workspace_bytes(d, 2, 32)
    B, L, r, n = 2, 1000, 32, 2 * 128

    def al(x):
        return (x + 255) // 256 * 256
    # status header; Y and Z ping-pong (fp32); Gram, diagonal-block inverses, R^-1 (fp64);
    # tolerances; R^-1 (fp32); bf16 hi / lo splits and the bf16 test matrix
    assert need == (256 + 2 * al(B * L * r * 4) + 2 * al(B * n * r * 4) + al(B * r * r * 8)
                    + al(B * 1 * 64 * 64 * 8) + al(B * r * r * 8) + al(B * 8) + al(B * r * r * 4)
                    + 2 * al(B * max(L, n) * r * 2) + al(n * r * 2))
    assert xkv.xkv_factorize_workspace_bytes(d, 2, 40) == 0
    args = [FAKE] * 2
    assert xkv.xkv_factorize_window(d, 2, 32, 0, FAKE, 1, FAKE, FAKE, FAKE, need, stream=0,
                                    check=False) == 1
    assert xkv.xkv_factorize_window(d, 2, 32, FAKE, FAKE + 4, 1, FAKE, FAKE, FAKE, need,
                                    stream=0, check=False) == 1
    assert "aligned" in xkv.last_error()
    assert xkv.xkv_factorize_window(d, 2, 32, *args, 1, FAKE, FAKE, FAKE, need - 1, stream=0,
                                    check=False) == 1
    assert "workspace" in xkv.last_error()


def test_factorize_fault_injection(xkv, monkeypatch):
    monkeypatch.setenv("XKV_FAULT", "xkv_factorize_window:4")
    d = _fd(xkv)
    need = xkv.xkv_factorize_workspace_bytes(d, 2, 32)
    assert xkv.xkv_factorize_window(d, 2, 32, FAKE, FAKE, 1, FAKE, FAKE, FAKE, need, stream=0,
                                    check=False) == 4
    assert "injected" in xkv.last_error()


def test_refold_argument_checks(xkv, monkeypatch):
    d = _fd(xkv)
    need = xkv.xkv_refold_workspace_bytes(d, 2, 32, 100)
    assert need > xkv.xkv_factorize_workspace_bytes(d, 2, 32)
    # the factorization's scratch and the extended caches (W x B x (L + T) x d_kv, bf16)
    assert need == (2 * 2 * 1100 * 128 * 2 + 255) // 256 * 256 + \
        xkv.xkv_factorize_workspace_bytes(_fd(xkv, ctx_len=1100), 2, 32)
    assert xkv.xkv_refold_workspace_bytes(d, 2, 32, -1) == 0
    args = dict(A_win=FAKE, Bt_win=FAKE, tail=FAKE, omega=FAKE, A_out=FAKE, Bt_out=FAKE, ws=FAKE)

    def call(**kw):
        a = {**args, **kw}
        return xkv.xkv_refold_window(kw.pop("d", d), 2, kw.pop("rank", 32), a["A_win"],
                                     a["Bt_win"], a["tail"], kw.get("n_tail", 100), a["omega"],
                                     kw.get("n_iter", 1), a["A_out"], a["Bt_out"], a["ws"],
                                     kw.get("ws_bytes", need), stream=0, check=False)
    assert call(n_tail=-1) == 1
    assert call(tail=0) == 1                       # a tail is needed when n_tail > 0
    assert call(A_win=FAKE + 8) == 1 and "aligned" in xkv.last_error()
    assert call(ws_bytes=need - 1) == 1 and "workspace" in xkv.last_error()
    assert call(n_iter=17) == 1
    assert call(rank=40) == 1
    monkeypatch.setenv("XKV_FAULT", "xkv_refold_window:3")
    assert call() == 3
    # no tail: NULL is accepted and only the factorization's scratch is added
    need0 = xkv.xkv_refold_workspace_bytes(d, 2, 32, 0)
    assert call(tail=0, n_tail=0, ws_bytes=need0) == 3


# --------------------------------------------------- allocation-free reconstruct+attend
def test_noalloc_arguments_rejected_before_any_cuda_call(xkv, monkeypatch):
    """xkv_reconstruct_attend_noalloc checks every argument on the host under its own
    name before it asks CUDA for anything, so these fail the same way with no GPU."""
    d = _d(xkv)

    def call(dd=d, ptrs=(FAKE,) * 6, n_sel=10, out=FAKE):
        return xkv.xkv_reconstruct_attend_noalloc(dd, *ptrs, n_sel, out, stream=0, check=False)
    assert call(dd=_d(xkv, head_dim=96)) == xkv.XKV_ERR_UNSUPPORTED
    assert call(dd=_d(xkv, chunk=12)) == xkv.XKV_ERR_INVALID_ARG
    assert "xkv_reconstruct_attend_noalloc" in xkv.last_error()
    assert call(ptrs=(0,) + (FAKE,) * 5) == xkv.XKV_ERR_INVALID_ARG          # NULL basis
    assert call(out=0) == xkv.XKV_ERR_INVALID_ARG                           # NULL output
    assert call(ptrs=(FAKE, FAKE + 8) + (FAKE,) * 4) == xkv.XKV_ERR_INVALID_ARG
    assert "aligned" in xkv.last_error()
    assert call(ptrs=(FAKE,) * 5 + (FAKE + 4,)) == xkv.XKV_ERR_INVALID_ARG   # misaligned sel
    assert call(n_sel=0) == xkv.XKV_ERR_INVALID_ARG                          # n_sel out of range
    assert call(n_sel=129) == xkv.XKV_ERR_INVALID_ARG
    # a call whose scratch exceeds the fixed array is refused before any CUDA call
    big = xkv.dims(64, 512, 32, 128, 1 << 20, 8, 512, 768, xkv.XKV_BF16)
    assert call(dd=big, ptrs=(FAKE,) * 5 + (None,), n_sel=0) == xkv.XKV_ERR_UNSUPPORTED
    assert "scratch" in xkv.last_error()
    # fault injection under this entry point's own name, after the checks
    monkeypatch.setenv("XKV_FAULT", "xkv_reconstruct_attend_noalloc:4")
    assert call() == 4 and "injected" in xkv.last_error()
    assert call(n_sel=0) == xkv.XKV_ERR_INVALID_ARG          # argument errors come first
    monkeypatch.setenv("XKV_FAULT", "xkv_reconstruct_attend:4")
    assert call(out=0) == xkv.XKV_ERR_INVALID_ARG
