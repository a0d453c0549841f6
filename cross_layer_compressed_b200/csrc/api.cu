// C ABI of the xKV decode-attention library (declared in include/xkv.h).
//
// Every entry point validates its arguments on the host before touching CUDA, so an
// argument error launches nothing and needs no GPU.  Launch failures map to
// XKV_ERR_CUDA.  The message of the last non-OK status is kept per calling thread.
//
// Host-side fault injection for tests: XKV_FAULT="<entry point>:<status code>" makes
// that entry point return the status before launching anything.
#include <cuda_runtime.h>

#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <string>

#include <nvtx3/nvToolsExt.h>

#include "xkv_internal.cuh"

using namespace xkv;

namespace {

// An NVTX range named after the entry point around each launching call, so profilers
// can select a call's kernels (no cost without a profiler attached).
struct Range {
    explicit Range(const char *name) { nvtxRangePushA(name); }
    ~Range() { nvtxRangePop(); }
    Range(const Range &) = delete;
    Range &operator=(const Range &) = delete;
};

thread_local std::string g_last_error;

xkv_status fail(xkv_status st, const char *fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof buf, fmt, ap);
    va_end(ap);
    g_last_error = buf;
    return st;
}

xkv_status ok() {
    g_last_error.clear();
    return XKV_OK;
}

// XKV_FAULT="name:code" -> that status for the named entry point (tests only).
bool injected(const char *name, xkv_status *st) {
    const char *f = getenv("XKV_FAULT");
    if (!f) return false;
    const char *colon = strchr(f, ':');
    if (!colon || (size_t)(colon - f) != strlen(name) || strncmp(f, name, colon - f) != 0)
        return false;
    *st = (xkv_status)atoi(colon + 1);
    g_last_error = std::string("injected fault in ") + name;
    return true;
}

bool aligned16(const void *p) { return ((uintptr_t)p & 15u) == 0; }

size_t esize(const xkv_dims &d) { return d.dtype == XKV_F32 ? 4 : 2; }

// Checks shared by every call that takes dims.  `need_xkv` adds the chunk / rank rules.
xkv_status check_dims(const xkv_dims *d, bool need_xkv, const char *who) {
    if (!d) return fail(XKV_ERR_INVALID_ARG, "%s: dims is NULL", who);
    if (d->batch <= 0 || d->n_q_heads <= 0 || d->n_kv_heads <= 0 || d->ctx_len <= 0)
        return fail(XKV_ERR_INVALID_ARG, "%s: batch, heads and ctx_len must be positive", who);
    if (d->n_q_heads % d->n_kv_heads)
        return fail(XKV_ERR_INVALID_ARG, "%s: n_q_heads %% n_kv_heads != 0", who);
    if (d->n_q_heads / d->n_kv_heads > 16)
        return fail(XKV_ERR_UNSUPPORTED, "%s: more than 16 query heads per KV head", who);
    if (d->head_dim != 64 && d->head_dim != 128)
        return fail(XKV_ERR_UNSUPPORTED, "%s: head_dim must be 64 or 128", who);
    if (d->dtype != XKV_F32 && d->dtype != XKV_BF16)
        return fail(XKV_ERR_INVALID_ARG, "%s: unknown dtype %d", who, d->dtype);
    if (d->batch > 65535 || d->n_kv_heads > 65535)
        return fail(XKV_ERR_UNSUPPORTED, "%s: batch or n_kv_heads above 65535", who);
    if (need_xkv) {
        if (d->chunk <= 0 || d->chunk % 8 || d->ctx_len % d->chunk)
            return fail(XKV_ERR_INVALID_ARG, "%s: chunk must be a positive multiple of 8 "
                        "dividing ctx_len", who);
        if (d->rank_k <= 0 || d->rank_v <= 0 || d->rank_k % 16 || d->rank_v % 16)
            return fail(XKV_ERR_INVALID_ARG, "%s: ranks must be positive multiples of 16", who);
        if (d->rank_k > 1024 || d->rank_v > 1024)
            return fail(XKV_ERR_UNSUPPORTED, "%s: rank above 1024", who);
    }
    return XKV_OK;
}

// The library is built for sm_100a only; check the current device once per device.
xkv_status check_device(const char *who) {
    static int checked[64] = {0};  // 0 unknown, 1 ok, 2 wrong arch
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess)
        return fail(XKV_ERR_CUDA, "%s: cudaGetDevice: %s", who, cudaGetErrorString(e));
    if (dev < 0 || dev >= 64) return XKV_OK;
    if (!checked[dev]) {
        int major = 0, minor = 0;
        cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
        checked[dev] = (major == 10 && minor == 0) ? 1 : 2;
    }
    if (checked[dev] != 1)
        return fail(XKV_ERR_UNSUPPORTED, "%s: needs a compute capability 10.0 device", who);
    return XKV_OK;
}

xkv_status launched(cudaError_t e, const char *who) {
    if (e != cudaSuccess)
        return fail(XKV_ERR_CUDA, "%s: launch failed: %s", who, cudaGetErrorString(e));
    return ok();
}

int64_t n_forced(int64_t nC, int n_sink, int n_recent) {
    int64_t f = 0;
    const int64_t sink = n_sink < nC ? n_sink : nC;
    const int64_t rec_lo = nC - n_recent > sink ? nC - n_recent : sink;
    f = sink + (nC - rec_lo);
    return f;
}

// Split plans of the two attention paths (rows = rows attended per unit).
SplitPlan plan_xkv(const xkv_dims &d, int64_t rows) {
    const int G = d.n_q_heads / d.n_kv_heads;
    const int64_t max_rows = 16384 / G < 1024 ? 16384 / G : 1024;
    return plan_splits(rows, (int64_t)d.batch * d.n_kv_heads, 64, max_rows);
}

SplitPlan plan_rcla(const xkv_dims &d, int64_t rows) {
    // at most 4096 / G rows per split (the logits of a split stay in shared memory), in
    // whole 256-row tiles once a split spans more than one tile
    const int G = d.n_q_heads / d.n_kv_heads;
    int64_t cap = (4096 / G) / 256 * 256;
    if (cap < 256) cap = 256;
    SplitPlan p = plan_splits(rows, (int64_t)d.batch * d.n_kv_heads, 256, cap);
    if (rows > 256) {
        p.rows_per_split = (p.rows_per_split + 255) / 256 * 256;
        p.n_split = (int)((rows + p.rows_per_split - 1) / p.rows_per_split);
    }
    return p;
}

}  // namespace

void xkv::set_last_error(const char *msg) { g_last_error = msg; }

// The switches are read on every call (a host-side lookup; no workspace size depends on
// them), so a process can change them between calls.
bool xkv::env_flag(EnvFlag f) {
    static const char *const names[3] = {"XKV_FORCE_SIMT", "XKV_NO_TC", "XKV_NO_PDL"};
    return getenv(names[(int)f]) != nullptr;
}

extern "C" {

const char *xkv_last_error(void) { return g_last_error.c_str(); }

int64_t xkv_n_selected(int64_t n_chunks, int32_t top_k, int32_t n_sink, int32_t n_recent) {
    if (n_chunks < 0 || top_k < 0 || n_sink < 0 || n_recent < 0) return -1;
    const int64_t f = n_forced(n_chunks, n_sink, n_recent);
    const int64_t cand = n_chunks - f;
    return (top_k < cand ? top_k : cand) + f;
}

size_t xkv_workspace_bytes(const xkv_dims *dims, int32_t n_sel, int32_t mode) {
    if (mode == XKV_MODE_RCLA) {
        if (check_dims(dims, false, "xkv_workspace_bytes") != XKV_OK) return 0;
        return ws_header_bytes(*dims) +
               partial_bytes(*dims, (int)plan_rcla(*dims, dims->ctx_len).n_bound);
    }
    if (check_dims(dims, true, "xkv_workspace_bytes") != XKV_OK) return 0;
    if (mode == XKV_MODE_REASSOC) {
        const int64_t nC = dims->ctx_len / dims->chunk;
        if (n_sel < 0 || n_sel > nC || !attend_ra_shape_ok(*dims)) return 0;
        return ws_header_bytes(*dims) +
               ra_call_scratch_bytes(*dims, n_sel == 0, n_sel ? n_sel : (int)nC);
    }
    int64_t rows;
    if (mode == XKV_MODE_SELECTIVE) {
        if (n_sel <= 0 || (int64_t)n_sel > dims->ctx_len / dims->chunk) return 0;
        rows = (int64_t)n_sel * dims->chunk;
    } else if (mode == XKV_MODE_DENSE) {
        rows = dims->ctx_len;
    } else {
        return 0;
    }
    int64_t n = plan_xkv(*dims, rows).n_bound;
    if (attend_tc_shape_ok(*dims)) {
        const int n_tc = tc_splits(*dims, (int)(rows / dims->chunk));
        if (n_tc > n) n = n_tc;
    }
    return ws_header_bytes(*dims) + partial_bytes(*dims, (int)n);
}

int64_t xkv_footprint_bytes(const xkv_dims *d, int32_t n_layers, int32_t window,
                            int32_t with_landmarks) {
    if (check_dims(d, true, "xkv_footprint_bytes") != XKV_OK || n_layers <= 0 || window <= 0)
        return -1;
    const int64_t e = (int64_t)esize(*d);
    const int64_t n_win = (n_layers + window - 1) / window;
    const int64_t d_kv = (int64_t)d->n_kv_heads * d->head_dim;
    const int64_t r = (int64_t)d->rank_k + d->rank_v;
    int64_t per_seq = n_win * d->ctx_len * r * e + (int64_t)n_layers * r * d_kv * e;
    if (with_landmarks) per_seq += (int64_t)n_layers * (d->ctx_len / d->chunk) * d_kv * e;
    return (int64_t)d->batch * per_seq;
}

int64_t rcla_cache_bytes(const xkv_dims *d, int32_t n_leaders, int64_t L_max) {
    if (check_dims(d, false, "rcla_cache_bytes") != XKV_OK || n_leaders <= 0 || L_max <= 0)
        return -1;
    return (int64_t)n_leaders * d->batch * d->n_kv_heads * L_max * d->head_dim * 2 *
           (int64_t)esize(*d);
}

xkv_status xkv_build_landmarks(const xkv_dims *dims, const void *Ak_win, const void *Bkt_layer,
                               void *lm_layer, void *stream) {
    Range nvtx_range("xkv_build_landmarks");
    const char *who = "xkv_build_landmarks";
    xkv_status st;
    if ((st = check_dims(dims, true, who)) != XKV_OK) return st;
    if (!Ak_win || !Bkt_layer || !lm_layer)
        return fail(XKV_ERR_INVALID_ARG, "%s: NULL tensor pointer", who);
    if (!aligned16(Ak_win) || !aligned16(Bkt_layer) || !aligned16(lm_layer))
        return fail(XKV_ERR_INVALID_ARG, "%s: pointers must be 16-byte aligned", who);
    if (dims->ctx_len / dims->chunk > (int64_t)65535 * 16)
        return fail(XKV_ERR_UNSUPPORTED, "%s: too many chunks", who);
    if (injected(who, &st)) return st;
    if ((st = check_device(who)) != XKV_OK) return st;
    return launched(launch_build_landmarks(*dims, Ak_win, Bkt_layer, lm_layer,
                                           (cudaStream_t)stream), who);
}

xkv_status xkv_score_landmarks(const xkv_dims *dims, const void *lm_layer, const void *q,
                               double *scores, void *stream) {
    Range nvtx_range("xkv_score_landmarks");
    const char *who = "xkv_score_landmarks";
    xkv_status st;
    if ((st = check_dims(dims, true, who)) != XKV_OK) return st;
    if (!lm_layer || !q || !scores)
        return fail(XKV_ERR_INVALID_ARG, "%s: NULL tensor pointer", who);
    if (!aligned16(lm_layer) || !aligned16(q) || !aligned16(scores))
        return fail(XKV_ERR_INVALID_ARG, "%s: pointers must be 16-byte aligned", who);
    if (dims->ctx_len / dims->chunk > (int64_t)65535 * 128)
        return fail(XKV_ERR_UNSUPPORTED, "%s: too many chunks", who);
    if (injected(who, &st)) return st;
    if ((st = check_device(who)) != XKV_OK) return st;
    return launched(launch_score(*dims, lm_layer, q, scores, (cudaStream_t)stream), who);
}

xkv_status xkv_select_chunks(const xkv_dims *dims, const double *scores, int32_t top_k,
                             int32_t n_sink, int32_t n_recent, int32_t *sel,
                             int32_t *n_sel_out, void *stream) {
    Range nvtx_range("xkv_select_chunks");
    const char *who = "xkv_select_chunks";
    xkv_status st;
    if ((st = check_dims(dims, true, who)) != XKV_OK) return st;
    if (!scores || !sel) return fail(XKV_ERR_INVALID_ARG, "%s: NULL tensor pointer", who);
    if (!aligned16(scores) || !aligned16(sel))
        return fail(XKV_ERR_INVALID_ARG, "%s: pointers must be 16-byte aligned", who);
    if (top_k < 0 || n_sink < 0 || n_recent < 0)
        return fail(XKV_ERR_INVALID_ARG, "%s: top_k, n_sink, n_recent must be >= 0", who);
    const int64_t nC = dims->ctx_len / dims->chunk;
    if (nC > 16384)
        return fail(XKV_ERR_UNSUPPORTED, "%s: more than 16384 chunks per unit", who);
    const int64_t n_sel = xkv_n_selected(nC, top_k, n_sink, n_recent);
    if (n_sel_out) *n_sel_out = (int32_t)n_sel;
    if (injected(who, &st)) return st;
    if ((st = check_device(who)) != XKV_OK) return st;
    return launched(launch_select(*dims, scores, top_k, n_sink, n_recent, sel, (int)n_sel,
                                  (cudaStream_t)stream), who);
}

size_t xkv_score_select_workspace_bytes(const xkv_dims *dims) {
    if (check_dims(dims, true, "xkv_score_select_workspace_bytes") != XKV_OK) return 0;
    return score_select_ws_bytes(*dims);
}

int64_t xkv_n_reserved(int64_t n_chunks, int32_t n_value, int32_t n_sink, int32_t n_recent) {
    if (n_chunks < 0 || n_value < 0 || n_sink < 0 || n_recent < 0) return -1;
    const int64_t cand = n_chunks - n_forced(n_chunks, n_sink, n_recent);
    return n_value < cand ? n_value : cand;
}

xkv_status xkv_build_value_ranges(const xkv_dims *dims, const void *Av_win,
                                  const void *Bvt_layer, float *rho_layer, unsigned *status,
                                  void *stream) {
    Range nvtx_range("xkv_build_value_ranges");
    const char *who = "xkv_build_value_ranges";
    xkv_status st;
    if ((st = check_dims(dims, true, who)) != XKV_OK) return st;
    if (!Av_win || !Bvt_layer || !rho_layer)
        return fail(XKV_ERR_INVALID_ARG, "%s: NULL tensor pointer", who);
    if (!aligned16(Av_win) || !aligned16(Bvt_layer) || !aligned16(rho_layer) ||
        (status && ((uintptr_t)status & 3u)))
        return fail(XKV_ERR_INVALID_ARG, "%s: pointers must be 16-byte aligned (status: 4)",
                    who);
    const int64_t nC = dims->ctx_len / dims->chunk;
    if (nC > (int64_t)1 << 31 || (int64_t)dims->batch * dims->ctx_len >= ((int64_t)1 << 31))
        return fail(XKV_ERR_UNSUPPORTED, "%s: too many rows", who);
    if (injected(who, &st)) return st;
    if ((st = check_device(who)) != XKV_OK) return st;
    cudaStream_t s = (cudaStream_t)stream;
    const bool tc = dims->dtype == XKV_BF16 && tma_available();
    cudaError_t e = cudaSuccess;
    if (status) e = cudaMemsetAsync(status, 0, sizeof(unsigned), s);
    if (e == cudaSuccess && tc)   // the tensor-core epilogue folds chunks in with atomicMax
        e = cudaMemsetAsync(rho_layer, 0, (size_t)dims->batch * dims->n_kv_heads * nC * 4, s);
    if (e != cudaSuccess) return launched(e, who);
    GemmDesc g{};
    g.mode = GM_VRANGE;
    g.tc = tc;
    g.M = (int)dims->ctx_len;
    g.N = dims->n_kv_heads * dims->head_dim;
    g.nb = dims->batch;
    g.nl = 1;
    g.n_seg = 1;
    g.P = 1;
    g.K_seg = dims->rank_v;
    g.A = Av_win;
    g.B0 = Bvt_layer;
    g.L = dims->ctx_len;
    g.dk = g.N;
    g.r = dims->rank_v;
    g.n_rows = g.N;
    g.W = 1;
    g.status = status;
    g.rho = rho_layer;
    g.hd = dims->head_dim;
    g.chunk = dims->chunk;
    g.Hkv = dims->n_kv_heads;
    g.nC = nC;
    return launched(launch_gemm(g, s), who);
}

xkv_status xkv_reserve_value_chunks(const xkv_dims *dims, const float *rho_layer,
                                    int32_t n_value, int32_t n_sink, int32_t n_recent,
                                    int32_t *reserved, int32_t *n_res_out, void *stream) {
    Range nvtx_range("xkv_reserve_value_chunks");
    const char *who = "xkv_reserve_value_chunks";
    xkv_status st;
    if ((st = check_dims(dims, true, who)) != XKV_OK) return st;
    if (n_value < 0 || n_sink < 0 || n_recent < 0)
        return fail(XKV_ERR_INVALID_ARG, "%s: n_value, n_sink, n_recent must be >= 0", who);
    const int64_t nC = dims->ctx_len / dims->chunk;
    if (nC > 16384)
        return fail(XKV_ERR_UNSUPPORTED, "%s: more than 16384 chunks per unit", who);
    const int64_t n_res = xkv_n_reserved(nC, n_value, n_sink, n_recent);
    if (!rho_layer || (n_res > 0 && !reserved))
        return fail(XKV_ERR_INVALID_ARG, "%s: NULL tensor pointer", who);
    if (!aligned16(rho_layer) || (reserved && !aligned16(reserved)))
        return fail(XKV_ERR_INVALID_ARG, "%s: pointers must be 16-byte aligned", who);
    if (n_res_out) *n_res_out = (int32_t)n_res;
    if (injected(who, &st)) return st;
    if ((st = check_device(who)) != XKV_OK) return st;
    if (n_res == 0) return ok();
    return launched(launch_reserve(*dims, rho_layer, (int)n_res, n_sink, n_recent, reserved,
                                   (cudaStream_t)stream),
                    who);
}

xkv_status xkv_score_select(const xkv_dims *dims, const void *lm_layer, const void *q,
                            int32_t top_k, int32_t n_sink, int32_t n_recent,
                            const int32_t *reserved, int32_t n_reserved, int32_t *sel,
                            int32_t *n_sel_out, void *ws, size_t ws_bytes, void *stream) {
    Range nvtx_range("xkv_score_select");
    const char *who = "xkv_score_select";
    xkv_status st;
    if ((st = check_dims(dims, true, who)) != XKV_OK) return st;
    if (!lm_layer || !q || !sel || !ws || (n_reserved > 0 && !reserved))
        return fail(XKV_ERR_INVALID_ARG, "%s: NULL tensor pointer", who);
    if (!aligned16(lm_layer) || !aligned16(q) || !aligned16(sel) || !aligned16(ws) ||
        (n_reserved > 0 && !aligned16(reserved)))
        return fail(XKV_ERR_INVALID_ARG, "%s: pointers must be 16-byte aligned", who);
    if (top_k < 0 || n_sink < 0 || n_recent < 0 || n_reserved < 0)
        return fail(XKV_ERR_INVALID_ARG, "%s: top_k, n_sink, n_recent, n_reserved must be >= 0",
                    who);
    const int64_t nC = dims->ctx_len / dims->chunk;
    if (nC > 16384)
        return fail(XKV_ERR_UNSUPPORTED, "%s: more than 16384 chunks per unit", who);
    const int64_t n_base = n_forced(nC, n_sink, n_recent);
    if (n_reserved > nC - n_base)
        return fail(XKV_ERR_INVALID_ARG, "%s: more reserved chunks than chunks outside the sink "
                    "and recent windows", who);
    if (!score_select_shape_ok(*dims))
        return fail(XKV_ERR_UNSUPPORTED, "%s: G = n_q_heads / n_kv_heads must be 1..8 or 16",
                    who);
    const size_t need = score_select_ws_bytes(*dims);
    if (ws_bytes < need)
        return fail(XKV_ERR_INVALID_ARG, "%s: workspace %zu bytes, need %zu", who, ws_bytes,
                    need);
    const int64_t rest = nC - n_base - n_reserved;
    const int64_t n_sel = n_base + n_reserved + (top_k < rest ? top_k : rest);
    if (n_sel_out) *n_sel_out = (int32_t)n_sel;
    if (injected(who, &st)) return st;
    if ((st = check_device(who)) != XKV_OK) return st;
    return launched(launch_score_select(*dims, lm_layer, q, top_k, n_sink, n_recent,
                                        n_reserved > 0 ? reserved : nullptr, n_reserved, sel,
                                        (int)n_sel, ws, (cudaStream_t)stream),
                    who);
}

}  // extern "C"

namespace {
xkv_status check_factorize(const xkv_dims *d, int32_t window, int32_t rank, const char *who) {
    if (!d) return fail(XKV_ERR_INVALID_ARG, "%s: dims is NULL", who);
    if (d->batch <= 0 || d->n_kv_heads <= 0 || d->ctx_len <= 0)
        return fail(XKV_ERR_INVALID_ARG, "%s: batch, n_kv_heads and ctx_len must be positive",
                    who);
    if (d->head_dim != 64 && d->head_dim != 128)
        return fail(XKV_ERR_UNSUPPORTED, "%s: head_dim must be 64 or 128", who);
    if (d->dtype != XKV_F32 && d->dtype != XKV_BF16)
        return fail(XKV_ERR_INVALID_ARG, "%s: unknown dtype %d", who, d->dtype);
    if (window < 1) return fail(XKV_ERR_INVALID_ARG, "%s: window must be >= 1", who);
    const int64_t n = (int64_t)window * d->n_kv_heads * d->head_dim;
    if (rank < 16 || rank % 16)
        return fail(XKV_ERR_INVALID_ARG, "%s: rank must be a positive multiple of 16", who);
    if (rank > 1024) return fail(XKV_ERR_UNSUPPORTED, "%s: rank above 1024", who);
    if (rank > d->ctx_len || rank > n)
        return fail(XKV_ERR_INVALID_ARG, "%s: rank above min(ctx_len, window * d_kv)", who);
    if (d->ctx_len > (1 << 24) || n > (1 << 24) || d->batch > 65535)
        return fail(XKV_ERR_UNSUPPORTED, "%s: ctx_len, window * d_kv or batch too large", who);
    return XKV_OK;
}
}  // namespace

extern "C" {

size_t xkv_refold_workspace_bytes(const xkv_dims *dims, int32_t window, int32_t rank,
                                  int64_t n_tail) {
    if (check_factorize(dims, window, rank, "xkv_refold_workspace_bytes") != XKV_OK ||
        n_tail < 0 || dims->ctx_len + n_tail > (1 << 24))
        return 0;
    return refold_ws_bytes(*dims, window, rank, n_tail);
}

xkv_status xkv_refold_window(const xkv_dims *dims, int32_t window, int32_t rank,
                             const void *A_win, const void *Bt_win, const void *tail,
                             int64_t n_tail, const float *omega, int32_t n_iter, void *A_out,
                             void *Bt_out, void *ws, size_t ws_bytes, void *stream) {
    Range nvtx_range("xkv_refold_window");
    const char *who = "xkv_refold_window";
    xkv_status st;
    if ((st = check_factorize(dims, window, rank, who)) != XKV_OK) return st;
    if (n_tail < 0 || dims->ctx_len + n_tail > (1 << 24))
        return fail(XKV_ERR_INVALID_ARG, "%s: need 0 <= n_tail and ctx_len + n_tail <= 2^24",
                    who);
    if (n_iter < 0 || n_iter > 16)
        return fail(XKV_ERR_INVALID_ARG, "%s: n_iter must be in [0, 16]", who);
    if (!A_win || !Bt_win || (n_tail > 0 && !tail) || !omega || !A_out || !Bt_out || !ws)
        return fail(XKV_ERR_INVALID_ARG, "%s: NULL pointer", who);
    if (!aligned16(A_win) || !aligned16(Bt_win) || (n_tail > 0 && !aligned16(tail)) ||
        !aligned16(omega) || !aligned16(A_out) || !aligned16(Bt_out) || !aligned16(ws))
        return fail(XKV_ERR_INVALID_ARG, "%s: pointers must be 16-byte aligned", who);
    const size_t need = refold_ws_bytes(*dims, window, rank, n_tail);
    if (ws_bytes < need)
        return fail(XKV_ERR_INVALID_ARG, "%s: workspace %zu bytes, need %zu", who, ws_bytes,
                    need);
    if (injected(who, &st)) return st;
    if ((st = check_device(who)) != XKV_OK) return st;
    return launched(launch_refold(*dims, window, rank, A_win, Bt_win, tail, n_tail, omega,
                                  n_iter, A_out, Bt_out, ws, (cudaStream_t)stream),
                    who);
}

size_t xkv_factorize_workspace_bytes(const xkv_dims *dims, int32_t window, int32_t rank) {
    if (check_factorize(dims, window, rank, "xkv_factorize_workspace_bytes") != XKV_OK) return 0;
    return factorize_ws_bytes(*dims, window, rank);
}

xkv_status xkv_factorize_window(const xkv_dims *dims, int32_t window, int32_t rank,
                                const void *X, const float *omega, int32_t n_iter,
                                void *A_out, void *Bt_out, void *ws, size_t ws_bytes,
                                void *stream) {
    Range nvtx_range("xkv_factorize_window");
    const char *who = "xkv_factorize_window";
    xkv_status st;
    if ((st = check_factorize(dims, window, rank, who)) != XKV_OK) return st;
    if (n_iter < 0 || n_iter > 16)
        return fail(XKV_ERR_INVALID_ARG, "%s: n_iter must be in [0, 16]", who);
    if (!X || !omega || !A_out || !Bt_out || !ws)
        return fail(XKV_ERR_INVALID_ARG, "%s: NULL pointer", who);
    if (!aligned16(X) || !aligned16(omega) || !aligned16(A_out) || !aligned16(Bt_out) ||
        !aligned16(ws))
        return fail(XKV_ERR_INVALID_ARG, "%s: pointers must be 16-byte aligned", who);
    const size_t need = factorize_ws_bytes(*dims, window, rank);
    if (ws_bytes < need)
        return fail(XKV_ERR_INVALID_ARG, "%s: workspace %zu bytes, need %zu", who, ws_bytes,
                    need);
    if (injected(who, &st)) return st;
    if ((st = check_device(who)) != XKV_OK) return st;
    return launched(launch_factorize(*dims, window, rank, X, omega, n_iter, A_out, Bt_out, ws,
                                     (cudaStream_t)stream),
                    who);
}

}  // extern "C"

namespace {

// Splits the tail of generated tokens adds to an attention call (0 without a tail).
int64_t tail_bound(const xkv_dims &d, int64_t T_max) {
    return T_max > 0 ? plan_rcla(d, T_max).n_bound : 0;
}

}  // namespace

// Host-side checks of a reconstruct-then-attend call: every argument rule, then the
// scratch the call needs (*need_out) against ws_bytes -- the caller's workspace when
// check_ws is set, else the size of the library's own fixed array (the allocation-free
// entry point: ws is not checked, a larger need is XKV_ERR_UNSUPPORTED).  Then the
// injected fault of `who`, then the device.  Nothing here launches.
xkv_status xkv::attend_validate(const char *who, const xkv_dims *dims, const void *Ak_win,
                           const void *Av_win, const void *Bkt_layer, const void *Bvt_layer,
                           const void *q, const int32_t *sel, int32_t n_sel,
                           const void *K_tail, const void *V_tail, int64_t T_max,
                           int64_t n_tail, const float *out, const void *ws, size_t ws_bytes,
                           bool check_ws, size_t *need_out) {
    xkv_status st;
    if ((st = check_dims(dims, true, who)) != XKV_OK) return st;
    if (!Ak_win || !Av_win || !Bkt_layer || !Bvt_layer || !q || !out || (check_ws && !ws))
        return fail(XKV_ERR_INVALID_ARG, "%s: NULL tensor pointer", who);
    if (!aligned16(Ak_win) || !aligned16(Av_win) || !aligned16(Bkt_layer) ||
        !aligned16(Bvt_layer) || !aligned16(q) || !aligned16(out) ||
        (check_ws && !aligned16(ws)) || (sel && !aligned16(sel)))
        return fail(XKV_ERR_INVALID_ARG, "%s: pointers must be 16-byte aligned", who);
    const int64_t nC = dims->ctx_len / dims->chunk;
    if (sel && (n_sel <= 0 || n_sel > nC))
        return fail(XKV_ERR_INVALID_ARG, "%s: n_sel must be in [1, n_chunks]", who);
    if (T_max < 0 || n_tail < 0 || n_tail > T_max)
        return fail(XKV_ERR_INVALID_ARG, "%s: need 0 <= n_tail <= T_max", who);
    if (n_tail > 0 && (!K_tail || !V_tail || !aligned16(K_tail) || !aligned16(V_tail)))
        return fail(XKV_ERR_INVALID_ARG, "%s: tail pointers must be 16-byte aligned", who);
    const int64_t rows = sel ? (int64_t)n_sel * dims->chunk : dims->ctx_len;
    const SplitPlan plan = plan_xkv(*dims, rows);
    const int n_tc = attend_tc_shape_ok(*dims) ? tc_splits(*dims, (int)(rows / dims->chunk)) : 0;
    const int64_t n_att = n_tc > plan.n_bound ? n_tc : plan.n_bound;
    const int64_t n_tail_bound = tail_bound(*dims, T_max);
    if (plan.n_split > 65535 || n_tc > 65535 || n_att + n_tail_bound > 65535)
        return fail(XKV_ERR_UNSUPPORTED, "%s: too many rows", who);
    // the same amount xkv_workspace_bytes / xkv_tail_workspace_bytes report, whichever
    // kernel runs
    const size_t need = ws_header_bytes(*dims) + partial_bytes(*dims, (int)(n_att + n_tail_bound));
    if (need_out) *need_out = need;
    if (check_ws && ws_bytes < need)
        return fail(XKV_ERR_INVALID_ARG, "%s: workspace %zu bytes, need %zu", who, ws_bytes,
                    need);
    if (!check_ws && need > ws_bytes)
        return fail(XKV_ERR_UNSUPPORTED,
                    "%s: this call needs %zu bytes of scratch, above the fixed %zu-byte array; "
                    "use xkv_reconstruct_attend with a caller-provided workspace",
                    who, need, ws_bytes);
    if (injected(who, &st)) return st;
    return check_device(who);
}

// Reconstruct-then-attend over the selected (or all) rows of the window, plus, when
// n_tail > 0, the first n_tail rows of an uncompressed tail K_tail / V_tail
// [B][Hkv][T_max][hd]: the attention kernel writes its splits, the R-CLA kernel writes
// the tail's splits after them, and one combine merges all of them.  The arguments were
// checked by attend_validate; ws holds at least the scratch it reported.
xkv_status xkv::attend_launch(const char *who, const xkv_dims *dims, const void *Ak_win,
                         const void *Av_win, const void *Bkt_layer, const void *Bvt_layer,
                         const void *q, const int32_t *sel, int32_t n_sel, const void *K_tail,
                         const void *V_tail, int64_t T_max, int64_t n_tail, float *out,
                         void *ws, void *stream) {
    const int64_t rows = sel ? (int64_t)n_sel * dims->chunk : dims->ctx_len;
    const SplitPlan plan = plan_xkv(*dims, rows);
    const int n_tc = attend_tc_shape_ok(*dims) ? tc_splits(*dims, (int)(rows / dims->chunk)) : 0;
    const bool use_tc = n_tc > 0 && attend_tc_supported(*dims) && !env_flag(ENV_FORCE_SIMT);
    cudaStream_t s = (cudaStream_t)stream;
    const size_t hdr = ws_header_bytes(*dims);
    unsigned *status = (unsigned *)ws;
    float *partials = (float *)((char *)ws + hdr);
    // device-side errors of this call (timeouts, selections out of range) are OR-ed
    // into the status word; the combine kernel turns a non-zero word into NaN outputs
    cudaError_t e = launch_clear_status(status, s);
    if (e != cudaSuccess) return launched(e, who);
    int used = 0;
    if (use_tc) {
        used = n_tc;
        e = launch_attend_tc(*dims, Ak_win, Av_win, Bkt_layer, Bvt_layer, q, sel,
                             sel ? n_sel : (int)(dims->ctx_len / dims->chunk), partials, status,
                             &used, s);
    } else {
        used = plan.n_split;
        e = launch_attend_simt(*dims, Ak_win, Av_win, Bkt_layer, Bvt_layer, q, sel, n_sel, plan,
                               partials, status, s);
    }
    if (e == cudaSuccess && n_tail > 0) {
        const SplitPlan tp = plan_rcla(*dims, n_tail);
        float *tail_partials = partials + (size_t)used * dims->batch * dims->n_q_heads *
                                              (dims->head_dim + 2);
        e = launch_rcla(*dims, 0, T_max, n_tail, -1, const_cast<void *>(K_tail),
                        const_cast<void *>(V_tail), nullptr, nullptr, q, tp, tail_partials, s);
        used += tp.n_split;
    }
    if (e == cudaSuccess) e = launch_combine(*dims, used, partials, out, status, s);
    return launched(e, who);
}

namespace {

xkv_status attend_impl(const char *who, const xkv_dims *dims, const void *Ak_win,
                       const void *Av_win, const void *Bkt_layer, const void *Bvt_layer,
                       const void *q, const int32_t *sel, int32_t n_sel, const void *K_tail,
                       const void *V_tail, int64_t T_max, int64_t n_tail, float *out, void *ws,
                       size_t ws_bytes, void *stream) {
    const xkv_status st = attend_validate(who, dims, Ak_win, Av_win, Bkt_layer, Bvt_layer, q,
                                          sel, n_sel, K_tail, V_tail, T_max, n_tail, out, ws,
                                          ws_bytes, true, nullptr);
    if (st != XKV_OK) return st;
    return attend_launch(who, dims, Ak_win, Av_win, Bkt_layer, Bvt_layer, q, sel, n_sel, K_tail,
                         V_tail, T_max, n_tail, out, ws, stream);
}

}  // namespace

extern "C" {

xkv_status xkv_reconstruct_attend(const xkv_dims *dims, const void *Ak_win, const void *Av_win,
                                  const void *Bkt_layer, const void *Bvt_layer, const void *q,
                                  const int32_t *sel, int32_t n_sel, float *out, void *ws,
                                  size_t ws_bytes, void *stream) {
    Range nvtx_range("xkv_reconstruct_attend");
    return attend_impl("xkv_reconstruct_attend", dims, Ak_win, Av_win, Bkt_layer, Bvt_layer, q,
                       sel, n_sel, nullptr, nullptr, 0, 0, out, ws, ws_bytes, stream);
}

xkv_status xkv_reconstruct_attend_tail(const xkv_dims *dims, const void *Ak_win,
                                       const void *Av_win, const void *Bkt_layer,
                                       const void *Bvt_layer, const void *q,
                                       const int32_t *sel, int32_t n_sel, const void *K_tail,
                                       const void *V_tail, int64_t T_max, int64_t n_tail,
                                       float *out, void *ws, size_t ws_bytes, void *stream) {
    Range nvtx_range("xkv_reconstruct_attend_tail");
    if (T_max <= 0)
        return fail(XKV_ERR_INVALID_ARG, "xkv_reconstruct_attend_tail: T_max must be positive");
    return attend_impl("xkv_reconstruct_attend_tail", dims, Ak_win, Av_win, Bkt_layer, Bvt_layer,
                       q, sel, n_sel, K_tail, V_tail, T_max, n_tail, out, ws, ws_bytes, stream);
}

size_t xkv_tail_workspace_bytes(const xkv_dims *dims, int32_t n_sel, int64_t T_max) {
    if (T_max <= 0) return 0;
    const size_t base = xkv_workspace_bytes(dims, n_sel,
                                            n_sel > 0 ? XKV_MODE_SELECTIVE : XKV_MODE_DENSE);
    if (!base) return 0;
    return base + partial_bytes(*dims, (int)tail_bound(*dims, T_max));
}

xkv_status xkv_reassociated_attend(const xkv_dims *dims, const void *Ak_win, const void *Av_win,
                                   const void *Bkt_layer, const void *Bvt_layer, const void *q,
                                   const int32_t *sel, int32_t n_sel, float *out, void *ws,
                                   size_t ws_bytes, void *stream) {
    Range nvtx_range("xkv_reassociated_attend");
    const char *who = "xkv_reassociated_attend";
    xkv_status st;
    if ((st = check_dims(dims, true, who)) != XKV_OK) return st;
    if (!Ak_win || !Av_win || !Bkt_layer || !Bvt_layer || !q || !out || !ws)
        return fail(XKV_ERR_INVALID_ARG, "%s: NULL tensor pointer", who);
    if (!aligned16(Ak_win) || !aligned16(Av_win) || !aligned16(Bkt_layer) ||
        !aligned16(Bvt_layer) || !aligned16(q) || !aligned16(out) || !aligned16(ws) ||
        (sel && !aligned16(sel)))
        return fail(XKV_ERR_INVALID_ARG, "%s: pointers must be 16-byte aligned", who);
    const int64_t nC = dims->ctx_len / dims->chunk;
    if (sel && (n_sel <= 0 || n_sel > nC))
        return fail(XKV_ERR_INVALID_ARG, "%s: n_sel must be in [1, n_chunks]", who);
    if (!attend_ra_shape_ok(*dims))
        return fail(XKV_ERR_UNSUPPORTED, "%s: needs bf16, head_dim 128, G in {1,2,4,5,8}, "
                    "ranks multiple of 128 (r_K <= 1024, or 512 when G > 4; r_V <= 1024) and "
                    "a chunk dividing 256", who);
    const int ns = sel ? n_sel : (int)nC;
    if (ra_splits(*dims, ns) > 65535 || (int64_t)dims->batch * dims->ctx_len >= (1ll << 31))
        return fail(XKV_ERR_UNSUPPORTED, "%s: too many rows", who);
    const size_t need = ws_header_bytes(*dims) + ra_call_scratch_bytes(*dims, !sel, ns);
    if (ws_bytes < need)
        return fail(XKV_ERR_INVALID_ARG, "%s: workspace %zu bytes, need %zu", who, ws_bytes,
                    need);
    if (injected(who, &st)) return st;
    if ((st = check_device(who)) != XKV_OK) return st;
    if (!tma_available()) return fail(XKV_ERR_UNSUPPORTED, "%s: no tensor-map encoder", who);
    cudaStream_t s = (cudaStream_t)stream;
    unsigned *status = (unsigned *)ws;     // cleared by the call's first kernel
    const cudaError_t e = launch_attend_ra(*dims, Ak_win, Av_win, Bkt_layer, Bvt_layer, q, sel,
                                           ns, (char *)ws + ws_header_bytes(*dims), status,
                                           out, s);
    return launched(e, who);
}

xkv_status rcla_decode_attend(const xkv_dims *dims, int32_t layer, const int32_t *leader_of,
                              int32_t n_layers, void *K_lead, void *V_lead, int64_t L_max,
                              int64_t len, const void *k_new, const void *v_new, const void *q,
                              float *out, void *ws, size_t ws_bytes, void *stream) {
    Range nvtx_range("rcla_decode_attend");
    const char *who = "rcla_decode_attend";
    xkv_status st;
    if ((st = check_dims(dims, false, who)) != XKV_OK) return st;
    if (!leader_of || !K_lead || !V_lead || !q || !out || !ws)
        return fail(XKV_ERR_INVALID_ARG, "%s: NULL pointer", who);
    if (!aligned16(K_lead) || !aligned16(V_lead) || !aligned16(q) || !aligned16(out) ||
        !aligned16(ws) || (k_new && !aligned16(k_new)) || (v_new && !aligned16(v_new)))
        return fail(XKV_ERR_INVALID_ARG, "%s: pointers must be 16-byte aligned", who);
    if (n_layers <= 0 || layer < 0 || layer >= n_layers)
        return fail(XKV_ERR_INVALID_ARG, "%s: layer outside [0, n_layers)", who);
    if (leader_of[0] != 0)
        return fail(XKV_ERR_INVALID_ARG, "%s: layer 0 must be a leader", who);
    int slot = 0, lead = leader_of[layer];
    for (int l = 0; l < n_layers; ++l) {
        const int32_t s = leader_of[l];
        if (s < 0 || s > l || leader_of[s] != s)
            return fail(XKV_ERR_INVALID_ARG, "%s: leader_of[%d] = %d is not an earlier leader",
                        who, l, s);
        if (l < lead && s == l) ++slot;
    }
    const bool is_leader = lead == layer;
    if ((k_new == nullptr) != (v_new == nullptr))
        return fail(XKV_ERR_INVALID_ARG, "%s: give both k_new and v_new or neither", who);
    if (!is_leader && k_new)
        return fail(XKV_ERR_INVALID_ARG, "%s: layer %d is not a leader and owns no cache", who,
                    layer);
    const bool update = is_leader && k_new;
    const int64_t n_rows = len + (update ? 1 : 0);
    if (len < 0 || L_max <= 0 || n_rows > L_max || n_rows <= 0)
        return fail(XKV_ERR_INVALID_ARG, "%s: need 0 < rows attended <= L_max", who);
    const SplitPlan plan = plan_rcla(*dims, n_rows);
    if (plan.n_split > 65535) return fail(XKV_ERR_UNSUPPORTED, "%s: too many rows", who);
    const size_t need = ws_header_bytes(*dims) + partial_bytes(*dims, plan.n_split);
    if (ws_bytes < need)
        return fail(XKV_ERR_INVALID_ARG, "%s: workspace %zu bytes, need %zu", who, ws_bytes,
                    need);
    if (injected(who, &st)) return st;
    if ((st = check_device(who)) != XKV_OK) return st;
    cudaStream_t s = (cudaStream_t)stream;
    float *partials = (float *)((char *)ws + ws_header_bytes(*dims));
    cudaError_t e = launch_rcla(*dims, slot, L_max, n_rows, update ? len : -1, K_lead, V_lead,
                                k_new, v_new, q, plan, partials, s);
    if (e == cudaSuccess) e = launch_combine(*dims, plan.n_split, partials, out, nullptr, s);
    return launched(e, who);
}

}  // extern "C"
