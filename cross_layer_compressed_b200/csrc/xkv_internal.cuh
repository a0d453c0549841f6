// Internal declarations shared by the kernels and the C-ABI layer of the xKV decode
// library.  Nothing here is part of the public ABI (include/xkv.h is).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <stdlib.h>

#include "xkv.h"

namespace xkv {

// ------------------------------------------------------------------ launch plans
// Work split of one attention call: `n_split` CTAs per (sequence, KV head) unit, each
// over a contiguous range of the unit's rows.  Partials go to the workspace as
// [n_split][B][Hq][hd + 2] fp32 = (running max m, sum l, unnormalised acc[hd]).
struct SplitPlan {
    int n_split;             // CTAs per unit (no split is empty)
    int64_t rows_per_split;
    int64_t n_bound;         // >= n_split and nondecreasing in `rows`: sizes workspaces
};

// A workspace sized with n_bound for the largest row count fits every smaller call.
SplitPlan plan_splits(int64_t rows, int64_t units, int64_t min_rows, int64_t max_rows);

size_t partial_bytes(const xkv_dims &d, int n_split);

// Raises a kernel's dynamic shared-memory limit on the current device only when a call
// needs more than was set before, so steady-state calls (and stream captures) make no
// attribute calls.
cudaError_t set_smem_limit(const void *kernel, size_t bytes);

// ------------------------------------------------------------------ launchers
// Each returns cudaSuccess or the launch error; arguments were validated by the caller.
cudaError_t launch_build_landmarks(const xkv_dims &d, const void *Ak, const void *Bkt, void *lm,
                                   cudaStream_t s);
cudaError_t launch_score(const xkv_dims &d, const void *lm, const void *q, double *scores,
                         cudaStream_t s);
cudaError_t launch_select(const xkv_dims &d, const double *scores, int top_k, int n_sink,
                          int n_recent, int32_t *sel, int n_sel, cudaStream_t s);
// fused scoring + selection (score_select.cu): the selection xkv_select_chunks makes from
// xkv_score_landmarks' scores, with fp32 scores and an fp64 rescore of the uncertain band
bool score_select_shape_ok(const xkv_dims &d);   // G in 1..8 or 16
size_t score_select_ws_bytes(const xkv_dims &d);
cudaError_t launch_score_select(const xkv_dims &d, const void *lm, const void *q, int top_k,
                                int n_sink, int n_recent, const int32_t *reserved, int n_res,
                                int32_t *sel, int n_sel, void *ws, cudaStream_t s);
// value-range reservation: per (b, g) the n_res candidates of largest rho, ascending
cudaError_t launch_reserve(const xkv_dims &d, const float *rho, int n_res, int n_sink,
                           int n_recent, int32_t *reserved, cudaStream_t s);
cudaError_t launch_attend_simt(const xkv_dims &d, const void *Ak, const void *Av,
                               const void *Bkt, const void *Bvt, const void *q,
                               const int32_t *sel, int n_sel, const SplitPlan &plan,
                               float *partials, unsigned *status, cudaStream_t s);
cudaError_t launch_rcla(const xkv_dims &d, int slot, int64_t L_max, int64_t n_rows,
                        int64_t update_row, void *K, void *V, const void *k_new,
                        const void *v_new, const void *q, const SplitPlan &plan,
                        float *partials, cudaStream_t s);
// R-CLA on the tensor cores (bf16, head_dim 128, G in {1, 2, 4, 5, 8}, splits of at most
// 1024 rows); launch_rcla picks it when rcla_tc_ok holds
bool rcla_tc_ok(const xkv_dims &d, int slot, int64_t L_max, const SplitPlan &plan);
cudaError_t launch_rcla_tc(const xkv_dims &d, int slot, int64_t L_max, int64_t n_rows,
                           int64_t update_row, void *K, void *V, const void *k_new,
                           const void *v_new, const void *q, const SplitPlan &plan,
                           float *partials, cudaStream_t s);
int sm_count();   // multiprocessors of the current device (cached)
bool tma_available();   // the driver exposes the tensor-map encoder
// reassociated attention (rank-space logits and values, tcgen05)
bool attend_ra_shape_ok(const xkv_dims &d);
int ra_splits(const xkv_dims &d, int n_sel);
size_t ra_scratch_bytes(const xkv_dims &d, int n_split);
// scratch of one reassociated call: dense (no selection) or n_sel selected chunks
size_t ra_call_scratch_bytes(const xkv_dims &d, bool dense, int n_sel);
bool attend_ra_dense_heads(const xkv_dims &d);
cudaError_t launch_attend_ra(const xkv_dims &d, const void *Ak, const void *Av, const void *Bkt,
                             const void *Bvt, const void *q, const int32_t *sel, int n_sel,
                             void *scratch, unsigned *status, float *out, cudaStream_t s);
cudaError_t launch_combine(const xkv_dims &d, int n_split, const float *partials, float *out,
                           const unsigned *status, cudaStream_t s);
// tensor-core path (bf16, head_dim 128, ranks multiple of 64, chunk dividing 256)
bool attend_tc_shape_ok(const xkv_dims &d);   // shapes only (sizes workspaces)
bool attend_tc_supported(const xkv_dims &d);  // shapes and a driver with TMA maps
int tc_splits(const xkv_dims &d, int n_sel);
cudaError_t launch_attend_tc(const xkv_dims &d, const void *Ak, const void *Av, const void *Bkt,
                             const void *Bvt, const void *q, const int32_t *sel, int n_sel,
                             float *partials, unsigned *status, int *n_split_out,
                             cudaStream_t s);

// The dense products of the factorization (gemm.cu), batched over sequences (nb) and an
// outer index (nl), each a sum over n_seg K segments of K_seg:
//   GM_XF      C[b]    = sum_s X[s / P][b] F_{s % P}[b][(s / P) d_kv ...]   (Y = X Omega / X Z)
//   GM_XT      C[l][b] = sum_s X[l][b]^T Q_s[b]                             (Z_l = X_l^T Q)
//   GM_APPLY   C[b]    = A[b] (R^-1)[b], B0 holding (R^-1)^T                (Y R^-1)
//   GM_REFOLD  C[l][b] = A[b] Bt[l][b]^T                                    (A B_l)
// tc: bf16 operands (TF32 for GM_APPLY) on the tensor cores; else fp32 on the CUDA cores.
//   GM_VRANGE  rho[b][g][c] = max over chunk c's rows of max - min of A[b] Bt[b]^T's
//              head-g columns (atomicMax into rho, which the caller zeroes)
enum GemmMode { GM_XF = 0, GM_XT = 1, GM_APPLY = 2, GM_REFOLD = 3, GM_VRANGE = 4 };
struct GemmDesc {
    int mode;
    bool tc;
    int M, N, nb, nl, n_seg, P;
    int64_t K_seg;
    const void *A, *B0, *B1;
    int b_shared;                 // GM_XF: F has no batch dimension
    int64_t L, dk, r, n_rows, W;  // rows of X (or of A), d_kv, rank, rows of F, layers
    void *C;
    int c_bf16;                   // C in bf16 (else fp32)
    int64_t ldc, c_b, c_l;        // C strides of a row, a sequence, an outer index
    unsigned *status;             // bits of device-side failures (bounded waits)
    float *rho;                   // GM_VRANGE output [nb][Hkv][nC]
    int hd, chunk, Hkv;
    int64_t nC;
};
cudaError_t launch_gemm(const GemmDesc &g, cudaStream_t s);

// cross-layer factorization of one window (clf.cu)
size_t factorize_ws_bytes(const xkv_dims &d, int W, int r);
cudaError_t launch_factorize(const xkv_dims &d, int W, int r, const void *X, const float *omega,
                             int n_iter, void *A_out, void *Bt_out, void *ws, cudaStream_t s);
// the tail of generated rows folded back: factorization of [A·B_l ; tail_l]
size_t refold_ws_bytes(const xkv_dims &d, int W, int r, int64_t n_tail);
cudaError_t launch_refold(const xkv_dims &d, int W, int r, const void *A, const void *Bt,
                          const void *tail, int64_t n_tail, const float *omega, int n_iter,
                          void *A_out, void *Bt_out, void *ws, cudaStream_t s);

// Clears the workspace status word of a call (a one-thread kernel launched with
// launch_chained, so that it and the attention kernel after it are scheduled while the
// previous kernel of the stream finishes).
cudaError_t launch_clear_status(unsigned *status, cudaStream_t s);

// ------------------------------------------------------------------ chained launches
// Kernels that follow one another in a stream are launched with programmatic dependent
// launch (CUDA 12): a grid so launched may be scheduled as soon as every CTA of the grid
// before it has executed griddepcontrol.launch_dependents (or exited).  Each kernel
// launched this way runs griddepcontrol.wait before it touches global memory that an
// earlier grid writes or reads (setup of shared memory, mbarriers and TMEM may come
// first), and that wait returns once the previous grid has completed and its writes are
// visible; without the launch attribute the wait returns at once.  Setting XKV_NO_PDL in
// the environment launches every kernel in plain stream order.
bool chain_enabled();
template <typename... P, typename... A>
cudaError_t launch_chained(void (*k)(P...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                           A &&...args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = at;
    cfg.numAttrs = chain_enabled() ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, k, static_cast<A &&>(args)...);
}

// Sets the calling thread's xkv_last_error() message (defined with the C ABI layer).
void set_last_error(const char *msg);

// Environment switches (documented in include/xkv.h), read on every call:
// XKV_FORCE_SIMT takes the CUDA-core kernels for both attentions, XKV_NO_TC the TMA +
// CUDA-core R-CLA kernel, XKV_NO_PDL plain stream order for every launch.
enum EnvFlag { ENV_FORCE_SIMT = 0, ENV_NO_TC = 1, ENV_NO_PDL = 2 };
bool env_flag(EnvFlag f);
// A test-only poll limit read from the environment on every call: the variable's value
// when it is a whole decimal number in [0, full), else `full`.  A limit of 0 makes the
// waits it governs give up without polling (mbarrier try_wait may itself suspend for a
// while, so even a limit of 1 can succeed when the data is already close).
inline uint32_t test_poll_limit(const char *name, uint32_t full) {
    const char *e = getenv(name);
    if (!e || !*e) return full;
    char *end = nullptr;
    const long v = strtol(e, &end, 10);
    return (*end == '\0' && v >= 0 && v < (long)full) ? (uint32_t)v : full;
}

// Host-side checks of xkv_reconstruct_attend(_tail) and its launches, shared with the
// allocation-free entry point.  attend_validate checks every argument rule, reports the
// scratch the call needs in *need_out and checks it against ws_bytes (with check_ws: the
// caller's workspace ws, too small = XKV_ERR_INVALID_ARG; without: a fixed array of
// ws_bytes, too small = XKV_ERR_UNSUPPORTED), applies the injected fault of `who` and
// checks the device; it launches nothing.
// attend_launch queues the kernels of a validated call on `stream`, with `ws` holding at
// least that scratch.
xkv_status attend_validate(const char *who, const xkv_dims *dims, const void *Ak_win,
                           const void *Av_win, const void *Bkt_layer, const void *Bvt_layer,
                           const void *q, const int32_t *sel, int32_t n_sel,
                           const void *K_tail, const void *V_tail, int64_t T_max,
                           int64_t n_tail, const float *out, const void *ws, size_t ws_bytes,
                           bool check_ws, size_t *need_out);
xkv_status attend_launch(const char *who, const xkv_dims *dims, const void *Ak_win,
                         const void *Av_win, const void *Bkt_layer, const void *Bvt_layer,
                         const void *q, const int32_t *sel, int32_t n_sel, const void *K_tail,
                         const void *V_tail, int64_t T_max, int64_t n_tail, float *out,
                         void *ws, void *stream);

// Workspace layout: a 256-byte header (word 0: device status bits, 1 << xkv_status) and
// then the partials.
inline size_t ws_header_bytes(const xkv_dims &) { return 256; }

// ------------------------------------------------------------------ device helpers
__host__ __device__ __forceinline__ int64_t min64(int64_t a, int64_t b) { return a < b ? a : b; }
__host__ __device__ __forceinline__ int64_t max64(int64_t a, int64_t b) { return a > b ? a : b; }

// Programmatic dependent launch, device side (see launch_chained).
__device__ __forceinline__ void grid_dep_wait() {
    asm volatile("griddepcontrol.wait;" ::: "memory");
}
__device__ __forceinline__ void grid_dep_launch() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

template <typename T> struct Elem;
template <> struct Elem<float> {
    static __device__ __forceinline__ float f32(float x) { return x; }
    static __device__ __forceinline__ double f64(float x) { return (double)x; }
};
template <> struct Elem<__nv_bfloat16> {
    static __device__ __forceinline__ float f32(__nv_bfloat16 x) { return __bfloat162float(x); }
    static __device__ __forceinline__ double f64(__nv_bfloat16 x) {
        return (double)__bfloat162float(x);  // both widenings are exact
    }
};

// Widen the low / high bf16 of a packed pair to fp32 (exact: a bf16 is the top half of
// an fp32 bit pattern).
__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// Round an fp64 value to the nearest bf16, ties to even, in one step (no fp32 detour).
// Method: round-half-even at bit 45 of the binary64 pattern by adding
// (2^44 - 1) + (bit 45) and truncating, then re-bias the exponent from 1023 to 127.
// Values below the bf16 normal range are first rounded to the fixed subnormal quantum
// 2^-133 (exactly representable in fp64), so the result is exact there too.
__device__ __forceinline__ uint16_t f64_to_bf16_rne(double x) {
    uint64_t u = (uint64_t)__double_as_longlong(x);
    uint64_t sign = u >> 63;
    uint64_t mag = u & 0x7fffffffffffffffull;
    if (mag == 0) return (uint16_t)(sign << 15);
    int e = (int)(mag >> 52) - 1023;  // unbiased exponent (normal fp64 inputs)
    if (e >= 128) return (uint16_t)((sign << 15) | 0x7f80u);  // overflow -> inf
    if (e < -126) {
        // subnormal bf16 range: k = rint(|x| * 2^133), value k * 2^-133, k <= 128
        double k = rint(fabs(x) * 0x1p133);
        uint32_t bits = (uint32_t)k;  // k == 128 is the smallest normal, same encoding
        return (uint16_t)((sign << 15) | bits);
    }
    uint64_t lsb = (mag >> 45) & 1ull;
    mag += 0x00000FFFFFFFFFFFull + lsb;  // 2^44 - 1 + lsb
    int e2 = (int)(mag >> 52) - 1023;
    if (e2 >= 128) return (uint16_t)((sign << 15) | 0x7f80u);
    uint32_t man7 = (uint32_t)((mag >> 45) & 0x7f);
    return (uint16_t)((sign << 15) | ((uint32_t)(e2 + 127) << 7) | man7);
}

// Key under which a larger double compares larger and -0 < +0.
__device__ __forceinline__ unsigned long long order_key(double s) {
    unsigned long long u = (unsigned long long)__double_as_longlong(s);
    return (u >> 63) ? ~u : (u | 0x8000000000000000ull);
}

}  // namespace xkv
