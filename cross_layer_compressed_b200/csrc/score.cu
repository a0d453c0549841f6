// Landmark scoring (xKV page, section 2.3: rank the chunks by the relevance of their
// landmark key to the current query, taking the max over the GQA group).
//
// score[b][g][c] = max_{h in group g} sum_{d < hd} lm[b][g][c][d] * q[b][h][d], with every
// product exact in fp64 and the sum in ascending d, so the value is reproducible bit for
// bit on any IEEE-754 machine.  HBM-bound: one pass over the landmarks.
//
#include "xkv_internal.cuh"

namespace xkv {
namespace {

constexpr int SC_THREADS = 256;
constexpr int SC_CPT = 2;      // chunks per thread: 2G independent fp64 chains
constexpr int SC_MAXG = 16;

// One thread scores SC_CPT chunks (rows c, c + 256 of the CTA's block).  Each row is read
// with 16-byte loads straight from global memory: a warp's 32 rows are one contiguous
// 8 KB run, and the rest of each 128-byte line is an L1 hit on the next loads.  The
// query of the group sits in shared memory in fp64, [d][G], so every step of the
// d-loop is one broadcast read per head pair.
template <typename T, int G>
__global__ void __launch_bounds__(SC_THREADS) k_score(const T *__restrict__ lm,
                                                      const T *__restrict__ q,
                                                      double *__restrict__ scores, int64_t nC,
                                                      int Hq, int Hkv, int hd, int g_rt) {
    constexpr int EPV = 16 / sizeof(T);  // elements per 16-byte vector
    constexpr int NG = G > 0 ? G : SC_MAXG;
    extern __shared__ __align__(16) double qs[];   // [hd][ng]
    const int ng = G > 0 ? G : g_rt;
    const int b = blockIdx.z, g = blockIdx.y;
    const T *qb = q + ((size_t)b * Hq + (size_t)g * ng) * hd;
    for (int e = threadIdx.x; e < hd * ng; e += SC_THREADS) {
        const int h = e / hd, dd = e % hd;
        qs[dd * ng + h] = Elem<T>::f64(qb[(size_t)h * hd + dd]);
    }
    __syncthreads();
    const int64_t cbase = (int64_t)blockIdx.x * SC_THREADS * SC_CPT + threadIdx.x;
    const int vpr = hd / EPV;
    const uint4 *rows[SC_CPT];
    bool valid[SC_CPT];
#pragma unroll
    for (int i = 0; i < SC_CPT; ++i) {
        const int64_t c = cbase + (int64_t)i * SC_THREADS;
        valid[i] = c < nC;
        rows[i] = reinterpret_cast<const uint4 *>(lm + (((size_t)b * Hkv + g) * nC +
                                                        (valid[i] ? c : 0)) * hd);
    }
    double acc[SC_CPT][NG];
#pragma unroll
    for (int i = 0; i < SC_CPT; ++i)
#pragma unroll
        for (int h = 0; h < NG; ++h) acc[i][h] = 0.0;
#pragma unroll 2
    for (int v = 0; v < vpr; ++v) {
        uint4 w[SC_CPT];
#pragma unroll
        for (int i = 0; i < SC_CPT; ++i) w[i] = __ldg(rows[i] + v);
#pragma unroll
        for (int k = 0; k < EPV; ++k) {
            const double *qd = qs + (v * EPV + k) * ng;
            double x[SC_CPT];
#pragma unroll
            for (int i = 0; i < SC_CPT; ++i) x[i] = Elem<T>::f64(reinterpret_cast<const T *>(&w[i])[k]);
            if constexpr (G > 0) {
#pragma unroll
                for (int h = 0; h < G; ++h) {
                    const double qv = qd[h];
#pragma unroll
                    for (int i = 0; i < SC_CPT; ++i) acc[i][h] = fma(x[i], qv, acc[i][h]);  // exact product
                }
            } else {
                for (int h = 0; h < ng; ++h) {
                    const double qv = qd[h];
#pragma unroll
                    for (int i = 0; i < SC_CPT; ++i) acc[i][h] = fma(x[i], qv, acc[i][h]);
                }
            }
        }
    }
#pragma unroll
    for (int i = 0; i < SC_CPT; ++i) {
        if (!valid[i]) continue;
        double best = acc[i][0];
        for (int h = 1; h < ng; ++h)
            if (order_key(acc[i][h]) > order_key(best)) best = acc[i][h];
        scores[((size_t)b * Hkv + g) * nC + cbase + (int64_t)i * SC_THREADS] = best;
    }
}

template <typename T>
cudaError_t launch_t(const xkv_dims &d, const void *lm, const void *q, double *scores,
                     cudaStream_t s) {
    const int G = d.n_q_heads / d.n_kv_heads;
    const int64_t nC = d.ctx_len / d.chunk;
    const int64_t per_cta = (int64_t)SC_THREADS * SC_CPT;
    dim3 grid((unsigned)((nC + per_cta - 1) / per_cta), d.n_kv_heads, d.batch);
    const size_t smem = (size_t)d.head_dim * G * sizeof(double);
    const T *l = (const T *)lm;
    const T *qq = (const T *)q;
#define XKV_SCORE_CASE(GG)                                                                  \
    case GG: {                                                                              \
        auto k = k_score<T, GG>;                                                            \
        set_smem_limit((const void *)k, smem);                                              \
        k<<<grid, SC_THREADS, smem, s>>>(l, qq, scores, nC, d.n_q_heads, d.n_kv_heads,      \
                                         d.head_dim, G);                                    \
        break;                                                                              \
    }
    switch (G) {
        XKV_SCORE_CASE(1)
        XKV_SCORE_CASE(2)
        XKV_SCORE_CASE(4)
        XKV_SCORE_CASE(5)
        XKV_SCORE_CASE(8)
        default: {
            auto k = k_score<T, 0>;
            set_smem_limit((const void *)k, smem);
            k<<<grid, SC_THREADS, smem, s>>>(l, qq, scores, nC, d.n_q_heads, d.n_kv_heads,
                                             d.head_dim, G);
        }
    }
#undef XKV_SCORE_CASE
    return cudaGetLastError();
}

// ---------------------------------------------------------------- bf16 streaming path
// The per-row kernel above reads each landmark row with one thread, so every 16-byte
// load of a warp touches 32 different 128-byte lines.  Here a warp first reads a batch
// of 32 rows with fully coalesced 16-byte loads (lane l, load v takes 16-byte piece
// 32 v + l of the 8 KB batch), parks it in a padded shared-memory block (row stride
// HD*2 + 16 bytes, conflict-free both ways), and then each thread walks its own row in
// ascending d exactly as above.  The next batch's loads are issued before the current
// batch is scored, so every warp keeps one batch in flight.  Work is split into
// contiguous runs of (unit, batch) per warp; the group's query is re-staged (fp64,
// [d][G]) whenever a warp's run crosses into another unit.
constexpr int SW_THREADS = 256;
constexpr int SW_WARPS = SW_THREADS / 32;

template <int HD, int G>
__global__ void __launch_bounds__(SW_THREADS, 2)
    k_score_stream(const __nv_bfloat16 *__restrict__ lm, const __nv_bfloat16 *__restrict__ q,
                   double *__restrict__ scores, int64_t nC, int Hq, int Hkv, int n_units,
                   int64_t batches_per_unit) {
    constexpr int VPR = HD / 8;                    // 16-byte pieces per row
    constexpr int PIECES = 32 * VPR / 32;          // pieces per lane per batch (= VPR)
    constexpr int STRIDE = HD * 2 + 16;            // padded row stride in bytes
    extern __shared__ __align__(16) unsigned char sw_smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    unsigned char *rows = sw_smem + (size_t)warp * (32 * STRIDE + HD * G * 8);
    double *qs = reinterpret_cast<double *>(rows + 32 * STRIDE);   // [HD][G]

    const int64_t total = (int64_t)n_units * batches_per_unit;
    const int64_t n_warps = (int64_t)gridDim.x * SW_WARPS;
    const int64_t wg = (int64_t)blockIdx.x * SW_WARPS + warp;
    const int64_t k_begin = total * wg / n_warps, k_end = total * (wg + 1) / n_warps;
    if (k_begin >= k_end) return;

    uint4 buf[PIECES];
    auto load = [&](int64_t k) {                   // coalesced loads of batch k
        const int64_t unit = k / batches_per_unit, bt = k % batches_per_unit;
        const int64_t r0 = bt * 32;
        const uint4 *src = reinterpret_cast<const uint4 *>(lm + ((size_t)unit * nC + r0) * HD);
        const int64_t lim = min64((int64_t)32, nC - r0) * VPR;   // valid pieces
#pragma unroll
        for (int v = 0; v < PIECES; ++v) {
            const int pc = v * 32 + lane;
            buf[v] = pc < lim ? __ldg(src + pc) : make_uint4(0u, 0u, 0u, 0u);
        }
    };
    auto park = [&]() {
#pragma unroll
        for (int v = 0; v < PIECES; ++v) {
            const int pc = v * 32 + lane, r = pc / VPR, c = pc % VPR;
            *reinterpret_cast<uint4 *>(rows + r * STRIDE + c * 16) = buf[v];
        }
    };
    int64_t cur_unit = -1;
    load(k_begin);
    for (int64_t k = k_begin; k < k_end; ++k) {
        const int64_t unit = k / batches_per_unit;
        __syncwarp();                              // previous batch's rows fully read
        park();
        if (unit != cur_unit) {
            cur_unit = unit;
            const int b = (int)(unit / Hkv), g = (int)(unit % Hkv);
            const __nv_bfloat16 *qb = q + ((size_t)b * Hq + (size_t)g * G) * HD;
            for (int e = lane; e < HD * G; e += 32) {
                const int h = e / HD, dd = e % HD;
                qs[dd * G + h] = (double)__bfloat162float(qb[(size_t)h * HD + dd]);
            }
        }
        __syncwarp();
        if (k + 1 < k_end) load(k + 1);            // in flight while this batch is scored
        const int64_t r = (k % batches_per_unit) * 32 + lane;
        double acc[G];
#pragma unroll
        for (int h = 0; h < G; ++h) acc[h] = 0.0;
        const unsigned char *my = rows + lane * STRIDE;
#pragma unroll 2
        for (int c = 0; c < VPR; ++c) {
            const uint4 w = *reinterpret_cast<const uint4 *>(my + c * 16);
            const uint32_t wv[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const double x = (double)__uint_as_float(e & 1 ? wv[e >> 1] & 0xffff0000u
                                                               : wv[e >> 1] << 16);
                const double *qd = qs + (c * 8 + e) * G;
#pragma unroll
                for (int h = 0; h < G; ++h) acc[h] = fma(x, qd[h], acc[h]);   // exact product
            }
        }
        if (r < nC) {
            double best = acc[0];
#pragma unroll
            for (int h = 1; h < G; ++h)
                if (order_key(acc[h]) > order_key(best)) best = acc[h];
            scores[(size_t)unit * nC + r] = best;
        }
    }
}

template <int HD, int G>
cudaError_t launch_stream(const xkv_dims &d, const void *lm, const void *q, double *scores,
                          cudaStream_t s) {
    const int64_t nC = d.ctx_len / d.chunk;
    const int n_units = d.batch * d.n_kv_heads;
    const int64_t bpu = (nC + 31) / 32;
    const size_t smem = (size_t)SW_WARPS * (32 * (HD * 2 + 16) + HD * G * 8);
    auto k = k_score_stream<HD, G>;
    cudaError_t e = set_smem_limit((const void *)k, smem);
    if (e != cudaSuccess) return e;
    const int64_t warps_needed = (int64_t)n_units * bpu;
    int64_t grid = 2 * (int64_t)sm_count();
    if (grid * SW_WARPS > warps_needed) grid = (warps_needed + SW_WARPS - 1) / SW_WARPS;
    k<<<(unsigned)grid, SW_THREADS, smem, s>>>((const __nv_bfloat16 *)lm,
                                               (const __nv_bfloat16 *)q, scores, nC,
                                               d.n_q_heads, d.n_kv_heads, n_units, bpu);
    return cudaGetLastError();
}

template <int HD>
cudaError_t launch_stream_hd(const xkv_dims &d, const void *lm, const void *q, double *scores,
                             cudaStream_t s) {
    switch (d.n_q_heads / d.n_kv_heads) {
        case 1: return launch_stream<HD, 1>(d, lm, q, scores, s);
        case 2: return launch_stream<HD, 2>(d, lm, q, scores, s);
        case 4: return launch_stream<HD, 4>(d, lm, q, scores, s);
        case 5: return launch_stream<HD, 5>(d, lm, q, scores, s);
        case 8: return launch_stream<HD, 8>(d, lm, q, scores, s);
        default: return cudaErrorInvalidValue;
    }
}

bool stream_ok(const xkv_dims &d) {
    const int G = d.n_q_heads / d.n_kv_heads;
    return d.dtype == XKV_BF16 && (d.head_dim == 64 || d.head_dim == 128) &&
           (G == 1 || G == 2 || G == 4 || G == 5 || G == 8) && !getenv("XKV_FORCE_SIMT");
}

}  // namespace

cudaError_t launch_score(const xkv_dims &d, const void *lm, const void *q, double *scores,
                         cudaStream_t s) {
    if (stream_ok(d))
        return d.head_dim == 128 ? launch_stream_hd<128>(d, lm, q, scores, s)
                                 : launch_stream_hd<64>(d, lm, q, scores, s);
    return d.dtype == XKV_F32 ? launch_t<float>(d, lm, q, scores, s)
                              : launch_t<__nv_bfloat16>(d, lm, q, scores, s);
}

}  // namespace xkv
