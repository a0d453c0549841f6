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

constexpr int SC_THREADS = 128;
constexpr int SC_CPT = 4;      // chunks per thread: 4G independent fp64 chains
constexpr int SC_MAXG = 16;

// One thread scores SC_CPT chunks (rows c, c + 128, c + 256, c + 384 of the CTA's
// block).  Each row is read with 16-byte loads straight from global memory: a warp's 32
// rows are one contiguous 8 KB run, and the rest of each 128-byte line is an L1 hit on
// the next loads.  The query of the group sits in shared memory in fp64, [d][G]; each
// broadcast read of it feeds the SC_CPT rows of the thread.  Profiles show the kernel
// bound by latency (shared-memory writeback, fp64 conversions and fma chains each
// 25-50 % busy); of the layouts measured (1, 2 and 4 rows per thread, warp-staged
// coalesced rows, TMA-staged rows) this one is the fastest.
template <typename T, int G>
__global__ void __launch_bounds__(SC_THREADS) k_score(const T *__restrict__ lm,
                                                      const T *__restrict__ q,
                                                      double *__restrict__ scores, int64_t nC,
                                                      int Hq, int Hkv, int hd, int g_rt) {
    constexpr int EPV = 16 / sizeof(T);  // elements per 16-byte vector
    constexpr int NG = G > 0 ? G : SC_MAXG;
    extern __shared__ __align__(16) double qs[];   // [hd][ng]
    grid_dep_launch();  // the selection kernel after this one may be scheduled
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

}  // namespace

cudaError_t launch_score(const xkv_dims &d, const void *lm, const void *q, double *scores,
                         cudaStream_t s) {
    return d.dtype == XKV_F32 ? launch_t<float>(d, lm, q, scores, s)
                              : launch_t<__nv_bfloat16>(d, lm, q, scores, s);
}

}  // namespace xkv
