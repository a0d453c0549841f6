// Landmark scoring (xKV page, section 2.3: rank the chunks by the relevance of their
// landmark key to the current query, taking the max over the GQA group).
//
// score[b][g][c] = max_{h in group g} sum_{d < hd} lm[b][g][c][d] * q[b][h][d], with every
// product exact in fp64 and the sum in ascending d, so the value is reproducible bit for
// bit on any IEEE-754 machine.  HBM-bound: one pass over the landmarks.
//
// One thread per chunk, 128 chunks per CTA.  The CTA's landmark rows are one contiguous
// block of memory; it is copied into shared memory with coalesced 16-byte loads and an
// XOR swizzle on the 16-byte column so that the row-per-thread reads are conflict-free.
#include "xkv_internal.cuh"

namespace xkv {
namespace {

constexpr int SC_ROWS = 128;
constexpr int SC_MAXG = 16;

template <typename T, int G>
__global__ void __launch_bounds__(SC_ROWS) k_score(const T *__restrict__ lm,
                                                   const T *__restrict__ q,
                                                   double *__restrict__ scores, int64_t nC,
                                                   int Hq, int Hkv, int hd, int g_rt) {
    constexpr int EPV = 16 / sizeof(T);  // elements per 16-byte vector
    extern __shared__ __align__(16) unsigned char smem[];
    const int ng = G > 0 ? G : g_rt;
    const int b = blockIdx.z, g = blockIdx.y;
    const int64_t c0 = (int64_t)blockIdx.x * SC_ROWS;
    const int rows = (int)min64(SC_ROWS, nC - c0);
    const int vpr = hd / EPV;  // 16-byte vectors per row (8..32)

    double *qs = reinterpret_cast<double *>(smem);               // [hd][ng]
    uint4 *tile = reinterpret_cast<uint4 *>(smem + (size_t)hd * ng * sizeof(double));

    const T *qb = q + ((size_t)b * Hq + (size_t)g * ng) * hd;
    for (int e = threadIdx.x; e < hd * ng; e += blockDim.x) {
        const int h = e / hd, dd = e % hd;
        qs[dd * ng + h] = Elem<T>::f64(qb[(size_t)h * hd + dd]);
    }
    const uint4 *src = reinterpret_cast<const uint4 *>(lm + (((size_t)b * Hkv + g) * nC + c0) * hd);
    for (int e = threadIdx.x; e < rows * vpr; e += blockDim.x) {
        const int r = e / vpr, v = e % vpr;
        tile[r * vpr + (v ^ (r & 7))] = __ldg(src + e);
    }
    __syncthreads();
    const int r = threadIdx.x;
    if (r >= rows) return;

    double acc[G > 0 ? G : SC_MAXG];
#pragma unroll
    for (int h = 0; h < (G > 0 ? G : SC_MAXG); ++h) acc[h] = 0.0;
    for (int v = 0; v < vpr; ++v) {
        const uint4 w = tile[r * vpr + (v ^ (r & 7))];
        const T *e = reinterpret_cast<const T *>(&w);
#pragma unroll
        for (int k = 0; k < EPV; ++k) {
            const double x = Elem<T>::f64(e[k]);
            const double *qd = qs + (v * EPV + k) * ng;
            if constexpr (G > 0) {
#pragma unroll
                for (int h = 0; h < G; ++h) acc[h] = fma(x, qd[h], acc[h]);  // exact product
            } else {
                for (int h = 0; h < ng; ++h) acc[h] = fma(x, qd[h], acc[h]);
            }
        }
    }
    double best = acc[0];
    for (int h = 1; h < ng; ++h)
        if (order_key(acc[h]) > order_key(best)) best = acc[h];
    scores[((size_t)b * Hkv + g) * nC + c0 + r] = best;
}

template <typename T>
cudaError_t launch_t(const xkv_dims &d, const void *lm, const void *q, double *scores,
                     cudaStream_t s) {
    const int G = d.n_q_heads / d.n_kv_heads;
    const int64_t nC = d.ctx_len / d.chunk;
    dim3 grid((unsigned)((nC + SC_ROWS - 1) / SC_ROWS), d.n_kv_heads, d.batch);
    const size_t smem = (size_t)d.head_dim * G * sizeof(double) +
                        (size_t)SC_ROWS * d.head_dim * sizeof(T);
    const T *l = (const T *)lm;
    const T *qq = (const T *)q;
#define XKV_SCORE_CASE(GG)                                                                  \
    case GG: {                                                                              \
        auto k = k_score<T, GG>;                                                            \
        set_smem_limit((const void *)k, smem);    \
        k<<<grid, SC_ROWS, smem, s>>>(l, qq, scores, nC, d.n_q_heads, d.n_kv_heads,         \
                                      d.head_dim, G);                                       \
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
            k<<<grid, SC_ROWS, smem, s>>>(l, qq, scores, nC, d.n_q_heads, d.n_kv_heads,
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
