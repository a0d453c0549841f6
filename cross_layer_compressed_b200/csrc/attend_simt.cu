// Selective / dense reconstruction followed by GQA attention on CUDA cores.
//
// xKV page, section 2.3: only the selected rows are rebuilt, K_hat = A^K[T] B^K_l and
// V_hat = A^V[T] B^V_l, then attended; section 4: the same over every row (dense).
// This is the fp32 path (fp32 factors keep fp32 products; the tensor cores would round
// them to tf32) and the reference CUDA path for bf16.
//
// Grid (split, KV head, sequence).  A CTA owns a contiguous range of its unit's rows
// and runs two phases: (1) rebuild key rows in tiles of AT_RT and store the G logits of
// every row in shared memory; then take the exact max / sum of its range; (2) rebuild
// value rows and accumulate p * V_hat.  It writes the partial (m, l, acc) of its range;
// a combine kernel merges the splits.  Thread j owns output column j of the head.
#include "xkv_internal.cuh"

namespace xkv {
namespace {

constexpr int AT_THREADS = 128;
constexpr int AT_RT = 16;

template <typename T, int G>
__global__ void __launch_bounds__(AT_THREADS) k_attend_simt(
    const T *__restrict__ Ak, const T *__restrict__ Av, const T *__restrict__ Bkt,
    const T *__restrict__ Bvt, const T *__restrict__ q, const int32_t *__restrict__ sel,
    int n_sel, int64_t L, int C, int rk, int rv, int Hq, int Hkv, int hd, int64_t rows_total,
    int64_t rows_per_split, float *__restrict__ partials, unsigned *__restrict__ status) {
    extern __shared__ __align__(16) float sm[];
    const int split = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
    const int B = gridDim.z;
    const int rmax = rk > rv ? rk : rv;
    float *As = sm;                         // [AT_RT][rmax]
    float *Ks = As + AT_RT * rmax;          // [AT_RT][hd]
    float *qs = Ks + AT_RT * hd;            // [G][hd]
    float *stat = qs + G * hd;              // [2][G] (m, l)
    float *z = stat + 2 * G;                // [rows_per_split][G]

    const int64_t r0 = (int64_t)split * rows_per_split;
    const int nr = (int)min64(rows_per_split, rows_total - r0);
    const int j = threadIdx.x;
    const int d_kv = Hkv * hd;
    const int32_t *su = sel ? sel + ((size_t)b * Hkv + g) * n_sel : nullptr;
    const int64_t nC = L / C;
    auto token = [&](int64_t i) -> int64_t {
        if (!su) return i;
        const int64_t c0 = su[i / C];
        if ((c0 < 0 || c0 >= nC) && status)   // the call fails (NaN outputs); reads stay
            atomicOr(status, 1u << XKV_ERR_INVALID_ARG);   // in bounds
        const int64_t c = min64(max64(c0, 0), nC - 1);
        return c * C + i % C;
    };
    const float scale = 1.0f / sqrtf((float)hd);

    for (int e = threadIdx.x; e < G * hd; e += AT_THREADS)
        qs[e] = Elem<T>::f32(q[((size_t)b * Hq + (size_t)g * G) * hd + e]);

    // ---------------- phase 1: logits over the reconstructed keys
    const T *Ab = Ak + (size_t)b * L * rk;
    const T *Bk = Bkt + ((size_t)b * d_kv + (size_t)g * hd + min(j, hd - 1)) * rk;
    for (int t0 = 0; t0 < nr; t0 += AT_RT) {
        const int nt = min(AT_RT, nr - t0);
        __syncthreads();
        for (int e = threadIdx.x; e < nt * rk; e += AT_THREADS) {
            const int r = e / rk, i = e % rk;
            As[r * rmax + i] = Elem<T>::f32(Ab[token(r0 + t0 + r) * rk + i]);
        }
        __syncthreads();
        float acc[AT_RT];
#pragma unroll
        for (int r = 0; r < AT_RT; ++r) acc[r] = 0.f;
        for (int i = 0; i < rk; ++i) {
            const float bv = Elem<T>::f32(Bk[i]);
#pragma unroll
            for (int r = 0; r < AT_RT; ++r) acc[r] = fmaf(As[r * rmax + i], bv, acc[r]);
        }
        if (j < hd)
            for (int r = 0; r < nt; ++r) Ks[r * hd + j] = acc[r];
        __syncthreads();
        for (int p = threadIdx.x; p < nt * G; p += AT_THREADS) {
            const int r = p / G, h = p % G;
            float dot = 0.f;
            for (int dd = 0; dd < hd; ++dd) dot = fmaf(qs[h * hd + dd], Ks[r * hd + dd], dot);
            z[(t0 + r) * G + h] = dot * scale;
        }
    }
    __syncthreads();

    // ---------------- softmax statistics of this range (exact: all logits are known)
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int h = warp; h < G; h += AT_THREADS / 32) {
        float m = -INFINITY;
        for (int r = lane; r < nr; r += 32) m = fmaxf(m, z[r * G + h]);
#pragma unroll
        for (int off = 16; off; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
        float l = 0.f;
        for (int r = lane; r < nr; r += 32) {
            const float p = expf(z[r * G + h] - m);
            z[r * G + h] = p;
            l += p;
        }
#pragma unroll
        for (int off = 16; off; off >>= 1) l += __shfl_xor_sync(0xffffffffu, l, off);
        if (lane == 0) {
            stat[h] = m;
            stat[G + h] = l;
        }
    }

    // ---------------- phase 2: weighted sum of the reconstructed values
    float o[G];
#pragma unroll
    for (int h = 0; h < G; ++h) o[h] = 0.f;
    const T *AvB = Av + (size_t)b * L * rv;
    const T *Bv = Bvt + ((size_t)b * d_kv + (size_t)g * hd + min(j, hd - 1)) * rv;
    for (int t0 = 0; t0 < nr; t0 += AT_RT) {
        const int nt = min(AT_RT, nr - t0);
        __syncthreads();
        for (int e = threadIdx.x; e < nt * rv; e += AT_THREADS) {
            const int r = e / rv, i = e % rv;
            As[r * rmax + i] = Elem<T>::f32(AvB[token(r0 + t0 + r) * rv + i]);
        }
        __syncthreads();
        float acc[AT_RT];
#pragma unroll
        for (int r = 0; r < AT_RT; ++r) acc[r] = 0.f;
        for (int i = 0; i < rv; ++i) {
            const float bv = Elem<T>::f32(Bv[i]);
#pragma unroll
            for (int r = 0; r < AT_RT; ++r) acc[r] = fmaf(As[r * rmax + i], bv, acc[r]);
        }
        for (int r = 0; r < nt; ++r)
#pragma unroll
            for (int h = 0; h < G; ++h) o[h] = fmaf(z[(t0 + r) * G + h], acc[r], o[h]);
    }
    if (j < hd) {
        for (int h = 0; h < G; ++h) {
            float *dst = partials + (((size_t)split * B + b) * Hq + (size_t)g * G + h) * (hd + 2);
            dst[2 + j] = o[h];
            if (j == 0) {
                dst[0] = stat[h];
                dst[1] = stat[G + h];
            }
        }
    }
}

template <typename T, int G>
cudaError_t launch_g(const xkv_dims &d, const void *Ak, const void *Av, const void *Bkt,
                     const void *Bvt, const void *q, const int32_t *sel, int n_sel,
                     const SplitPlan &plan, float *partials, unsigned *status, cudaStream_t s) {
    const int rmax = d.rank_k > d.rank_v ? d.rank_k : d.rank_v;
    const size_t smem = sizeof(float) * ((size_t)AT_RT * rmax + (size_t)AT_RT * d.head_dim +
                                         (size_t)G * d.head_dim + 2 * G +
                                         (size_t)plan.rows_per_split * G);
    const int64_t rows = sel ? (int64_t)n_sel * d.chunk : d.ctx_len;
    auto k = k_attend_simt<T, G>;
    set_smem_limit((const void *)k, smem);
    dim3 grid(plan.n_split, d.n_kv_heads, d.batch);
    k<<<grid, AT_THREADS, smem, s>>>((const T *)Ak, (const T *)Av, (const T *)Bkt,
                                     (const T *)Bvt, (const T *)q, sel, n_sel, d.ctx_len,
                                     d.chunk, d.rank_k, d.rank_v, d.n_q_heads, d.n_kv_heads,
                                     d.head_dim, rows, plan.rows_per_split, partials, status);
    return cudaGetLastError();
}

template <typename T>
cudaError_t launch_t(const xkv_dims &d, const void *Ak, const void *Av, const void *Bkt,
                     const void *Bvt, const void *q, const int32_t *sel, int n_sel,
                     const SplitPlan &plan, float *partials, unsigned *status, cudaStream_t s) {
    switch (d.n_q_heads / d.n_kv_heads) {
#define XKV_G(GG) \
    case GG:                                                                               \
        return launch_g<T, GG>(d, Ak, Av, Bkt, Bvt, q, sel, n_sel, plan, partials, status, s);
        XKV_G(1) XKV_G(2) XKV_G(3) XKV_G(4) XKV_G(5) XKV_G(6) XKV_G(7) XKV_G(8)
        XKV_G(9) XKV_G(10) XKV_G(11) XKV_G(12) XKV_G(13) XKV_G(14) XKV_G(15) XKV_G(16)
#undef XKV_G
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace

cudaError_t launch_attend_simt(const xkv_dims &d, const void *Ak, const void *Av,
                               const void *Bkt, const void *Bvt, const void *q,
                               const int32_t *sel, int n_sel, const SplitPlan &plan,
                               float *partials, unsigned *status, cudaStream_t s) {
    return d.dtype == XKV_F32
               ? launch_t<float>(d, Ak, Av, Bkt, Bvt, q, sel, n_sel, plan, partials, status, s)
               : launch_t<__nv_bfloat16>(d, Ak, Av, Bkt, Bvt, q, sel, n_sel, plan, partials,
                                         status, s);
}

}  // namespace xkv
