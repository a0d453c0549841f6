// R-CLA decode attention over a leader's KV cache (Stochastic KV Routing page: at
// inference a fixed set S of layers stores KV; a layer outside S reads the nearest
// previous leader's cache and skips its own K/V load and update, the page's
// Algorithm 2).  HBM-bound stream of K and V; CUDA cores.
//
// Grid (split, KV head, sequence), flash-decoding style: a CTA owns a contiguous range
// of rows.  Phase 1 stages K tiles of 128 rows in shared memory (coalesced 16-byte
// loads, XOR-swizzled 16-byte columns) and one thread per row forms the G logits.
// The range's max and sum are then exact.  Phase 2 stages V tiles the same way and
// thread j accumulates column j of the G outputs.  Partials (m, l, acc) per range go
// to the workspace; a combine kernel merges them.
//
// The leader's update: when `update_row` >= 0, the CTAs of split 0 copy k_new / v_new
// into that row of the cache, and every CTA reads that row from k_new / v_new (never
// from the cache), so no CTA depends on another's write.
#include "xkv_internal.cuh"

namespace xkv {
namespace {

constexpr int RC_THREADS = 128;
constexpr int RC_TILE = 128;

template <typename T, int G>
__global__ void __launch_bounds__(RC_THREADS) k_rcla(
    T *__restrict__ K, T *__restrict__ V, const T *__restrict__ k_new,
    const T *__restrict__ v_new, const T *__restrict__ q, int slot, int Hq, int Hkv, int hd,
    int64_t L_max, int64_t n_rows, int64_t update_row, int64_t rows_per_split,
    float *__restrict__ partials) {
    constexpr int EPV = 16 / sizeof(T);
    extern __shared__ __align__(16) unsigned char smem[];
    const int split = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
    const int B = gridDim.z;
    const int vpr = hd / EPV;
    uint4 *tile = reinterpret_cast<uint4 *>(smem);                         // [RC_TILE][vpr]
    float *qs = reinterpret_cast<float *>(smem + (size_t)RC_TILE * hd * sizeof(T));  // [hd][G]
    float *stat = qs + hd * G;                                              // [2][G]
    float *z = stat + 2 * G;                                                // [rows][G]

    const size_t cache_off = (((size_t)slot * B + b) * Hkv + g) * (size_t)L_max * hd;
    const size_t new_off = ((size_t)b * Hkv + g) * hd;
    if (update_row >= 0 && split == 0) {
        for (int e = threadIdx.x; e < hd; e += RC_THREADS) {
            K[cache_off + (size_t)update_row * hd + e] = k_new[new_off + e];
            V[cache_off + (size_t)update_row * hd + e] = v_new[new_off + e];
        }
    }
    for (int e = threadIdx.x; e < G * hd; e += RC_THREADS) {
        const int h = e / hd, dd = e % hd;
        qs[dd * G + h] = Elem<T>::f32(q[((size_t)b * Hq + (size_t)g * G + h) * hd + dd]);
    }
    const int64_t r0 = (int64_t)split * rows_per_split;
    const int nr = (int)min64(rows_per_split, n_rows - r0);
    const float scale = 1.0f / sqrtf((float)hd);

    auto stage = [&](const T *cache, const T *newrow, int t0, int nt) {
        const uint4 *src = reinterpret_cast<const uint4 *>(cache + cache_off + (size_t)(r0 + t0) * hd);
        const uint4 *nsrc = reinterpret_cast<const uint4 *>(newrow + new_off);
        for (int e = threadIdx.x; e < nt * vpr; e += RC_THREADS) {
            const int r = e / vpr, v = e % vpr;
            const bool is_new = (r0 + t0 + r) == update_row;
            tile[r * vpr + (v ^ (r & 7))] = is_new ? nsrc[v] : src[e];  // plain loads: this kernel writes the cache
        }
    };

    // ---------------- phase 1: logits
    for (int t0 = 0; t0 < nr; t0 += RC_TILE) {
        const int nt = min(RC_TILE, nr - t0);
        __syncthreads();
        stage(K, k_new, t0, nt);
        __syncthreads();
        const int r = threadIdx.x;
        if (r < nt) {
            float acc[G];
#pragma unroll
            for (int h = 0; h < G; ++h) acc[h] = 0.f;
            for (int v = 0; v < vpr; ++v) {
                const uint4 w = tile[r * vpr + (v ^ (r & 7))];
                const T *e = reinterpret_cast<const T *>(&w);
#pragma unroll
                for (int k = 0; k < EPV; ++k) {
                    const float x = Elem<T>::f32(e[k]);
                    const float *qd = qs + (v * EPV + k) * G;
#pragma unroll
                    for (int h = 0; h < G; ++h) acc[h] = fmaf(x, qd[h], acc[h]);
                }
            }
#pragma unroll
            for (int h = 0; h < G; ++h) z[(t0 + r) * G + h] = acc[h] * scale;
        }
    }
    __syncthreads();

    // ---------------- softmax statistics of the range
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int h = warp; h < G; h += RC_THREADS / 32) {
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

    // ---------------- phase 2: p . V
    float o[G];
#pragma unroll
    for (int h = 0; h < G; ++h) o[h] = 0.f;
    const int j = threadIdx.x;
    const int jv = j / EPV, jk = j % EPV;
    for (int t0 = 0; t0 < nr; t0 += RC_TILE) {
        const int nt = min(RC_TILE, nr - t0);
        __syncthreads();
        stage(V, v_new, t0, nt);
        __syncthreads();
        if (j < hd) {
            for (int r = 0; r < nt; ++r) {
                const T *row = reinterpret_cast<const T *>(tile + r * vpr + (jv ^ (r & 7)));
                const float x = Elem<T>::f32(row[jk]);
#pragma unroll
                for (int h = 0; h < G; ++h) o[h] = fmaf(z[(t0 + r) * G + h], x, o[h]);
            }
        }
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
cudaError_t launch_g(const xkv_dims &d, int slot, int64_t L_max, int64_t n_rows,
                     int64_t update_row, void *K, void *V, const void *k_new,
                     const void *v_new, const void *q, const SplitPlan &plan, float *partials,
                     cudaStream_t s) {
    const size_t smem = (size_t)RC_TILE * d.head_dim * sizeof(T) +
                        sizeof(float) * ((size_t)d.head_dim * G + 2 * G +
                                         (size_t)plan.rows_per_split * G);
    auto k = k_rcla<T, G>;
    set_smem_limit((const void *)k, smem);
    dim3 grid(plan.n_split, d.n_kv_heads, d.batch);
    k<<<grid, RC_THREADS, smem, s>>>((T *)K, (T *)V, (const T *)k_new, (const T *)v_new,
                                     (const T *)q, slot, d.n_q_heads, d.n_kv_heads, d.head_dim,
                                     L_max, n_rows, update_row, plan.rows_per_split, partials);
    return cudaGetLastError();
}

template <typename T>
cudaError_t launch_t(const xkv_dims &d, int slot, int64_t L_max, int64_t n_rows,
                     int64_t update_row, void *K, void *V, const void *k_new,
                     const void *v_new, const void *q, const SplitPlan &plan, float *partials,
                     cudaStream_t s) {
    switch (d.n_q_heads / d.n_kv_heads) {
#define XKV_G(GG)                                                                            \
    case GG:                                                                                 \
        return launch_g<T, GG>(d, slot, L_max, n_rows, update_row, K, V, k_new, v_new, q,    \
                               plan, partials, s);
        XKV_G(1) XKV_G(2) XKV_G(3) XKV_G(4) XKV_G(5) XKV_G(6) XKV_G(7) XKV_G(8)
        XKV_G(9) XKV_G(10) XKV_G(11) XKV_G(12) XKV_G(13) XKV_G(14) XKV_G(15) XKV_G(16)
#undef XKV_G
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace

cudaError_t launch_rcla(const xkv_dims &d, int slot, int64_t L_max, int64_t n_rows,
                        int64_t update_row, void *K, void *V, const void *k_new,
                        const void *v_new, const void *q, const SplitPlan &plan,
                        float *partials, cudaStream_t s) {
    return d.dtype == XKV_F32
               ? launch_t<float>(d, slot, L_max, n_rows, update_row, K, V, k_new, v_new, q,
                                 plan, partials, s)
               : launch_t<__nv_bfloat16>(d, slot, L_max, n_rows, update_row, K, V, k_new,
                                         v_new, q, plan, partials, s);
}

}  // namespace xkv
