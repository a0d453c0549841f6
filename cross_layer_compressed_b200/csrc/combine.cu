// Merge of split-K partial attention results (flash-decoding): each split s of a
// (sequence, query head) left (m_s, l_s, acc_s) with acc_s = sum_t exp(z_t - m_s) v_t
// over its rows.  out = sum_s exp(m_s - M) acc_s / sum_s exp(m_s - M) l_s, M = max m_s.
#include <cstdlib>
#include <map>
#include <mutex>
#include <utility>

#include "xkv_internal.cuh"

namespace xkv {
namespace {

__global__ void __launch_bounds__(128) k_combine(const float *__restrict__ partials,
                                                 float *__restrict__ out, int n_split,
                                                 int BH, int hd,
                                                 const unsigned *__restrict__ status) {
    const int bh = blockIdx.x;
    const int j = threadIdx.x;
    grid_dep_wait();  // the partials and the status word come from the kernels before
    if (status && *(volatile const unsigned *)status) {  // the attention kernel gave up
        if (j < hd) out[(size_t)bh * hd + j] = __int_as_float(0x7fc00000);
        return;
    }
    const size_t stride = (size_t)BH * (hd + 2);
    const float *p = partials + (size_t)bh * (hd + 2);
    // the splits' loads are independent: unrolled, several are in flight at once
    float M = -INFINITY;
#pragma unroll 8
    for (int s = 0; s < n_split; ++s) M = fmaxf(M, p[s * stride]);
    float l = 0.f, acc = 0.f;
#pragma unroll 8
    for (int s = 0; s < n_split; ++s) {
        const float w = expf(p[s * stride] - M);
        l = fmaf(w, p[s * stride + 1], l);
        if (j < hd) acc = fmaf(w, p[s * stride + 2 + j], acc);
    }
    if (j < hd) out[(size_t)bh * hd + j] = acc / l;
}

// More than a few splits (9 for a selective call at 32K, hundreds for dense 128K): one
// CTA per (b, h) of 8 warps; the splits' running max comes from a block reduction, then warp w sums splits
// w, w + 8, ... with each lane holding 4 columns, so many loads are in flight, and the
// warps' sums meet in shared memory.  Same merge as k_combine, in another order.
constexpr int CW_THREADS = 256;
__global__ void __launch_bounds__(CW_THREADS) k_combine_wide(const float *__restrict__ partials,
                                                             float *__restrict__ out,
                                                             int n_split, int BH, int hd,
                                                             const unsigned *__restrict__ status) {
    constexpr int NW = CW_THREADS / 32;
    __shared__ float red[NW][128];
    __shared__ float s_m[NW], s_l[NW];
    const int bh = blockIdx.x;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    grid_dep_wait();
    if (status && *(volatile const unsigned *)status) {  // the attention kernel gave up
        if (threadIdx.x < hd) out[(size_t)bh * hd + threadIdx.x] = __int_as_float(0x7fc00000);
        return;
    }
    const size_t stride = (size_t)BH * (hd + 2);
    const float *p = partials + (size_t)bh * (hd + 2);
    float M = -INFINITY;
    for (int s = threadIdx.x; s < n_split; s += CW_THREADS) M = fmaxf(M, p[s * stride]);
#pragma unroll
    for (int off = 16; off; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
    if (lane == 0) s_m[warp] = M;
    __syncthreads();
    M = s_m[0];
#pragma unroll
    for (int w = 1; w < NW; ++w) M = fmaxf(M, s_m[w]);
    float acc[4] = {0.f, 0.f, 0.f, 0.f}, l = 0.f;
#pragma unroll 4
    for (int s = warp; s < n_split; s += NW) {
        const float *ps = p + s * stride;
        const float w = expf(ps[0] - M);
        l = fmaf(w, ps[1], l);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const int j = lane + 32 * k;
            if (j < hd) acc[k] = fmaf(w, ps[2 + j], acc[k]);
        }
    }
#pragma unroll
    for (int k = 0; k < 4; ++k) red[warp][lane + 32 * k] = acc[k];
    if (lane == 0) s_l[warp] = l;
    __syncthreads();
    if (threadIdx.x < hd) {
        float sum = 0.f, ls = 0.f;
#pragma unroll
        for (int w = 0; w < NW; ++w) {
            sum += red[w][threadIdx.x];
            ls += s_l[w];
        }
        out[(size_t)bh * hd + threadIdx.x] = sum / ls;
    }
}

}  // namespace

cudaError_t launch_combine(const xkv_dims &d, int n_split, const float *partials, float *out,
                           const unsigned *status, cudaStream_t s) {
    const int BH = d.batch * d.n_q_heads;
    if (n_split > 4)
        return launch_chained(k_combine_wide, dim3(BH), dim3(CW_THREADS), 0, s, partials, out,
                              n_split, BH, d.head_dim, status);
    return launch_chained(k_combine, dim3(BH), dim3(128), 0, s, partials, out, n_split, BH,
                          d.head_dim, status);
}

namespace {
// Lets the kernels after it be scheduled at once, then waits for the grid before it, so
// that a grid waiting on this one also waits on that one.
__global__ void k_clear_status(unsigned *status) {
    grid_dep_launch();
    grid_dep_wait();
    *status = 0u;
}
}  // namespace

cudaError_t launch_clear_status(unsigned *status, cudaStream_t s) {
    return launch_chained(k_clear_status, dim3(1), dim3(1), 0, s, status);
}

bool chain_enabled() { return !env_flag(ENV_NO_PDL); }

SplitPlan plan_splits(int64_t rows, int64_t units, int64_t min_rows, int64_t max_rows) {
    // Aim for about four CTAs per SM over the 148 SMs of a B200, with at least
    // min_rows rows per split and at most max_rows (the logits held in shared memory).
    const int64_t target_ctas = 148 * 4;
    int64_t n = (target_ctas + units - 1) / units;
    n = n < (rows + min_rows - 1) / min_rows ? n : (rows + min_rows - 1) / min_rows;
    const int64_t n_hi = (rows + max_rows - 1) / max_rows;
    if (n < n_hi) n = n_hi;
    if (n < 1) n = 1;
    SplitPlan p;
    p.n_bound = n;
    p.rows_per_split = (rows + n - 1) / n;
    p.n_split = (int)((rows + p.rows_per_split - 1) / p.rows_per_split);  // no empty split
    return p;
}

cudaError_t set_smem_limit(const void *kernel, size_t bytes) {
    static std::mutex mu;
    static std::map<std::pair<const void *, int>, size_t> done;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    std::lock_guard<std::mutex> lock(mu);
    size_t &cur = done[std::make_pair(kernel, dev)];
    if (bytes <= cur) return cudaSuccess;
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
    if (e == cudaSuccess) cur = bytes;
    return e;
}

size_t partial_bytes(const xkv_dims &d, int n_split) {
    return (size_t)n_split * d.batch * d.n_q_heads * (d.head_dim + 2) * sizeof(float);
}

}  // namespace xkv
