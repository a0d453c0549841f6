// Landmark keys of one layer (built once per cache, outside the decode step).
//
// xKV page, section 2.3: chunk selection is landmark-based; a chunk's landmark is the
// mean of its reconstructed key rows.  By linearity the mean of the rows A[t] B is
// (sum_t A[t]) B / C, so each CTA first sums the C basis rows of its chunks and then
// multiplies by B_l's group-g columns, all in fp64, and rounds once to the storage type.
#include "xkv_internal.cuh"

namespace xkv {
namespace {

constexpr int LM_CHUNKS = 16;  // chunks per CTA
constexpr int LM_ITILE = 64;   // rank slice staged in shared memory

template <typename T>
__global__ void __launch_bounds__(128) k_build_landmarks(const T *__restrict__ Ak,
                                                         const T *__restrict__ Bkt,
                                                         T *__restrict__ lm, int64_t L, int C,
                                                         int rk, int Hkv, int hd) {
    __shared__ double abar[LM_CHUNKS][LM_ITILE];
    const int b = blockIdx.z, g = blockIdx.y;
    const int64_t nC = L / C;
    const int64_t c0 = (int64_t)blockIdx.x * LM_CHUNKS;
    const int nch = (int)min64(LM_CHUNKS, nC - c0);
    const int j = threadIdx.x;
    const T *A = Ak + (size_t)b * L * rk;
    const T *Bcol = Bkt + ((size_t)b * Hkv * hd + (size_t)g * hd + min(j, hd - 1)) * rk;
    double acc[LM_CHUNKS];
#pragma unroll
    for (int c = 0; c < LM_CHUNKS; ++c) acc[c] = 0.0;

    for (int i0 = 0; i0 < rk; i0 += LM_ITILE) {
        const int ni = min(LM_ITILE, rk - i0);
        __syncthreads();
        for (int e = threadIdx.x; e < LM_CHUNKS * LM_ITILE; e += blockDim.x) {
            const int c = e / LM_ITILE, i = e % LM_ITILE;
            double s = 0.0;
            if (c < nch && i < ni) {
                const T *row = A + ((c0 + c) * C) * rk + i0 + i;
                for (int u = 0; u < C; ++u) s += Elem<T>::f64(row[(size_t)u * rk]);
            }
            abar[c][i] = s;
        }
        __syncthreads();
        for (int i = 0; i < ni; ++i) {
            const double bv = Elem<T>::f64(Bcol[i0 + i]);
#pragma unroll
            for (int c = 0; c < LM_CHUNKS; ++c) acc[c] = fma(abar[c][i], bv, acc[c]);
        }
    }
    if (j >= hd) return;
    for (int c = 0; c < nch; ++c) {
        const double mean = acc[c] / (double)C;
        T *dst = lm + (((size_t)b * Hkv + g) * nC + c0 + c) * hd + j;
        if constexpr (sizeof(T) == 4) {
            *dst = __double2float_rn(mean);
        } else {
            *reinterpret_cast<uint16_t *>(dst) = f64_to_bf16_rne(mean);
        }
    }
}

}  // namespace

cudaError_t launch_build_landmarks(const xkv_dims &d, const void *Ak, const void *Bkt, void *lm,
                                   cudaStream_t s) {
    const int64_t nC = d.ctx_len / d.chunk;
    dim3 grid((unsigned)((nC + LM_CHUNKS - 1) / LM_CHUNKS), d.n_kv_heads, d.batch);
    if (d.dtype == XKV_F32)
        k_build_landmarks<float><<<grid, 128, 0, s>>>((const float *)Ak, (const float *)Bkt,
                                                      (float *)lm, d.ctx_len, d.chunk, d.rank_k,
                                                      d.n_kv_heads, d.head_dim);
    else
        k_build_landmarks<__nv_bfloat16><<<grid, 128, 0, s>>>(
            (const __nv_bfloat16 *)Ak, (const __nv_bfloat16 *)Bkt, (__nv_bfloat16 *)lm,
            d.ctx_len, d.chunk, d.rank_k, d.n_kv_heads, d.head_dim);
    return cudaGetLastError();
}

}  // namespace xkv
