// Cross-layer factorization of one window (xKV page, section 2.2: the caches of the W
// layers of a window are concatenated side by side, a rank-r SVD of the concatenation
// gives one token basis A shared by the window and one reconstruction matrix B_l per
// layer, so that A·B_l stands in for layer l's cache).
//
// Per sequence the concatenation X = [X_0 | ... | X_{W-1}] (L x n, n = W·d_kv) is never
// built: every product addresses layer l's block of columns in place.  The rank-r
// factorization comes from randomized subspace iteration (Halko, Martinsson and Tropp,
// "Finding structure with randomness", SIAM Review 2011, Algorithm 4.4) with the
// caller's Gaussian test matrix Omega (n x r):
//
//     Y = X Omega,  Q = orth(Y);   n_iter times:  Z = orth(X^T Q),  Q = orth(X Z);
//     A = Q,  B_l^T = X_l^T Q.
//
// A spans the dominant rank-r left singular subspace once the iteration has converged
// (the error shrinks like (s_{r+1} / s_r)^(2 n_iter + 1)), so A·B_l is the truncated
// SVD's product; A itself is one orthonormal basis of that subspace, not U_r (the two
// differ by an r x r rotation that no product sees).
//
// orth() is CholeskyQR2 (two passes of: G = Y^T Y in fp64, G = R^T R by Cholesky in
// fp64, Y <- Y R^-1).  A column whose Cholesky pivot is below 1e-12 of the largest
// diagonal entry of G (a direction the data does not have: rank(X) < r) is zeroed
// rather than normalised, so A keeps orthonormal columns and zero columns.
//
// The products are fp32 CUDA-core GEMMs (fp32 accumulation); the Gram matrices,
// Cholesky factors and triangular inverses are fp64.
#include <cuda_runtime.h>

#include "xkv_internal.cuh"

namespace xkv {
namespace {

// A matrix operand of one sequence: element (row i, column j) of sequence b sits at
// b*s_b + i*s_r + j*s_c, plus jump_r for every whole block of blk_r rows before i and
// jump_c for every whole block of blk_c columns before j (blk = 0: no blocks).  The
// blocks let one operand walk the W layer buffers of a window as one matrix.
struct Mat {
    const void *p;
    int64_t s_r, s_c, s_b;
    int32_t blk_r, blk_c;
    int64_t jump_r, jump_c;
};

__device__ __forceinline__ int64_t row_part(const Mat &m, int i) {
    int64_t o = (int64_t)i * m.s_r;
    if (m.blk_r) o += (int64_t)(i / m.blk_r) * m.jump_r;
    return o;
}
__device__ __forceinline__ int64_t col_part(const Mat &m, int j) {
    int64_t o = (int64_t)j * m.s_c;
    if (m.blk_c) o += (int64_t)(j / m.blk_c) * m.jump_c;
    return o;
}

template <typename T> __device__ __forceinline__ float load_f32(const void *p, int64_t o) {
    return Elem<T>::f32(reinterpret_cast<const T *>(p)[o]);
}
template <typename T> __device__ __forceinline__ void store_f32(void *p, int64_t o, float v);
template <> __device__ __forceinline__ void store_f32<float>(void *p, int64_t o, float v) {
    reinterpret_cast<float *>(p)[o] = v;
}
template <> __device__ __forceinline__ void store_f32<__nv_bfloat16>(void *p, int64_t o, float v) {
    reinterpret_cast<__nv_bfloat16 *>(p)[o] = __float2bfloat16_rn(v);
}

// ------------------------------------------------------------------ fp32 GEMM
// C (M x N) = A (M x K) · B (K x N) per sequence (blockIdx.z).  128 x 128 tile per CTA,
// 16-deep slices of K staged in shared memory, 8 x 8 outputs per thread.  Loads follow
// whichever index of the operand is contiguous, so X and X^T are both read coalesced.
constexpr int GM = 128, GN = 128, GK = 16, G_THREADS = 256;

template <typename TA, typename TC>
__global__ void __launch_bounds__(G_THREADS) k_gemm(const Mat A, const Mat Bm, const Mat C,
                                                    int M, int N, int K) {
    __shared__ __align__(16) float As[GK][GM + 4];
    __shared__ __align__(16) float Bs[GK][GN + 4];
    const int tid = threadIdx.x, tx = tid % 16, ty = tid / 16;
    const int m0 = blockIdx.y * GM, n0 = blockIdx.x * GN, b = blockIdx.z;
    const bool a_kc = A.s_c == 1 && A.s_r != 1;   // K is A's contiguous index
    const bool b_nc = Bm.s_c == 1;                // N is B's contiguous index
    const int64_t a_b = (int64_t)b * A.s_b, b_b = (int64_t)b * Bm.s_b;
    float acc[8][8];
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] = 0.f;

    for (int k0 = 0; k0 < K; k0 += GK) {
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int e = tid + j * G_THREADS;
            const int mm = a_kc ? e / GK : e % GM, kk = a_kc ? e % GK : e / GM;
            const int gm = m0 + mm, gk = k0 + kk;
            As[kk][mm] = (gm < M && gk < K)
                             ? load_f32<TA>(A.p, a_b + row_part(A, gm) + col_part(A, gk))
                             : 0.f;
        }
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int e = tid + j * G_THREADS;
            const int nn = b_nc ? e % GN : e / GK, kk = b_nc ? e / GN : e % GK;
            const int gn = n0 + nn, gk = k0 + kk;
            Bs[kk][nn] = (gn < N && gk < K)
                             ? load_f32<float>(Bm.p, b_b + row_part(Bm, gk) + col_part(Bm, gn))
                             : 0.f;
        }
        __syncthreads();
#pragma unroll
        for (int kk = 0; kk < GK; ++kk) {
            const float4 a0 = *reinterpret_cast<const float4 *>(&As[kk][ty * 4]);
            const float4 a1 = *reinterpret_cast<const float4 *>(&As[kk][64 + ty * 4]);
            const float4 b0 = *reinterpret_cast<const float4 *>(&Bs[kk][tx * 4]);
            const float4 b1 = *reinterpret_cast<const float4 *>(&Bs[kk][64 + tx * 4]);
            const float av[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
            const float bv[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
            for (int i = 0; i < 8; ++i)
#pragma unroll
                for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
        }
        __syncthreads();
    }
    const int64_t c_b = (int64_t)b * C.s_b;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int gm = m0 + (i < 4 ? ty * 4 + i : 64 + ty * 4 + i - 4);
        if (gm >= M) continue;
        const int64_t ro = c_b + row_part(C, gm);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int gn = n0 + (j < 4 ? tx * 4 + j : 64 + tx * 4 + j - 4);
            if (gn < N) store_f32<TC>(const_cast<void *>(C.p), ro + col_part(C, gn), acc[i][j]);
        }
    }
}

// ------------------------------------------------------------------ fp64 Gram
// G[b] += Y[b]^T Y[b] over one slice of rows, for the 64 x 64 tiles on or above the
// diagonal (the Cholesky reads the upper triangle only).  fp32 x fp32 products are exact
// in fp64; the slices meet through fp64 atomics.
constexpr int GR_T = 64, GR_ROWS = 32;

__global__ void __launch_bounds__(256) k_gram(const float *__restrict__ Y, int rows, int r,
                                              int rows_per_split, int n_split,
                                              double *__restrict__ G) {
    const int ti = blockIdx.y, tj = blockIdx.x;
    if (tj < ti) return;
    const int b = blockIdx.z / n_split, sp = blockIdx.z % n_split;
    __shared__ float Yi[GR_ROWS][GR_T + 1], Yj[GR_ROWS][GR_T + 1];
    const int tid = threadIdx.x, tx = tid % 16, ty = tid / 16;
    const float *y = Y + (int64_t)b * rows * r;
    const int t_lo = sp * rows_per_split;
    const int t_hi = min(rows, t_lo + rows_per_split);
    double acc[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = 0.0;
    for (int t0 = t_lo; t0 < t_hi; t0 += GR_ROWS) {
        for (int e = tid; e < GR_ROWS * GR_T; e += 256) {
            const int tt = e / GR_T, c = e % GR_T, t = t0 + tt;
            const int ci = ti * GR_T + c, cj = tj * GR_T + c;
            Yi[tt][c] = (t < t_hi && ci < r) ? y[(int64_t)t * r + ci] : 0.f;
            Yj[tt][c] = (t < t_hi && cj < r) ? y[(int64_t)t * r + cj] : 0.f;
        }
        __syncthreads();
#pragma unroll 4
        for (int tt = 0; tt < GR_ROWS; ++tt) {
            double a[4], c[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) a[i] = (double)Yi[tt][ty * 4 + i];
#pragma unroll
            for (int j = 0; j < 4; ++j) c[j] = (double)Yj[tt][tx * 4 + j];
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[i][j] = fma(a[i], c[j], acc[i][j]);
        }
        __syncthreads();
    }
    double *g = G + (int64_t)b * r * r;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int gi = ti * GR_T + ty * 4 + i;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int gj = tj * GR_T + tx * 4 + j;
            if (gi < r && gj < r && gi <= gj) atomicAdd(&g[(int64_t)gi * r + gj], acc[i][j]);
        }
    }
}

// ------------------------------------------------- fp64 Cholesky and R^-1 (one CTA)
// G = R^T R with R upper triangular, in place on G's upper triangle (right-looking,
// one pivot at a time), then R^-1 by back substitution, one column per thread.  A pivot
// at or below `tol` marks a dependent column: its row of R and its column of R^-1 are
// zero.  Requires r <= CH_THREADS.
constexpr int CH_THREADS = 1024;

__global__ void __launch_bounds__(CH_THREADS) k_chol_inv(double *__restrict__ G, int r,
                                                         double *__restrict__ R64,
                                                         float *__restrict__ R32) {
    __shared__ double rowj[CH_THREADS];
    __shared__ double red[CH_THREADS / 32];
    __shared__ int s_dep;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    double *g = G + (int64_t)blockIdx.x * r * r;
    double *ri = R64 + (int64_t)blockIdx.x * r * r;
    float *ro = R32 + (int64_t)blockIdx.x * r * r;

    double mx = 0.0;
    for (int i = tid; i < r; i += CH_THREADS) mx = fmax(mx, g[(int64_t)i * r + i]);
#pragma unroll
    for (int off = 16; off; off >>= 1) mx = fmax(mx, __shfl_xor_sync(0xffffffffu, mx, off));
    if (lane == 0) red[warp] = mx;
    __syncthreads();
    mx = 0.0;
    for (int w = 0; w < CH_THREADS / 32; ++w) mx = fmax(mx, red[w]);
    const double tol = 1e-12 * mx;

    for (int j = 0; j < r; ++j) {
        if (tid == 0) {
            const double p = g[(int64_t)j * r + j];
            const int dep = !(p > tol);  // NaN counts as dependent too
            s_dep = dep;
            g[(int64_t)j * r + j] = dep ? 0.0 : sqrt(p);
        }
        __syncthreads();
        const int dep = s_dep;
        const double rjj = g[(int64_t)j * r + j];
        for (int c = j + 1 + tid; c < r; c += CH_THREADS) {
            const double v = dep ? 0.0 : g[(int64_t)j * r + c] / rjj;
            g[(int64_t)j * r + c] = v;
            rowj[c] = v;
        }
        __syncthreads();
        if (!dep) {
            const int n = r - j - 1;
            for (int e = tid; e < n * n; e += CH_THREADS) {
                const int i = j + 1 + e / n, c = j + 1 + e % n;
                if (i <= c) g[(int64_t)i * r + c] -= rowj[i] * rowj[c];
            }
        }
        __syncthreads();
    }

    for (int c = tid; c < r; c += CH_THREADS) {
        for (int i = r - 1; i >= 0; --i) {
            double x = 0.0;
            if (i <= c) {
                const double rii = g[(int64_t)i * r + i];
                if (rii != 0.0) {
                    double s = i == c ? 1.0 : 0.0;
                    for (int m = i + 1; m <= c; ++m)
                        s -= g[(int64_t)i * r + m] * ri[(int64_t)m * r + c];
                    x = s / rii;
                }
            }
            ri[(int64_t)i * r + c] = x;
            ro[(int64_t)i * r + c] = (float)x;
        }
    }
}

template <typename T>
__global__ void k_to_storage(const float *__restrict__ src, T *__restrict__ dst, int64_t n) {
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
         i += (int64_t)gridDim.x * blockDim.x)
        store_f32<T>(dst, i, src[i]);
}

// ------------------------------------------------------------------ host side
Mat dense(const void *p, int64_t rows, int64_t cols) {
    Mat m{};
    m.p = p;
    m.s_r = cols;
    m.s_c = 1;
    m.s_b = rows * cols;
    return m;
}

template <typename TA, typename TC>
cudaError_t gemm(const Mat &A, const Mat &B, const Mat &C, int M, int N, int K, int batch,
                 cudaStream_t s) {
    const dim3 grid((N + GN - 1) / GN, (M + GM - 1) / GM, batch);
    k_gemm<TA, TC><<<grid, G_THREADS, 0, s>>>(A, B, C, M, N, K);
    return cudaGetLastError();
}

struct Scratch {
    float *y[2], *z[2];
    double *g, *r64;
    float *r32;
};

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

Scratch carve(void *ws, int64_t B, int64_t L, int64_t n, int64_t r) {
    char *p = (char *)ws;
    Scratch s;
    for (int i = 0; i < 2; ++i) {
        s.y[i] = (float *)p;
        p += align256((size_t)B * L * r * 4);
    }
    for (int i = 0; i < 2; ++i) {
        s.z[i] = (float *)p;
        p += align256((size_t)B * n * r * 4);
    }
    s.g = (double *)p;
    p += align256((size_t)B * r * r * 8);
    s.r64 = (double *)p;
    p += align256((size_t)B * r * r * 8);
    s.r32 = (float *)p;
    return s;
}

// CholeskyQR2 of the `rows` x r matrices of every sequence in buf[0]; buf[1] is the
// other half of the ping-pong, and the result ends in buf[0].
cudaError_t orth(float *const buf[2], int64_t rows, int r, int B, const Scratch &sc,
                 cudaStream_t s) {
    const int T = (r + GR_T - 1) / GR_T;
    int n_split = (int)((rows + 1023) / 1024);
    const int cap = 65535 / B;
    if (n_split > cap) n_split = cap;
    const int rps = (int)((rows + n_split - 1) / n_split);
    for (int pass = 0; pass < 2; ++pass) {
        float *src = buf[pass], *dst = buf[pass ^ 1];
        cudaError_t e = cudaMemsetAsync(sc.g, 0, (size_t)B * r * r * sizeof(double), s);
        if (e != cudaSuccess) return e;
        k_gram<<<dim3(T, T, B * n_split), 256, 0, s>>>(src, (int)rows, r, rps, n_split, sc.g);
        k_chol_inv<<<B, CH_THREADS, 0, s>>>(sc.g, r, sc.r64, sc.r32);
        Mat Rm = dense(sc.r32, r, r);
        e = gemm<float, float>(dense(src, rows, r), Rm, dense(dst, rows, r), (int)rows, r, r,
                               B, s);
        if (e != cudaSuccess) return e;
    }
    return cudaGetLastError();
}

template <typename T>
cudaError_t factorize_t(const xkv_dims &d, int W, int r, const void *X, const float *omega,
                        int n_iter, void *A_out, void *Bt_out, void *ws, cudaStream_t s) {
    const int B = d.batch;
    const int64_t L = d.ctx_len, dk = (int64_t)d.n_kv_heads * d.head_dim, n = W * dk;
    const Scratch sc = carve(ws, B, L, n, r);
    // X as L x n (token rows, layer-major feature columns) and as its transpose
    Mat Xr{};
    Xr.p = X;
    Xr.s_r = dk;
    Xr.s_c = 1;
    Xr.s_b = L * dk;
    Xr.blk_c = (int32_t)dk;
    Xr.jump_c = (int64_t)B * L * dk - dk;
    Mat Xt{};
    Xt.p = X;
    Xt.s_r = 1;
    Xt.s_c = dk;
    Xt.s_b = L * dk;
    Xt.blk_r = (int32_t)dk;
    Xt.jump_r = (int64_t)B * L * dk - dk;
    Mat Om = dense(omega, n, r);
    Om.s_b = 0;
    const Mat Y = dense(sc.y[0], L, r), Z = dense(sc.z[0], n, r);

    cudaError_t e = gemm<T, float>(Xr, Om, Y, (int)L, r, (int)n, B, s);
    if (e == cudaSuccess) e = orth(sc.y, L, r, B, sc, s);
    for (int it = 0; it < n_iter && e == cudaSuccess; ++it) {
        e = gemm<T, float>(Xt, Y, Z, (int)n, r, (int)L, B, s);
        if (e == cudaSuccess) e = orth(sc.z, n, r, B, sc, s);
        if (e == cudaSuccess) e = gemm<T, float>(Xr, Z, Y, (int)L, r, (int)n, B, s);
        if (e == cudaSuccess) e = orth(sc.y, L, r, B, sc, s);
    }
    if (e != cudaSuccess) return e;
    const int64_t na = (int64_t)B * L * r;
    k_to_storage<T><<<(int)((na + 255) / 256 < 65535 ? (na + 255) / 256 : 65535), 256, 0, s>>>(
        sc.y[0], (T *)A_out, na);
    // B_l^T = X_l^T A, written as [W][B][d_kv][r]
    Mat Bt{};
    Bt.p = Bt_out;
    Bt.s_r = r;
    Bt.s_c = 1;
    Bt.s_b = dk * r;
    Bt.blk_r = (int32_t)dk;
    Bt.jump_r = ((int64_t)B * dk - dk) * r;
    return gemm<T, T>(Xt, Y, Bt, (int)n, r, (int)L, B, s);
}

}  // namespace

size_t factorize_ws_bytes(const xkv_dims &d, int W, int r) {
    const int64_t B = d.batch, L = d.ctx_len, n = (int64_t)W * d.n_kv_heads * d.head_dim;
    return 2 * align256((size_t)B * L * r * 4) + 2 * align256((size_t)B * n * r * 4) +
           2 * align256((size_t)B * r * r * 8) + align256((size_t)B * r * r * 4);
}

cudaError_t launch_factorize(const xkv_dims &d, int W, int r, const void *X, const float *omega,
                             int n_iter, void *A_out, void *Bt_out, void *ws, cudaStream_t s) {
    return d.dtype == XKV_F32
               ? factorize_t<float>(d, W, r, X, omega, n_iter, A_out, Bt_out, ws, s)
               : factorize_t<__nv_bfloat16>(d, W, r, X, omega, n_iter, A_out, Bt_out, ws, s);
}

}  // namespace xkv
