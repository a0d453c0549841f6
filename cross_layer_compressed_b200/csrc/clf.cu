// Cross-layer factorization of one window (xKV page, section 2.2: the caches of the W
// layers of a window are concatenated side by side, a rank-r SVD of the concatenation
// gives one token basis A shared by the window and one reconstruction matrix B_l per
// layer, so that A·B_l stands in for layer l's cache).
//
// Per sequence the concatenation X = [X_0 | ... | X_{W-1}] (L x n, n = W·d_kv) is never
// built: every product runs layer by layer on the W cache buffers.  The rank-r
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
// orth() is CholeskyQR: G = Y^T Y (fp64), G = R^T R (blocked Cholesky, fp64), Y <- Y R^-1
// (R^-1 by blocked triangular inversion, fp64); twice (CholeskyQR2) for the returned
// basis, once for the intermediate ones, which only have to stay well conditioned.  A column whose Cholesky
// pivot is below 1e-12 of the largest diagonal entry of G (a direction the data does
// not have: rank(X) < r) is zeroed rather than normalised.
//
// The large products run in gemm.cu on the tensor cores: for bf16 caches the fp32
// operand (Q, Z) is split into bf16 hi + lo parts (about 16 significant bits; the test
// matrix is used at bf16 precision, which only makes it another test matrix) and the
// products with R^-1 use TF32; for fp32 caches every product is a plain fp32 product on
// the CUDA cores.  The Gram matrices, the Cholesky factorization and the inversion are
// this file's own fp64 kernels.
//
// Device-side failures (a bounded wait of a product kernel that gave up) set bits in the
// status word at the start of the workspace; the factors are then written as NaN.
#include <cuda_runtime.h>

#include "xkv_internal.cuh"

namespace xkv {
namespace {

constexpr int NB = 64;         // block size of the Cholesky factorization and inversion
constexpr int NBP = NB + 1;    // padded shared-memory row

// ------------------------------------------------------------------ fp64 Gram
// G[b] += Y[b]^T Y[b] over one slice of rows, for the 128 x 128 tiles on or above the
// diagonal (the factorization reads the upper triangle only), on the fp64 tensor cores:
// mma.sync m8n8k4 f64 (exact fp32 x fp32 products, fp64 accumulation; the order of the
// fp64 sums is the tensor core's, which only rounding sees).  16 warps, each owning a
// 32 x 32 block of the tile as 4 x 4 fragments of 8 x 8; 16-row slices of the tile's two
// column blocks are staged in shared memory already widened to fp64 (rows padded by 4
// doubles), the next slice waiting in registers.  The slices of rows meet through fp64
// atomics.
constexpr int GR_T = 128, GR_ROWS = 16, GR_THREADS = 512, GR_PAD = GR_T + 4;

__global__ void __launch_bounds__(GR_THREADS, 1) k_gram(const float *__restrict__ Y, int rows,
                                                        int r, int rows_per_split, int n_split,
                                                        double *__restrict__ G) {
    const int ti = blockIdx.y, tj = blockIdx.x;
    if (tj < ti) return;
    const int b = blockIdx.z / n_split, sp = blockIdx.z % n_split;
    __shared__ __align__(16) double Yi[GR_ROWS][GR_PAD], Yj[GR_ROWS][GR_PAD];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int wi = (warp >> 2) * 32, wj = (warp & 3) * 32;   // the warp's 32 x 32 block
    const int fr = lane >> 2, fk = lane & 3;                 // fragment row / k of this lane
    const float *y = Y + (int64_t)b * rows * r;
    const int t_lo = sp * rows_per_split;
    const int t_hi = min(rows, t_lo + rows_per_split);
    double acc[4][4][2];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j][0] = acc[i][j][1] = 0.0;
    constexpr int PER = GR_ROWS * GR_T / GR_THREADS;   // 4
    float ni[PER], nj[PER];
    auto fetch = [&](int t0) {
#pragma unroll
        for (int u = 0; u < PER; ++u) {
            const int e = tid + u * GR_THREADS, tt = e / GR_T, c = e % GR_T, t = t0 + tt;
            const int ci = ti * GR_T + c, cj = tj * GR_T + c;
            ni[u] = (t < t_hi && ci < r) ? y[(int64_t)t * r + ci] : 0.f;
            nj[u] = (t < t_hi && cj < r) ? y[(int64_t)t * r + cj] : 0.f;
        }
    };
    fetch(t_lo);
    for (int t0 = t_lo; t0 < t_hi; t0 += GR_ROWS) {
#pragma unroll
        for (int u = 0; u < PER; ++u) {
            const int e = tid + u * GR_THREADS, tt = e / GR_T, c = e % GR_T;
            Yi[tt][c] = (double)ni[u];
            Yj[tt][c] = (double)nj[u];
        }
        __syncthreads();
        if (t0 + GR_ROWS < t_hi) fetch(t0 + GR_ROWS);
#pragma unroll
        for (int k0 = 0; k0 < GR_ROWS; k0 += 4) {
            // A[i][k] = Y[t0 + k][i], B[k][j] = Y[t0 + k][j]: lane (fr, fk) holds
            // A[fr][fk] and B[fk][fr] of each 8-wide fragment
            double a[4], c[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) a[i] = Yi[k0 + fk][wi + 8 * i + fr];
#pragma unroll
            for (int j = 0; j < 4; ++j) c[j] = Yj[k0 + fk][wj + 8 * j + fr];
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    asm volatile(
                        "mma.sync.aligned.m8n8k4.row.col.f64.f64.f64.f64 {%0, %1}, {%2}, {%3}, "
                        "{%0, %1};"
                        : "+d"(acc[i][j][0]), "+d"(acc[i][j][1])
                        : "d"(a[i]), "d"(c[j]));
        }
        __syncthreads();
    }
    double *g = G + (int64_t)b * r * r;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int gi = ti * GR_T + wi + 8 * i + fr;
#pragma unroll
        for (int j = 0; j < 4; ++j)
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                // accumulator (row fr, column 2 fk + h) of fragment (i, j)
                const int gj = tj * GR_T + wj + 8 * j + 2 * fk + h;
                if (gi < r && gj < r && gi <= gj) atomicAdd(&g[(int64_t)gi * r + gj], acc[i][j][h]);
            }
    }
}

// ------------------------------------------- blocked Cholesky G = R^T R (fp64)
// Per sequence the pivot tolerance: 1e-12 of the largest diagonal entry of G.
__global__ void __launch_bounds__(256) k_maxdiag(const double *__restrict__ G, int r,
                                                 double *__restrict__ tol) {
    __shared__ double red[8];
    const double *g = G + (int64_t)blockIdx.x * r * r;
    double mx = 0.0;
    for (int i = threadIdx.x; i < r; i += 256) mx = fmax(mx, g[(int64_t)i * r + i]);
#pragma unroll
    for (int off = 16; off; off >>= 1) mx = fmax(mx, __shfl_xor_sync(0xffffffffu, mx, off));
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = mx;
    __syncthreads();
    if (threadIdx.x == 0) {
        mx = red[0];
        for (int w = 1; w < 8; ++w) mx = fmax(mx, red[w]);
        tol[blockIdx.x] = 1e-12 * mx;
    }
}

// Diagonal block k: unblocked right-looking Cholesky in shared memory (one thread per
// column), then the block's inverse D_k = R_kk^-1 by back substitution.  A dependent
// pivot gives a zero row of R and a zero row and column of D_k.
__global__ void __launch_bounds__(256) k_potrf_diag(double *__restrict__ G, int r, int k,
                                                    const double *__restrict__ tol,
                                                    double *__restrict__ D) {
    extern __shared__ double sm[];
    double (*a)[NBP] = reinterpret_cast<double (*)[NBP]>(sm);
    double (*di)[NBP] = reinterpret_cast<double (*)[NBP]>(sm + NB * NBP);
    __shared__ int s_dep;
    const int b = blockIdx.x, tid = threadIdx.x, o = k * NB;
    const int bk = min(NB, r - o);
    double *g = G + (int64_t)b * r * r;
    for (int e = tid; e < NB * NB; e += blockDim.x) {       // coalesced block copy
        const int p = e / NB, c = e % NB;
        a[p][c] = (p < bk && c < bk && p <= c) ? g[(int64_t)(o + p) * r + o + c] : 0.0;
    }
    const double t = tol[b];
    __syncthreads();
    // four threads per column: thread 4c + q updates rows i = q (mod 4) of column c
    const int c = tid >> 2, q = tid & 3;
    for (int j = 0; j < bk; ++j) {
        if (tid == 0) {
            const double pv = a[j][j];
            const int dep = !(pv > t);  // NaN counts as dependent too
            s_dep = dep;
            a[j][j] = dep ? 0.0 : sqrt(pv);
        }
        __syncthreads();
        const int dep = s_dep;
        if (q == 0 && c > j && c < bk) a[j][c] = dep ? 0.0 : a[j][c] / a[j][j];
        __syncthreads();
        if (!dep && c > j && c < bk)
            for (int i = j + 1 + q; i <= c; i += 4) a[i][c] -= a[j][i] * a[j][c];
        __syncthreads();
    }
    // D = R_kk^-1 by back substitution, all 64 columns at once: four adjacent lanes per
    // column split each dot product
    {
        const int cc = tid >> 2, q = tid & 3;
        for (int i = NB - 1; i >= 0; --i) {
            double part = 0.0;
            if (i < cc)
                for (int m = i + 1 + q; m <= cc; m += 4) part += a[i][m] * di[m][cc];
            part += __shfl_xor_sync(0xffffffffu, part, 1);
            part += __shfl_xor_sync(0xffffffffu, part, 2);
            double x = 0.0;
            if (i <= cc && cc < bk && a[i][i] != 0.0) x = ((i == cc ? 1.0 : 0.0) - part) / a[i][i];
            if (q == 0) di[i][cc] = x;
            __syncwarp();
        }
    }
    __syncthreads();
    double *dk = D + ((int64_t)b * ((r + NB - 1) / NB) + k) * NB * NB;
    for (int e = tid; e < NB * NB; e += blockDim.x) {
        const int p = e / NB, q = e % NB;
        dk[e] = di[p][q];
        if (p < bk && q < bk && p <= q) g[(int64_t)(o + p) * r + o + q] = a[p][q];
    }
}

// 64 x 64 block product: acc[i][j] += sum_q Lm[q][row_i] * Rm[q][col_j] (the left
// operand stored transposed) over q < nq, for the thread's 4 x 4 outputs.
__device__ __forceinline__ void mm_tn(const double (*Lm)[NBP], const double (*Rm)[NBP], int nq,
                                      int ty, int tx, double acc[4][4]) {
    for (int q = 0; q < nq; ++q) {
        double a[4], c[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) a[i] = Lm[q][ty * 4 + i];
#pragma unroll
        for (int j = 0; j < 4; ++j) c[j] = Rm[q][tx * 4 + j];
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j) acc[i][j] = fma(a[i], c[j], acc[i][j]);
    }
}

__device__ __forceinline__ void load_block(double (*dst)[NBP], const double *src, int64_t ld,
                                           int rows, int cols) {
    for (int e = threadIdx.x; e < NB * NB; e += blockDim.x) {
        const int p = e / NB, c = e % NB;
        dst[p][c] = (p < rows && c < cols) ? src[(int64_t)p * ld + c] : 0.0;
    }
}

// Row panel of block row k: R_kj = D_k^T G_kj for every block column j > k.
__global__ void __launch_bounds__(256) k_trsm_panel(double *__restrict__ G, int r, int k,
                                                    const double *__restrict__ D) {
    extern __shared__ double sm[];
    double (*dv)[NBP] = reinterpret_cast<double (*)[NBP]>(sm);
    double (*gb)[NBP] = reinterpret_cast<double (*)[NBP]>(sm + NB * NBP);
    const int b = blockIdx.y, J = k + 1 + blockIdx.x;
    const int KB = (r + NB - 1) / NB;
    const int o = k * NB, oj = J * NB, bk = min(NB, r - o), bj = min(NB, r - oj);
    double *g = G + (int64_t)b * r * r;
    load_block(dv, D + ((int64_t)b * KB + k) * NB * NB, NB, NB, NB);
    load_block(gb, g + (int64_t)o * r + oj, r, bk, bj);
    __syncthreads();
    const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
    double acc[4][4] = {};
    mm_tn(dv, gb, bk, ty, tx, acc);  // out[p][c] = sum_q D[q][p] G[q][c]
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int p = ty * 4 + i, c = tx * 4 + j;
            if (p < bk && c < bj) g[(int64_t)(o + p) * r + oj + c] = acc[i][j];
        }
}

// Trailing update after block row k: G_IJ -= R_kI^T R_kJ for k < I <= J.
__global__ void __launch_bounds__(256) k_syrk_update(double *__restrict__ G, int r, int k) {
    extern __shared__ double sm[];
    double (*ri)[NBP] = reinterpret_cast<double (*)[NBP]>(sm);
    double (*rj)[NBP] = reinterpret_cast<double (*)[NBP]>(sm + NB * NBP);
    const int b = blockIdx.y;
    const int KB = (r + NB - 1) / NB, m = KB - k - 1;
    int I = 0, rem = blockIdx.x;            // blockIdx.x -> (I, J), 0 <= I <= J < m
    while (rem >= m - I) {
        rem -= m - I;
        ++I;
    }
    const int J = I + rem + k + 1;
    I += k + 1;
    const int o = k * NB, oi = I * NB, oj = J * NB;
    const int bk = min(NB, r - o), bi = min(NB, r - oi), bj = min(NB, r - oj);
    double *g = G + (int64_t)b * r * r;
    load_block(ri, g + (int64_t)o * r + oi, r, bk, bi);
    load_block(rj, g + (int64_t)o * r + oj, r, bk, bj);
    __syncthreads();
    const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
    double acc[4][4] = {};
    mm_tn(ri, rj, bk, ty, tx, acc);
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int p = ty * 4 + i, c = tx * 4 + j;
            if (p < bi && c < bj) g[(int64_t)(oi + p) * r + oj + c] -= acc[i][j];
        }
}

// Block row i of R^-1 (the block rows below it are done):
//   X_ii = D_i,  X_iJ = -D_i sum_{K=i+1..J} R_iK X_KJ  (J > i).
__global__ void __launch_bounds__(256) k_trinv_row(const double *__restrict__ G, int r, int i,
                                                   const double *__restrict__ D,
                                                   double *__restrict__ X64,
                                                   float *__restrict__ X32) {
    extern __shared__ double sm[];
    double (*s0)[NBP] = reinterpret_cast<double (*)[NBP]>(sm);
    double (*s1)[NBP] = reinterpret_cast<double (*)[NBP]>(sm + NB * NBP);
    const int b = blockIdx.y, J = i + blockIdx.x;
    const int KB = (r + NB - 1) / NB;
    const int oi = i * NB, oj = J * NB, bi = min(NB, r - oi), bj = min(NB, r - oj);
    const double *g = G + (int64_t)b * r * r;
    double *x = X64 + (int64_t)b * r * r;
    float *x32 = X32 + (int64_t)b * r * r;
    const double *di = D + ((int64_t)b * KB + i) * NB * NB;
    const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
    double acc[4][4] = {};
    if (J == i) {
#pragma unroll
        for (int a = 0; a < 4; ++a)
#pragma unroll
            for (int c = 0; c < 4; ++c) acc[a][c] = di[(ty * 4 + a) * NB + tx * 4 + c];
    } else {
        // T = sum_K R_iK X_KJ, R_iK loaded transposed so that mm_tn applies
        for (int K = i + 1; K <= J; ++K) {
            const int oK = K * NB, bK = min(NB, r - oK);
            for (int e = threadIdx.x; e < NB * NB; e += blockDim.x) {
                const int q = e / NB, p = e % NB;  // s0[q][p] = R[oi + p][oK + q]
                s0[q][p] = (p < bi && q < bK) ? g[(int64_t)(oi + p) * r + oK + q] : 0.0;
            }
            load_block(s1, x + (int64_t)oK * r + oj, r, bK, bj);
            __syncthreads();
            mm_tn(s0, s1, bK, ty, tx, acc);
            __syncthreads();
        }
        // X_iJ = -D_i T: T to shared memory, D_i transposed beside it
#pragma unroll
        for (int a = 0; a < 4; ++a)
#pragma unroll
            for (int c = 0; c < 4; ++c) s1[ty * 4 + a][tx * 4 + c] = acc[a][c];
        for (int e = threadIdx.x; e < NB * NB; e += blockDim.x) {
            const int q = e / NB, p = e % NB;  // s0[q][p] = D_i[p][q]
            s0[q][p] = di[p * NB + q];
        }
        __syncthreads();
        double out[4][4] = {};
        mm_tn(s0, s1, NB, ty, tx, out);
#pragma unroll
        for (int a = 0; a < 4; ++a)
#pragma unroll
            for (int c = 0; c < 4; ++c) acc[a][c] = -out[a][c];
    }
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            const int p = ty * 4 + a, q = tx * 4 + c;
            if (p < bi && q < bj) {
                x[(int64_t)(oi + p) * r + oj + q] = acc[a][c];
                x32[(int64_t)(oj + q) * r + oi + p] = (float)acc[a][c];   // transposed
            }
        }
}

// ------------------------------------------------------------ small elementwise kernels
// x = hi + lo with hi = bf16(x) and lo = bf16(x - hi): about 16 significant bits.
__global__ void k_split_hi_lo(const float *__restrict__ src, __nv_bfloat16 *__restrict__ hi,
                              __nv_bfloat16 *__restrict__ lo, int64_t n) {
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
         i += (int64_t)gridDim.x * blockDim.x) {
        const float x = src[i];
        const __nv_bfloat16 h = __float2bfloat16_rn(x);
        hi[i] = h;
        lo[i] = __float2bfloat16_rn(x - __bfloat162float(h));
    }
}

template <typename T> __device__ __forceinline__ T from_f32(float v);
template <> __device__ __forceinline__ float from_f32<float>(float v) { return v; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float v) {
    return __float2bfloat16_rn(v);
}

template <typename T>
__global__ void k_to_storage(const float *__restrict__ src, T *__restrict__ dst, int64_t n,
                             const unsigned *__restrict__ status) {
    const bool failed = *status != 0u;           // a failed call leaves NaN factors
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
         i += (int64_t)gridDim.x * blockDim.x)
        dst[i] = from_f32<T>(failed ? __int_as_float(0x7fc00000) : src[i]);
}

// Z [B][W·d_kv][r] (fp32) -> Bt [W][B][d_kv][r] (storage dtype)
template <typename T>
__global__ void k_store_bt(const float *__restrict__ Z, T *__restrict__ Bt, int B, int W,
                           int64_t dk, int r, const unsigned *__restrict__ status) {
    const bool failed = *status != 0u;
    const int64_t total = (int64_t)B * W * dk * r;
    for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < total;
         e += (int64_t)gridDim.x * blockDim.x) {
        const int64_t i = e % r, j = (e / r) % dk, l = (e / (r * dk)) % W, b = e / (r * dk * W);
        Bt[((l * B + b) * dk + j) * r + i] = from_f32<T>(failed ? __int_as_float(0x7fc00000) : Z[e]);
    }
}

int grid_for(int64_t n) {
    const int64_t g = (n + 255) / 256;
    return (int)(g < 8192 ? (g > 0 ? g : 1) : 8192);
}

// ------------------------------------------------------------------ host side
size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

struct Scratch {
    unsigned *status;       // device-side failures of the call (bits 1 << xkv_status)
    float *y[2], *z[2];
    double *g, *d, *r64, *tol;
    float *r32;             // R^-1 transposed, fp32
    __nv_bfloat16 *hi, *lo, *om_hi;
};

struct Shape {
    int B, W, r;
    int64_t L, dk, n;
    bool bf16;
};

Shape shape_of(const xkv_dims &d, int W, int r) {
    Shape s;
    s.B = d.batch;
    s.W = W;
    s.r = r;
    s.L = d.ctx_len;
    s.dk = (int64_t)d.n_kv_heads * d.head_dim;
    s.n = W * s.dk;
    s.bf16 = d.dtype == XKV_BF16;
    return s;
}

// Lays the scratch out in ws (when given) and returns its size: a 256-byte header holding
// the status word, then the bases and the small factors.
size_t carve(const Shape &s, void *ws, Scratch *out) {
    char *p = (char *)ws;
    size_t off = 0;
    auto take = [&](size_t bytes) {
        char *q = p ? p + off : nullptr;
        off += align256(bytes);
        return q;
    };
    const int64_t B = s.B, r = s.r, KB = (r + NB - 1) / NB;
    const int64_t rows_max = s.L > s.n ? s.L : s.n;
    Scratch sc{};
    sc.status = (unsigned *)take(256);
    for (int i = 0; i < 2; ++i) sc.y[i] = (float *)take((size_t)B * s.L * r * 4);
    for (int i = 0; i < 2; ++i) sc.z[i] = (float *)take((size_t)B * s.n * r * 4);
    sc.g = (double *)take((size_t)B * r * r * 8);
    sc.d = (double *)take((size_t)B * KB * NB * NB * 8);
    sc.r64 = (double *)take((size_t)B * r * r * 8);
    sc.tol = (double *)take((size_t)B * 8);
    sc.r32 = (float *)take((size_t)B * r * r * 4);
    if (s.bf16) {
        sc.hi = (__nv_bfloat16 *)take((size_t)B * rows_max * r * 2);
        sc.lo = (__nv_bfloat16 *)take((size_t)B * rows_max * r * 2);
        sc.om_hi = (__nv_bfloat16 *)take((size_t)s.n * r * 2);
    }
    if (out) *out = sc;
    return off;
}

struct Run {
    Shape s;
    Scratch sc;
    cudaStream_t st;
    const void *X;
    cudaError_t err = cudaSuccess;

    bool ok() const { return err == cudaSuccess; }
    void check(cudaError_t e) {
        if (e != cudaSuccess && err == cudaSuccess) err = e;
    }

    void split(const float *src, int64_t n) {
        k_split_hi_lo<<<grid_for(n), 256, 0, st>>>(src, sc.hi, sc.lo, n);
        check(cudaGetLastError());
    }

    GemmDesc base(int mode) const {
        GemmDesc g{};
        g.mode = mode;
        g.tc = s.bf16;
        g.nb = s.B;
        g.nl = 1;
        g.P = 1;
        g.n_seg = 1;
        g.L = s.L;
        g.dk = s.dk;
        g.r = s.r;
        g.n_rows = s.n;
        g.W = s.W;
        g.status = sc.status;
        return g;
    }

    // Y = sum_l X_l F_l, F [B][n][r] fp32; F == nullptr: the test matrix (shared by the
    // sequences; bf16 caches read its bf16 copy).  One product: the layers (and the hi /
    // lo parts of F) are consecutive K segments of one accumulation.
    void x_times(const float *F, const float *omega, float *Y) {
        GemmDesc g = base(GM_XF);
        g.M = (int)s.L;
        g.N = s.r;
        g.K_seg = s.dk;
        g.A = X;
        if (s.bf16) {
            if (F) {
                split(F, (int64_t)s.B * s.n * s.r);
                g.P = 2;
                g.B0 = sc.hi;
                g.B1 = sc.lo;
            } else {
                g.B0 = sc.om_hi;
                g.b_shared = 1;
            }
        } else {
            g.B0 = F ? F : omega;
            g.b_shared = F ? 0 : 1;
        }
        g.n_seg = s.W * g.P;
        g.C = Y;
        g.ldc = s.r;
        g.c_b = s.L * s.r;
        if (ok()) check(launch_gemm(g, st));
    }

    // Z_l = X_l^T Q for every layer: Z [B][n][r] fp32 (the hi and lo parts of Q are two K
    // segments of one accumulation)
    void xt_times(const float *Q, float *Z) {
        GemmDesc g = base(GM_XT);
        g.M = (int)s.dk;
        g.N = s.r;
        g.nl = s.W;
        g.K_seg = s.L;
        g.A = X;
        if (s.bf16) {
            split(Q, (int64_t)s.B * s.L * s.r);
            g.P = 2;
            g.B0 = sc.hi;
            g.B1 = sc.lo;
        } else {
            g.B0 = Q;
        }
        g.n_seg = g.P;
        g.C = Z;
        g.ldc = s.r;
        g.c_b = s.n * s.r;
        g.c_l = s.dk * s.r;
        if (ok()) check(launch_gemm(g, st));
    }

    // CholeskyQR of the rows x r matrices in buf[0] (buf[1]: the other ping-pong half),
    // `passes` times (2: CholeskyQR2); the result ends in buf[0]
    void orth(float *buf[2], int64_t rows, int passes) {
        const int B = s.B, r = s.r, KB = (r + NB - 1) / NB, T = (r + GR_T - 1) / GR_T;
        int n_split = (int)((rows + 1023) / 1024);
        const int cap = 65535 / B;
        if (n_split > cap) n_split = cap;
        const int rps = (int)((rows + n_split - 1) / n_split);
        const size_t blk_smem = 2 * NB * NBP * sizeof(double);
        for (int pass = 0; pass < passes && ok(); ++pass) {
            float *src = buf[0], *dst = buf[1];
            check(cudaMemsetAsync(sc.g, 0, (size_t)B * r * r * sizeof(double), st));
            check(cudaMemsetAsync(sc.r64, 0, (size_t)B * r * r * sizeof(double), st));
            check(cudaMemsetAsync(sc.r32, 0, (size_t)B * r * r * sizeof(float), st));
            k_gram<<<dim3(T, T, B * n_split), GR_THREADS, 0, st>>>(src, (int)rows, r, rps,
                                                                   n_split, sc.g);
            k_maxdiag<<<B, 256, 0, st>>>(sc.g, r, sc.tol);
            for (int k = 0; k < KB; ++k) {
                k_potrf_diag<<<B, 256, blk_smem, st>>>(sc.g, r, k, sc.tol, sc.d);
                const int m = KB - k - 1;
                if (m > 0) {
                    k_trsm_panel<<<dim3(m, B), 256, blk_smem, st>>>(sc.g, r, k, sc.d);
                    k_syrk_update<<<dim3(m * (m + 1) / 2, B), 256, blk_smem, st>>>(sc.g, r, k);
                }
            }
            for (int i = KB - 1; i >= 0; --i)
                k_trinv_row<<<dim3(KB - i, B), 256, blk_smem, st>>>(sc.g, r, i, sc.d, sc.r64,
                                                                    sc.r32);
            check(cudaGetLastError());
            if (!ok()) return;
            // dst = src R^-1 (TF32 on the tensor cores for bf16 caches)
            GemmDesc g = base(GM_APPLY);
            g.M = (int)rows;
            g.N = r;
            g.K_seg = r;
            g.L = rows;
            g.A = src;
            g.B0 = sc.r32;
            g.C = dst;
            g.ldc = r;
            g.c_b = rows * r;
            check(launch_gemm(g, st));
            buf[0] = dst;
            buf[1] = src;
        }
    }
};

cudaError_t set_block_smem() {
    const size_t bytes = 2 * NB * NBP * sizeof(double);
    cudaError_t e = set_smem_limit((const void *)k_potrf_diag, bytes);
    if (e == cudaSuccess) e = set_smem_limit((const void *)k_trsm_panel, bytes);
    if (e == cudaSuccess) e = set_smem_limit((const void *)k_syrk_update, bytes);
    if (e == cudaSuccess) e = set_smem_limit((const void *)k_trinv_row, bytes);
    return e;
}

// clear_status: false when the caller (the refold) already cleared the call's status word
template <typename T>
cudaError_t factorize_t(const Shape &s, const void *X, const float *omega, int n_iter,
                        void *A_out, void *Bt_out, void *ws, cudaStream_t st, bool clear_status) {
    cudaError_t e = set_block_smem();
    if (e != cudaSuccess) return e;
    Run run;
    run.s = s;
    carve(s, ws, &run.sc);
    run.st = st;
    run.X = X;
    const int B = s.B, r = s.r;
    const Scratch &sc = run.sc;  // y[0] / z[0] follow the ping-pong of orth()
    if (clear_status) run.check(cudaMemsetAsync(sc.status, 0, sizeof(unsigned), st));

    if (s.bf16) {
        k_split_hi_lo<<<grid_for(s.n * r), 256, 0, st>>>(omega, sc.om_hi, sc.lo, s.n * r);
        run.check(cudaGetLastError());
    }
    // The intermediate bases only have to stay well conditioned: one CholeskyQR pass
    // each; the final basis (the returned A) gets two.
    Scratch &sw = run.sc;
    run.x_times(nullptr, omega, sw.y[0]);
    if (run.ok()) run.orth(sw.y, s.L, n_iter == 0 ? 2 : 1);
    for (int it = 0; it < n_iter && run.ok(); ++it) {
        run.xt_times(sw.y[0], sw.z[0]);
        if (run.ok()) run.orth(sw.z, s.n, 1);
        if (run.ok()) run.x_times(sw.z[0], omega, sw.y[0]);
        if (run.ok()) run.orth(sw.y, s.L, it == n_iter - 1 ? 2 : 1);
    }
    if (run.ok()) {
        const int64_t na = (int64_t)B * s.L * r;
        k_to_storage<T><<<grid_for(na), 256, 0, st>>>(sc.y[0], (T *)A_out, na, sc.status);
        run.check(cudaGetLastError());
        run.xt_times(sc.y[0], sc.z[0]);
        const int64_t nb = (int64_t)B * s.n * r;
        if (run.ok())
            k_store_bt<T><<<grid_for(nb), 256, 0, st>>>(sc.z[0], (T *)Bt_out, B, s.W, s.dk, r,
                                                         sc.status);
        run.check(cudaGetLastError());
    }
    return run.err;
}

// Refold (the decode loop's tail of generated rows folded back into the factors): the
// extended caches [A·B_l ; tail_l] are built in the workspace after the factorization's
// scratch -- the reconstruction in the storage type, as the decode calls would see it --
// and factored again.
template <typename T>
cudaError_t refold_t(const Shape &s, int64_t n_tail, const void *A, const void *Bt,
                     const void *tail, const float *omega, int n_iter, void *A_out,
                     void *Bt_out, void *ws, cudaStream_t st) {
    const int64_t L = s.L - n_tail, e = sizeof(T);
    Scratch sc{};
    const size_t fac_bytes = carve(s, ws, &sc);
    char *xbuf = (char *)ws + fac_bytes;
    cudaError_t c = cudaMemsetAsync(sc.status, 0, sizeof(unsigned), st);
    if (c != cudaSuccess) return c;
    // X'_l[b][0:L] = A_b B_l,b for every layer (B_l stored column-major: Bt_l,b d_kv x r)
    GemmDesc g{};
    g.mode = GM_REFOLD;
    g.tc = s.bf16;
    g.M = (int)L;
    g.N = (int)s.dk;
    g.nb = s.B;
    g.nl = s.W;
    g.n_seg = 1;
    g.P = 1;
    g.K_seg = s.r;
    g.A = A;
    g.B0 = Bt;
    g.L = L;
    g.dk = s.dk;
    g.r = s.r;
    g.n_rows = s.n;
    g.W = s.W;
    g.C = xbuf;
    g.c_bf16 = s.bf16;
    g.ldc = s.dk;
    g.c_b = s.L * s.dk;
    g.c_l = (int64_t)s.B * s.L * s.dk;
    g.status = sc.status;
    c = launch_gemm(g, st);
    if (c != cudaSuccess) return c;
    if (n_tail > 0) {
        for (int l = 0; l < s.W; ++l) {
            c = cudaMemcpy2DAsync(
                xbuf + ((size_t)l * s.B * s.L + L) * s.dk * e, (size_t)s.L * s.dk * e,
                (const char *)tail + (size_t)l * s.B * n_tail * s.dk * e,
                (size_t)n_tail * s.dk * e, (size_t)n_tail * s.dk * e, (size_t)s.B,
                cudaMemcpyDeviceToDevice, st);
            if (c != cudaSuccess) return c;
        }
    }
    return factorize_t<T>(s, xbuf, omega, n_iter, A_out, Bt_out, ws, st, false);
}

size_t refold_x_bytes(const Shape &s) {
    return align256((size_t)s.W * s.B * s.L * s.dk * (s.bf16 ? 2 : 4));
}

}  // namespace

size_t refold_ws_bytes(const xkv_dims &d, int W, int r, int64_t n_tail) {
    xkv_dims e = d;
    e.ctx_len = d.ctx_len + n_tail;
    const Shape s = shape_of(e, W, r);
    return refold_x_bytes(s) + carve(s, nullptr, nullptr);
}

cudaError_t launch_refold(const xkv_dims &d, int W, int r, const void *A, const void *Bt,
                          const void *tail, int64_t n_tail, const float *omega, int n_iter,
                          void *A_out, void *Bt_out, void *ws, cudaStream_t s) {
    xkv_dims e = d;
    e.ctx_len = d.ctx_len + n_tail;
    const Shape sh = shape_of(e, W, r);
    return sh.bf16 ? refold_t<__nv_bfloat16>(sh, n_tail, A, Bt, tail, omega, n_iter, A_out,
                                             Bt_out, ws, s)
                   : refold_t<float>(sh, n_tail, A, Bt, tail, omega, n_iter, A_out, Bt_out, ws,
                                     s);
}

size_t factorize_ws_bytes(const xkv_dims &d, int W, int r) {
    return carve(shape_of(d, W, r), nullptr, nullptr);
}

cudaError_t launch_factorize(const xkv_dims &d, int W, int r, const void *X, const float *omega,
                             int n_iter, void *A_out, void *Bt_out, void *ws, cudaStream_t s) {
    const Shape sh = shape_of(d, W, r);
    return sh.bf16 ? factorize_t<__nv_bfloat16>(sh, X, omega, n_iter, A_out, Bt_out, ws, s, true)
                   : factorize_t<float>(sh, X, omega, n_iter, A_out, Bt_out, ws, s, true);
}

}  // namespace xkv
