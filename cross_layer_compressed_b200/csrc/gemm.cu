// The dense products of the cross-layer factorization (xKV page, section 2.2: the
// rank-r SVD of a window's concatenated caches, computed here by randomized subspace
// iteration), on this library's own kernels.
//
// Four products, batched over the sequences of a window (X_l = layer l's cache
// [B][L][d_kv], F and Q fp32 bases, R^-1 the inverse Cholesky factor of a basis):
//   GM_XF      Y      = sum_l X_l F_l        (M = L,    N = r, K = d_kv per layer)
//   GM_XT      Z_l    = X_l^T Q              (M = d_kv, N = r, K = L)
//   GM_APPLY   Y'     = Y R^-1               (M = rows, N = r, K = r)
//   GM_REFOLD  X'_l   = A B_l                (M = L,    N = d_kv, K = r)
//   GM_VRANGE  V_hat  = A^V B^V_l, reduced in the epilogue to the value range of each
//              (chunk, KV head) -- the statistic of the value-range-aware selection
// For bf16 caches the fp32 bases are split into bf16 hi + lo parts (two K segments of the
// same product), so XF / XT keep ~16 significant bits at bf16 tensor-core rate; APPLY
// runs in TF32.  These go to k_gemm_tc: TMA tiles into a 4-stage ring, tcgen05.mma
// (M = 128, N = 256) into a double-buffered TMEM accumulator, a 4-warp epilogue.  fp32
// caches take k_gemm_simt, an fp32 CUDA-core kernel (every product in plain fp32).
//
// Operand layouts for the tensor cores: X is K-major in XF (token rows, d_kv contiguous)
// and MN-major in XT (the contraction runs over tokens); F and Q are MN-major (rank
// contiguous); APPLY reads R^-1 transposed (K-major), which the factorization writes;
// REFOLD reads A and B_l (column-major B) K-major.  Every mbarrier wait is bounded; a CTA
// that gives up sets XKV_ERR_TIMEOUT in the status word, drains its copies and MMAs,
// frees TMEM and returns.
#include "sm100_util.cuh"

namespace xkv {
namespace {

constexpr int GT_BM = 128, GT_BN = 256, GT_STAGES = 4;
constexpr int GT_A_BYTES = GT_BM * 128;         // 16 KB: 128 rows of 128 bytes of K
constexpr int GT_B_BYTES = GT_BN * 128;         // 32 KB
constexpr int GT_STAGE = GT_A_BYTES + GT_B_BYTES;
constexpr int GT_THREADS = 192;                 // warp 0 TMA, warp 1 MMA, warps 2-5 epilogue
constexpr uint32_t GT_SPIN = 1u << 24;

struct GtParams {
    int mode, tf32;
    int M, N, nb, nl;
    int n_seg, P, kb_seg;
    int dk;                  // XF: rows of F per layer
    int b_shared;            // XF: F has no batch dimension (the test matrix)
    int m_tiles, n_tiles;
    int64_t n_tiles_total;
    void *C;
    int c_bf16;
    int64_t ldc, c_b, c_l;
    unsigned *status;
    // value-range epilogue (GM_VRANGE): rho [B][Hkv][nC] fp32, the max over a chunk's rows
    // of max - min of a head's hd columns, folded in with atomicMax on the (>= 0) bits
    float *rho;
    int hd, chunk, Hkv;
    int64_t nC;
    uint32_t mma_spin;       // poll limit of the MMA issuer's waits for staged data
};

struct GtShared {
    uint64_t full[GT_STAGES], empty[GT_STAGES], accf[2], acce[2], idle;
    uint32_t tmem;
    int abort;
};

struct Tile {
    int l, b, m0, n0;
};
__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {   // a in the low half
    __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t *>(&h);
}
// Barrier 1 over the 128 epilogue threads that also ORs `flag` across them, so a decision
// taken after a bounded wait is the same in all four warps.
__device__ __forceinline__ bool epi_any(bool flag) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred pin, pout;\n\t"
        "setp.ne.u32 pin, %1, 0;\n\t"
        "bar.red.or.pred pout, 1, 128, pin;\n\t"
        "selp.u32 %0, 1, 0, pout;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)flag)
        : "memory");
    return r != 0;
}
__device__ __forceinline__ Tile gt_decode(const GtParams &p, int64_t t) {
    Tile x;
    const int nt = (int)(t % p.n_tiles);
    int64_t rest = t / p.n_tiles;
    const int mt = (int)(rest % p.m_tiles);
    rest /= p.m_tiles;
    x.b = (int)(rest % p.nb);
    x.l = (int)(rest / p.nb);
    x.m0 = mt * GT_BM;
    x.n0 = nt * GT_BN;
    return x;
}

__device__ __forceinline__ bool gt_wait(uint64_t *bar, uint32_t parity, GtShared *sh,
                                        const GtParams &p, uint32_t limit = GT_SPIN) {
    if (mbar_wait_bounded(bar, parity, &sh->abort, limit)) return true;
    if (!*(volatile int *)&sh->abort) {
        *(volatile int *)&sh->abort = 1;
        if (p.status) atomicOr(p.status, 1u << XKV_ERR_TIMEOUT);
    }
    return false;
}

__global__ void __launch_bounds__(GT_THREADS, 1)
    k_gemm_tc(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB0,
              const __grid_constant__ CUtensorMap tmB1, const GtParams p) {
    extern __shared__ unsigned char gt_raw[];
    unsigned char *smem = (unsigned char *)(((uintptr_t)gt_raw + 1023) & ~(uintptr_t)1023);
    GtShared *sh = reinterpret_cast<GtShared *>(smem + GT_STAGES * GT_STAGE);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < GT_STAGES; ++s) {
            mbar_init(&sh->full[s], 1);
            mbar_init(&sh->empty[s], 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&sh->accf[a], 1);
            mbar_init(&sh->acce[a], 1);
        }
        mbar_init(&sh->idle, 1);
        sh->abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        prefetch_tmap(&tmA);
        prefetch_tmap(&tmB0);
        prefetch_tmap(&tmB1);
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 512;" ::"r"(
                         su32(&sh->tmem))
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tcgen05_before();
    __syncthreads();
    tcgen05_after();
    const uint32_t tmem = sh->tmem;
    grid_dep_wait();
    const int kb_tile = p.n_seg * p.kb_seg;     // K blocks of one output tile
    const bool a_mn = p.mode == GM_XT;
    const bool b_mn = p.mode == GM_XF || p.mode == GM_XT;

    if (warp == 0) {
        // ---------------------------------------------------------------- TMA producer
        if (lane == 0) {
            int64_t it = 0;
            bool ok = true;
            for (int64_t t = blockIdx.x; t < p.n_tiles_total && ok; t += gridDim.x) {
                const Tile x = gt_decode(p, t);
                int nbq = 4;                     // MN-major B boxes inside N (the rest is masked)
                if (b_mn) nbq = min(4, (p.N - x.n0 + 63) / 64);
                const uint32_t bytes = GT_A_BYTES + (b_mn ? nbq * 8192 : GT_B_BYTES);
                for (int kb = 0; kb < kb_tile; ++kb, ++it) {
                    const int s = (int)(it % GT_STAGES);
                    const uint32_t n = (uint32_t)(it / GT_STAGES);
                    if (!gt_wait(&sh->empty[s], (n & 1) ^ 1, sh, p)) { ok = false; break; }
                    const int seg = kb / p.kb_seg, k = kb % p.kb_seg;
                    unsigned char *sa = smem + s * GT_STAGE, *sb = sa + GT_A_BYTES;
                    mbar_expect_tx(&sh->full[s], bytes);
                    switch (p.mode) {
                        case GM_XF: {
                            const int layer = seg / p.P;
                            const CUtensorMap *mb = (seg % p.P) ? &tmB1 : &tmB0;
                            tma_load_4d(&tmA, &sh->full[s], sa, k * 64, x.m0, x.b, layer);
                            for (int q = 0; q < nbq; ++q)
                                tma_load_3d(mb, &sh->full[s], sb + q * 8192, x.n0 + 64 * q,
                                            layer * p.dk + k * 64, p.b_shared ? 0 : x.b);
                            break;
                        }
                        case GM_XT: {
                            const CUtensorMap *mb = seg ? &tmB1 : &tmB0;
                            tma_load_4d(&tmA, &sh->full[s], sa, x.m0, k * 64, x.b, x.l);
                            tma_load_4d(&tmA, &sh->full[s], sa + 8192, x.m0 + 64, k * 64, x.b, x.l);
                            for (int q = 0; q < nbq; ++q)
                                tma_load_3d(mb, &sh->full[s], sb + q * 8192, x.n0 + 64 * q, k * 64,
                                            x.b);
                            break;
                        }
                        case GM_APPLY:
                            tma_load_3d(&tmA, &sh->full[s], sa, k * 32, x.m0, x.b);
                            tma_load_3d(&tmB0, &sh->full[s], sb, k * 32, x.n0, x.b);
                            break;
                        default:   // GM_REFOLD, GM_VRANGE
                            tma_load_3d(&tmA, &sh->full[s], sa, k * 64, x.m0, x.b);
                            tma_load_4d(&tmB0, &sh->full[s], sb, k * 64, x.n0, x.b, x.l);
                            break;
                    }
                }
            }
            if (!ok) {
                // every stage issued so far lands before the CTA may leave
                for (int64_t j = it - GT_STAGES > 0 ? it - GT_STAGES : 0; j < it; ++j)
                    for (uint32_t i = 0; i < GT_SPIN; ++i)
                        if (mbar_test(&sh->full[j % GT_STAGES], (uint32_t)(j / GT_STAGES) & 1))
                            break;
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ---------------------------------------------------------------- MMA issuer
        if (lane == 0) {
            const uint32_t base = su32(smem);
            const uint32_t idesc = p.tf32 ? idesc_tf32(GT_BM, GT_BN, a_mn, b_mn)
                                          : idesc_f16(GT_BM, GT_BN, a_mn, b_mn);
            int64_t it = 0;
            int i = 0;
            bool ok = true;
            for (int64_t t = blockIdx.x; t < p.n_tiles_total && ok; t += gridDim.x, ++i) {
                const int acc = i & 1;
                if (!gt_wait(&sh->acce[acc], ((i >> 1) & 1) ^ 1, sh, p)) { ok = false; break; }
                tcgen05_after();
                const uint32_t d = tmem + acc * GT_BN;
                for (int kb = 0; kb < kb_tile; ++kb, ++it) {
                    const int s = (int)(it % GT_STAGES);
                    const uint32_t n = (uint32_t)(it / GT_STAGES);
                    if (!gt_wait(&sh->full[s], n & 1, sh, p, p.mma_spin)) { ok = false; break; }
                    tcgen05_after();
                    const uint32_t sa = base + s * GT_STAGE, sb = sa + GT_A_BYTES;
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk) {   // 32 bytes of K per instruction
                        const uint64_t da = a_mn ? smem_desc_sw128(sa + kk * 2048, 8192, 1024)
                                                 : smem_desc_sw128(sa + kk * 32, 16, 1024);
                        const uint64_t db = b_mn ? smem_desc_sw128(sb + kk * 2048, 8192, 1024)
                                                 : smem_desc_sw128(sb + kk * 32, 16, 1024);
                        const uint32_t accum = (kb | kk) ? 1u : 0u;
                        if (p.tf32) umma_tf32(d, da, db, idesc, accum);
                        else umma_f16(d, da, db, idesc, accum);
                    }
                    umma_arrive(&sh->empty[s]);
                }
                if (!ok) break;
                umma_arrive(&sh->accf[acc]);
            }
            umma_arrive(&sh->idle);          // fires once every MMA issued here completed
            for (uint32_t j = 0; j < GT_SPIN; ++j)
                if (mbar_test(&sh->idle, 0)) break;
        }
        __syncwarp();
    } else {
        // ---------------------------------------------------------------- epilogue
        const int quad = warp & 3;                     // TMEM lanes 32 quad .. 32 quad + 31
        const int row = quad * 32 + lane;
        const uint32_t lane_base = (uint32_t)(quad * 32) << 16;
        int i = 0;
        for (int64_t t = blockIdx.x; t < p.n_tiles_total; t += gridDim.x, ++i) {
            const int acc = i & 1;
            bool ok = true;
            if (lane == 0) ok = gt_wait(&sh->accf[acc], (i >> 1) & 1, sh, p);
            if (epi_any(!ok)) break;             // the same decision in all four warps
            tcgen05_after();
            const Tile x = gt_decode(p, t);
            const int64_t m = (int64_t)x.m0 + row;
            const bool mrow = m < p.M;
            if (p.mode == GM_VRANGE) {
                // per head slice of the tile: this row's max - min, then the max over the
                // rows of its chunk (lanes of one warp when the chunk divides 32)
                for (int h0 = 0; h0 < GT_BN && x.n0 + h0 < p.N; h0 += p.hd) {
                    float lo = INFINITY, hi = -INFINITY;
                    for (int c0 = h0; c0 < h0 + p.hd; c0 += 32) {
                        float v[32];
                        tmem_load32(tmem + lane_base + acc * GT_BN + c0, v);
#pragma unroll
                        for (int j = 0; j < 32; ++j) {
                            lo = fminf(lo, v[j]);
                            hi = fmaxf(hi, v[j]);
                        }
                    }
                    float rg = mrow ? hi - lo : 0.f;
                    const int seg = 32 % p.chunk == 0 ? p.chunk : 1;
                    for (int off = 1; off < seg; off <<= 1)
                        rg = fmaxf(rg, __shfl_xor_sync(0xffffffffu, rg, off));
                    if (mrow && lane % seg == 0) {
                        const int g = (x.n0 + h0) / p.hd;
                        atomicMax(reinterpret_cast<unsigned *>(
                                      p.rho + ((int64_t)x.b * p.Hkv + g) * p.nC + m / p.chunk),
                                  __float_as_uint(rg));
                    }
                }
                tcgen05_before();
                asm volatile("bar.sync 1, 128;" ::: "memory");
                if (warp == 2 && lane == 0) mbar_arrive(&sh->acce[acc]);
                continue;
            }
            const int64_t off = (int64_t)x.l * p.c_l + (int64_t)x.b * p.c_b + m * p.ldc;
            for (int c0 = 0; c0 < GT_BN && x.n0 + c0 < p.N; c0 += 32) {
                float v[32];
                tmem_load32(tmem + lane_base + acc * GT_BN + c0, v);
                const int nvalid = min(32, p.N - (x.n0 + c0));   // a multiple of 16
                if (!mrow) continue;
                if (p.c_bf16) {
                    __nv_bfloat16 *dst = (__nv_bfloat16 *)p.C + off + x.n0 + c0;
                    for (int j = 0; j < nvalid; j += 8) {
                        uint4 w;
                        w.x = pack_bf16(v[j], v[j + 1]);
                        w.y = pack_bf16(v[j + 2], v[j + 3]);
                        w.z = pack_bf16(v[j + 4], v[j + 5]);
                        w.w = pack_bf16(v[j + 6], v[j + 7]);
                        *reinterpret_cast<uint4 *>(dst + j) = w;
                    }
                } else {
                    float *dst = (float *)p.C + off + x.n0 + c0;
                    for (int j = 0; j < nvalid; j += 4)
                        *reinterpret_cast<float4 *>(dst + j) =
                            make_float4(v[j], v[j + 1], v[j + 2], v[j + 3]);
                }
            }
            tcgen05_before();
            asm volatile("bar.sync 1, 128;" ::: "memory");
            if (warp == 2 && lane == 0) mbar_arrive(&sh->acce[acc]);
        }
    }
    tcgen05_before();
    __syncthreads();
    tcgen05_after();
    if (warp == 1)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 512;" ::"r"(tmem)
                     : "memory");
}

// ---------------------------------------------------------------- fp32 CUDA cores
// C = sum over segments of A_s B_s in plain fp32 (64 x 64 tiles, 16-deep K slices staged
// in shared memory, 4 x 4 outputs per thread).  Operand element addresses follow the
// same four products as k_gemm_tc, from plain pointers.
struct GsParams {
    int mode;
    int M, N, nb, nl, n_seg, P;
    int64_t K_seg;
    const float *A, *B0, *B1;
    int b_shared;
    int64_t L, dk, r, n_rows;   // n_rows: rows of F / Z (W d_kv); L: rows of X / Q / Y
    int64_t a_l, a_b;           // XF / XT: X strides of a layer and a sequence
    float *C;
    int64_t ldc, c_b, c_l;
};

__device__ __forceinline__ float gs_a(const GsParams &p, int seg, int l, int b, int64_t m,
                                      int64_t k) {
    switch (p.mode) {
        case GM_XF: return p.A[(seg / p.P) * p.a_l + b * p.a_b + m * p.dk + k];
        case GM_XT: return p.A[l * p.a_l + b * p.a_b + k * p.dk + m];
        case GM_APPLY: return p.A[(int64_t)b * p.L * p.r + m * p.r + k];
        default: return p.A[(int64_t)b * p.L * p.r + m * p.r + k];
    }
}
__device__ __forceinline__ float gs_b(const GsParams &p, int seg, int l, int b, int64_t k,
                                      int64_t n) {
    switch (p.mode) {
        case GM_XF: {
            const float *B = (seg % p.P) ? p.B1 : p.B0;
            const int64_t bb = p.b_shared ? 0 : b;
            return B[bb * p.n_rows * p.r + ((seg / p.P) * p.dk + k) * p.r + n];
        }
        case GM_XT: return ((seg % p.P) ? p.B1 : p.B0)[(int64_t)b * p.L * p.r + k * p.r + n];
        case GM_APPLY: return p.B0[(int64_t)b * p.r * p.r + n * p.r + k];   // (R^-1)^T
        default: return p.B0[((int64_t)l * p.nb + b) * p.dk * p.r + n * p.r + k];
    }
}

__global__ void __launch_bounds__(256) k_gemm_simt(const GsParams p) {
    __shared__ float As[16][64 + 4], Bs[16][64 + 4];
    const int l = blockIdx.z / p.nb, b = blockIdx.z % p.nb;
    const int64_t m0 = (int64_t)blockIdx.y * 64, n0 = (int64_t)blockIdx.x * 64;
    const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
    float acc[4][4] = {};
    for (int seg = 0; seg < p.n_seg; ++seg) {
        for (int64_t k0 = 0; k0 < p.K_seg; k0 += 16) {
            for (int e = threadIdx.x; e < 16 * 64; e += 256) {
                const int kk = e / 64, mm = e % 64;
                const int64_t m = m0 + mm, n = n0 + mm, k = k0 + kk;
                As[kk][mm] = (m < p.M && k < p.K_seg) ? gs_a(p, seg, l, b, m, k) : 0.f;
                Bs[kk][mm] = (n < p.N && k < p.K_seg) ? gs_b(p, seg, l, b, k, n) : 0.f;
            }
            __syncthreads();
#pragma unroll
            for (int kk = 0; kk < 16; ++kk) {
                float a[4], c[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    a[i] = As[kk][ty * 4 + i];
                    c[i] = Bs[kk][tx * 4 + i];
                }
#pragma unroll
                for (int i = 0; i < 4; ++i)
#pragma unroll
                    for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], c[j], acc[i][j]);
            }
            __syncthreads();
        }
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int64_t m = m0 + ty * 4 + i;
        if (m >= p.M) continue;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int64_t n = n0 + tx * 4 + j;
            if (n < p.N) p.C[l * p.c_l + b * p.c_b + m * p.ldc + n] = acc[i][j];
        }
    }
}

// Value ranges in plain fp32 (fp32 caches): one CTA per (chunk, KV head, sequence), a
// thread per head column; each row of the chunk is rebuilt, reduced to max - min.
__global__ void __launch_bounds__(128) k_vrange_simt(const float *__restrict__ Av,
                                                     const float *__restrict__ Bvt,
                                                     float *__restrict__ rho, int64_t L, int C,
                                                     int rv, int hd, int Hkv) {
    __shared__ float red[2][4];
    const int64_t c = blockIdx.x;
    const int g = blockIdx.y, b = blockIdx.z, j = threadIdx.x;
    const int d_kv = Hkv * hd;
    const float *bt = Bvt + ((int64_t)b * d_kv + (int64_t)g * hd + j) * rv;
    float best = 0.f;
    for (int t = 0; t < C; ++t) {
        const float *a = Av + ((int64_t)b * L + c * C + t) * rv;
        float v = 0.f;
        for (int i = 0; i < rv; ++i) v = fmaf(a[i], bt[i], v);
        float lo = v, hi = v;
        for (int off = 16; off; off >>= 1) {
            lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, off));
            hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, off));
        }
        if ((j & 31) == 0) {
            red[0][j >> 5] = lo;
            red[1][j >> 5] = hi;
        }
        __syncthreads();
        if (j == 0) {
            for (int w = 1; w < hd / 32; ++w) {
                lo = fminf(lo, red[0][w]);
                hi = fmaxf(hi, red[1][w]);
            }
            best = fmaxf(best, hi - lo);
        }
        __syncthreads();
    }
    if (j == 0) rho[((int64_t)b * Hkv + g) * (L / C) + c] = best;
}

}  // namespace

cudaError_t launch_gemm(const GemmDesc &g, cudaStream_t s) {
    if (g.mode == GM_VRANGE && !g.tc) {
        k_vrange_simt<<<dim3((unsigned)g.nC, g.Hkv, g.nb), g.hd, 0, s>>>(
            (const float *)g.A, (const float *)g.B0, g.rho, g.L, g.chunk, (int)g.r, g.hd, g.Hkv);
        return cudaGetLastError();
    }
    if (!g.tc) {
        GsParams p{};
        p.mode = g.mode;
        p.M = g.M;
        p.N = g.N;
        p.nb = g.nb;
        p.nl = g.nl;
        p.n_seg = g.n_seg;
        p.P = g.P;
        p.K_seg = g.K_seg;
        p.A = (const float *)g.A;
        p.B0 = (const float *)g.B0;
        p.B1 = (const float *)g.B1;
        p.b_shared = g.b_shared;
        p.L = g.L;
        p.dk = g.dk;
        p.r = g.r;
        p.n_rows = g.n_rows;
        p.a_l = (int64_t)g.nb * g.L * g.dk;
        p.a_b = g.L * g.dk;
        p.C = (float *)g.C;
        p.ldc = g.ldc;
        p.c_b = g.c_b;
        p.c_l = g.c_l;
        const dim3 grid((unsigned)((g.N + 63) / 64), (unsigned)((g.M + 63) / 64),
                        (unsigned)(g.nb * g.nl));
        k_gemm_simt<<<grid, 256, 0, s>>>(p);
        return cudaGetLastError();
    }
    CUtensorMap tA, tB0, tB1;
    const uint64_t B = (uint64_t)g.nb, W = (uint64_t)g.W;
    const uint64_t L = (uint64_t)g.L, dk = (uint64_t)g.dk, r = (uint64_t)g.r;
    bool ok = true;
    switch (g.mode) {
        case GM_XF: {
            const uint64_t da[4] = {dk, L, B, W}, sa[3] = {dk * 2, L * dk * 2, B * L * dk * 2};
            const uint32_t ba[4] = {64, 128, 1, 1};
            ok = make_map_sw128(&tA, g.A, false, 4, da, sa, ba);
            const uint64_t bb = g.b_shared ? 1 : B, nr = (uint64_t)g.n_rows;
            const uint64_t db[3] = {r, nr, bb}, sb[2] = {r * 2, nr * r * 2};
            const uint32_t bx[3] = {64, 64, 1};
            ok = ok && make_map_sw128(&tB0, g.B0, false, 3, db, sb, bx) &&
                 make_map_sw128(&tB1, g.B1 ? g.B1 : g.B0, false, 3, db, sb, bx);
            break;
        }
        case GM_XT: {
            const uint64_t da[4] = {dk, L, B, W}, sa[3] = {dk * 2, L * dk * 2, B * L * dk * 2};
            const uint32_t ba[4] = {64, 64, 1, 1};
            ok = make_map_sw128(&tA, g.A, false, 4, da, sa, ba);
            const uint64_t db[3] = {r, L, B}, sb[2] = {r * 2, L * r * 2};
            const uint32_t bx[3] = {64, 64, 1};
            ok = ok && make_map_sw128(&tB0, g.B0, false, 3, db, sb, bx) &&
                 make_map_sw128(&tB1, g.B1 ? g.B1 : g.B0, false, 3, db, sb, bx);
            break;
        }
        case GM_APPLY: {   // tf32: A [B][rows][r], B0 = (R^-1)^T [B][r][r], both K-major
            const uint64_t rows = (uint64_t)g.M;
            const uint64_t da[3] = {r, rows, B}, sa[2] = {r * 4, rows * r * 4};
            const uint32_t ba[3] = {32, 128, 1};
            const uint64_t db[3] = {r, r, B}, sb[2] = {r * 4, r * r * 4};
            const uint32_t bx[3] = {32, 256, 1};
            ok = make_map_sw128(&tA, g.A, true, 3, da, sa, ba) &&
                 make_map_sw128(&tB0, g.B0, true, 3, db, sb, bx);
            tB1 = tB0;
            break;
        }
        default: {         // GM_REFOLD: A [B][L][r], B0 = Bt [W][B][d_kv][r] (GM_VRANGE: W = 1)
            const uint64_t da[3] = {r, L, B}, sa[2] = {r * 2, L * r * 2};
            const uint32_t ba[3] = {64, 128, 1};
            const uint64_t db[4] = {r, dk, B, W}, sb[3] = {r * 2, dk * r * 2, B * dk * r * 2};
            const uint32_t bx[4] = {64, 256, 1, 1};
            ok = make_map_sw128(&tA, g.A, false, 3, da, sa, ba) &&
                 make_map_sw128(&tB0, g.B0, false, 4, db, sb, bx);
            tB1 = tB0;
            break;
        }
    }
    if (!ok) return cudaErrorInvalidValue;
    GtParams p{};
    p.mode = g.mode;
    p.tf32 = g.mode == GM_APPLY;
    p.M = g.M;
    p.N = g.N;
    p.nb = g.nb;
    p.nl = g.nl;
    p.n_seg = g.n_seg;
    p.P = g.P;
    p.kb_seg = (int)((g.K_seg * (p.tf32 ? 4 : 2) + 127) / 128);
    p.dk = (int)g.dk;
    p.b_shared = g.b_shared;
    p.m_tiles = (g.M + GT_BM - 1) / GT_BM;
    p.n_tiles = (g.N + GT_BN - 1) / GT_BN;
    p.n_tiles_total = (int64_t)p.m_tiles * p.n_tiles * g.nb * g.nl;
    p.C = g.C;
    p.c_bf16 = g.c_bf16;
    p.ldc = g.ldc;
    p.c_b = g.c_b;
    p.c_l = g.c_l;
    p.status = g.status;
    p.rho = g.rho;
    p.hd = g.hd;
    p.chunk = g.chunk;
    p.Hkv = g.Hkv;
    p.nC = g.nC;
    // XKV_TEST_MMA_SPIN (tests only, read on every call): the poll limit of the MMA
    // issuer's waits on staged data, so a test can make them give up; every other wait,
    // and the drain that follows, keeps its full bound
    p.mma_spin = test_poll_limit("XKV_TEST_MMA_SPIN", GT_SPIN);
    const size_t smem = 1024 + (size_t)GT_STAGES * GT_STAGE + sizeof(GtShared);
    cudaError_t e = set_smem_limit((const void *)k_gemm_tc, smem);
    if (e != cudaSuccess) return e;
    const int64_t grid = p.n_tiles_total < sm_count() ? p.n_tiles_total : sm_count();
    k_gemm_tc<<<(unsigned)grid, GT_THREADS, smem, s>>>(tA, tB0, tB1, p);
    return cudaGetLastError();
}

}  // namespace xkv
