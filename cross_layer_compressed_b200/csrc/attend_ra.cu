// Reassociated xKV attention: the same result as reconstruct-then-attend, computed in
// the rank space of the window's basis.
//
// xKV page, section 2.2 (K_hat = A^K B^K_l, V_hat = A^V B^V_l) and section 2.3 (attend
// over the rows T of the selected chunks).  By associativity,
//   z_h[t] = q_h . (A^K[t] B^K_g) / sqrt(hd) = A^K[t] . q~_h / sqrt(hd),  q~_h = B^K_g q_h
//   o_h    = sum_t p_h[t] (A^V[t] B^V_g)    = (sum_t p_h[t] A^V[t]) B^V_g = u_h B^V_g,
// so a decode step reads the selected rows of A once, does r-deep dot products instead of
// r x hd GEMMs, and touches B_l only twice per (sequence, KV head): once for q~ and once
// in the final projection.  Four kernels:
//   k_qtilde     q~_h = B^K_g q_h (fp32), stored as two bf16 terms (hi + lo, ~16 bits)
//   k_xkv_ra     per work item (b, g, <= 256 selected rows), on tcgen05:
//                  logits  D_z[t][n] = A^K[t][:] . Q~[n][:]    (M = 128 rows, N = 8)
//                  output  D_u[r][n] = sum_t A^V[t][r] P[n][t] (M = 128 columns of A^V,
//                          read MN-major straight from the staged rows; N = 8)
//                with P holding each probability as two bf16 terms, as in the R-CLA kernel;
//                partials (m, l, u) in rank space
//   k_merge_ra   merges an item's splits in rank space (U_h, L_h)
//   k_project_ra o_h = U_h B^V_g / L_h
// or, for calls with many splits, k_merge_project_ra, which does both, one slice of r_V
// per CTA.
// Warp roles of k_xkv_ra: warp 0 TMEM + MMA issue, warps 1-4 TMA producers, warps 5-8
// epilogue.  A stage holds 128 columns of the item's rows; each 8-row group arrives in
// one copy of a 3D view of A (64 elements x 8 rows x 2 column blocks) as two consecutive
// 128-byte-swizzled atoms, so a stage takes one copy per group instead of two (the
// kernel is bound by the copy engine's per-copy cost: it does almost no arithmetic).
// The operand descriptors follow the [group][column block][8 rows x 128 B] layout:
// 8-row groups 2 KB apart, the two column blocks 1 KB apart.  Every mbarrier wait is bounded; on
// expiry the CTA sets XKV_ERR_TIMEOUT in the workspace status word, drains its copies
// and MMAs (bounded), frees TMEM and returns, and the combine writes NaN outputs.
#include "sm100_util.cuh"

namespace xkv {
namespace {

constexpr int RA_ROWS = 256;                    // rows per work item
constexpr int RA_GROUP = 2048;                  // one 8-row group: two 64-column atoms
constexpr int RA_STAGE = RA_ROWS / 8 * RA_GROUP;  // 128 columns of the item's rows: 64 KB
constexpr int RA_STAGES = 3;
constexpr int RA_QBUF = 16 * 1024;              // Q~: NO rows x r_K, K-major
constexpr int RA_PBUF = 8 * 1024;               // P: NO rows x 256 tokens, K-major
constexpr uint32_t TM_Z = 0;                    // logits: 2 token halves x NO columns
constexpr uint32_t TM_U = 64;                   // output: r_V / 128 blocks x NO columns
// Q~ and P rows: the hi terms of the G heads, then the lo terms, padded to the MMA's N
template <int G> struct RaCfg {
    static constexpr int NO = (2 * G + 7) / 8 * 8;
    static constexpr int ATOM = NO / 8 * 1024;          // bytes per 64-wide K atom
    static constexpr int MAXR = RA_QBUF / ATOM * 64;    // r_K the Q~ buffer holds
};
constexpr int W_MMA = 0, W_LOAD = 1, N_LOAD = 4, W_EPI = 5, N_EPI = 4;
constexpr int RA_THREADS = 32 * (W_EPI + N_EPI);  // 288
constexpr int EPI_THREADS = 32 * N_EPI;           // 128
constexpr uint32_t RA_SPIN = 1u << 24;

struct RaShared {
    uint64_t full[RA_STAGES], empty[RA_STAGES];
    uint64_t q_full, z_full, p_full, o_full, idle;
    uint32_t tmem_base;
    int abort;
    float red[N_EPI][8];
};

struct RaParams {
    const __nv_bfloat16 *qt_hi, *qt_lo;   // [B][Hq][r_K]
    const int32_t *sel;                   // [B][Hkv][n_sel] or null (dense)
    float *partials;                      // [n_split][B][Hq][r_V + 2]
    unsigned *status;
    int64_t L;
    int n_sel, C, rk, rv, Hq, Hkv, B;
    int chunks_per_item, n_split, n_items;
    float qscale;                         // log2(e) / sqrt(hd)
    uint32_t mma_spin;                    // poll limit of the MMA issuer's waits for staged data
};

struct RaItem {
    int b, g, split, c0, nch, nr;
};
// split-major, as in the explicit kernel: the heads that read the same rows run together
__device__ __forceinline__ RaItem ra_decode(const RaParams &p, int item) {
    RaItem it;
    const int units = p.B * p.Hkv;
    const int u = item % units;
    it.split = item / units;
    it.b = u / p.Hkv;
    it.g = u % p.Hkv;
    it.c0 = it.split * p.chunks_per_item;
    it.nch = min(p.chunks_per_item, p.n_sel - it.c0);
    it.nr = it.nch * p.C;
    return it;
}

// byte offset of element (n, k) of a K-major 128-byte-swizzled operand: 64-wide K atoms
// `atom` bytes apart, 8-row groups 1 KB apart inside an atom
__device__ __forceinline__ uint32_t kmaj_off(int n, int k, int atom) {
    const int kin = k & 63;
    return (uint32_t)((k >> 6) * atom + (n >> 3) * 1024 + (n & 7) * 128 +
                      ((((kin >> 3) ^ (n & 7)) & 7) << 4) + (kin & 7) * 2);
}
__device__ __forceinline__ void ra_epi_bar() {
    asm volatile("bar.sync 1, %0;" ::"n"(EPI_THREADS) : "memory");
}
__device__ __forceinline__ bool ra_epi_bar_any(bool flag) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred pin, pout;\n\t"
        "setp.ne.u32 pin, %1, 0;\n\t"
        "bar.red.or.pred pout, 1, %2, pin;\n\t"
        "selp.u32 %0, 1, 0, pout;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)flag), "n"(EPI_THREADS)
        : "memory");
    return r != 0;
}
__device__ __forceinline__ bool ra_wait(uint64_t *b, uint32_t parity, RaShared *sh,
                                        const RaParams &p, uint32_t limit = RA_SPIN) {
    if (mbar_wait_bounded(b, parity, &sh->abort, limit)) return true;
    if (!*(volatile int *)&sh->abort) {
        *(volatile int *)&sh->abort = 1;
        grid_dep_wait();    // after q~'s clear of the status word
        if (p.status) atomicOr(p.status, 1u << XKV_ERR_TIMEOUT);
    }
    return false;
}
__device__ __forceinline__ bool ra_warp_wait(uint64_t *b, uint32_t parity, RaShared *sh,
                                             const RaParams &p, int lane) {
    int got = 0;
    if (lane == 0) got = ra_wait(b, parity, sh, p) ? 1 : 0;
    return __shfl_sync(0xffffffffu, got, 0) != 0;
}

template <int G>
__global__ void __launch_bounds__(RA_THREADS, 1)
    k_xkv_ra(const __grid_constant__ CUtensorMap tmAk, const __grid_constant__ CUtensorMap tmAv,
             const RaParams p) {
    using Cfg = RaCfg<G>;
    constexpr int NO = Cfg::NO, ATOM = Cfg::ATOM;
    static_assert(Cfg::MAXR >= 512, "the Q~ buffer holds a rank-512 query at least");
    extern __shared__ unsigned char smem_raw[];
    unsigned char *smem = (unsigned char *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    unsigned char *qbuf = smem + RA_STAGES * RA_STAGE;
    unsigned char *pbuf = qbuf + RA_QBUF;
    RaShared *sh = reinterpret_cast<RaShared *>(pbuf + RA_PBUF);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t nC = p.L / p.C;
    const int gpc = p.C / 8;

    if (threadIdx.x == 0) {
        for (int s = 0; s < RA_STAGES; ++s) {
            mbar_init(&sh->full[s], 1);
            mbar_init(&sh->empty[s], 1);
        }
        mbar_init(&sh->q_full, 1);
        mbar_init(&sh->z_full, 1);
        mbar_init(&sh->p_full, 1);
        mbar_init(&sh->o_full, 1);
        mbar_init(&sh->idle, 1);
        sh->abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        prefetch_tmap(&tmAk);
        prefetch_tmap(&tmAv);
    }
    if (warp == W_MMA) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 256;" ::"r"(
                         su32(&sh->tmem_base))
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tcgen05_before();
    __syncthreads();
    tcgen05_after();
    const uint32_t tmem = sh->tmem_base;

    if (warp >= W_LOAD && warp < W_LOAD + N_LOAD) {
        // ------------------------------------------------------------ TMA producers
        const int pi = warp - W_LOAD;
        const int gi = pi + N_LOAD * lane;         // this lane's 8-row group of an item
        int it = 0;
        bool ok = true;
        for (int item = blockIdx.x; item < p.n_items && ok; item += gridDim.x) {
            const RaItem w = ra_decode(p, item);
            const int ng = w.nr / 8;
            // an odd group count is padded to a whole 16-row MMA step with a copy of group
            // 0: finite rows whose weight is zero
            const int ngl = (ng + 1) & ~1;
            int row = 0;
            if (gi < ngl) {
                const int gg = gi < ng ? gi : 0;
                const int ci = gg / gpc, sub = gg % gpc;
                int64_t c = w.c0 + ci;
                if (p.sel) c = p.sel[((int64_t)w.b * p.Hkv + w.g) * p.n_sel + c];
                if (gi < ng && (c < 0 || c >= nC) && p.status) {  // the call fails: NaN outputs
                    grid_dep_wait();    // after q~'s clear of the status word
                    atomicOr(p.status, 1u << XKV_ERR_INVALID_ARG);
                }
                c = min64(max64(c, 0), nC - 1);                   // the copy stays in bounds
                row = (int)((int64_t)w.b * p.L + c * p.C + sub * 8);
            }
            for (int phase = 0; phase < 2 && ok; ++phase) {
                const int nst = (phase == 0 ? p.rk : p.rv) / 128;
                const CUtensorMap *m = phase == 0 ? &tmAk : &tmAv;
                for (int st = 0; st < nst; ++st, ++it) {
                    const int s = it % RA_STAGES, n = it / RA_STAGES;
                    if (!ra_warp_wait(&sh->empty[s], (n & 1) ^ 1, sh, p, lane)) {
                        ok = false;
                        break;
                    }
                    unsigned char *dst = smem + s * RA_STAGE;
                    if (pi == 0 && lane == 0)
                        mbar_expect_tx(&sh->full[s], (uint32_t)(ngl * 2 * 1024));
                    __syncwarp();
                    if (gi < ngl)   // both 64-column blocks of the group's 8 rows in one copy
                        tma_load_3d(m, &sh->full[s], dst + gi * RA_GROUP, 0, row, st * 2);
                    __syncwarp();
                }
            }
        }
        if (!ok && pi == 0 && lane == 0) {
            // Every stage the four warps issued lands before the CTA may leave: the last
            // RA_STAGES fills (each issued whole: a warp checks for abort only in its wait
            // on `empty`, which completes for all four warps alike) complete their phase.
            for (int j = it - RA_STAGES > 0 ? it - RA_STAGES : 0; j < it; ++j)
                for (uint32_t i = 0; i < RA_SPIN; ++i)
                    if (mbar_test(&sh->full[j % RA_STAGES], (uint32_t)(j / RA_STAGES) & 1)) break;
        }
    } else if (warp == W_MMA) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint32_t sbase = su32(smem), qb = su32(qbuf), pb = su32(pbuf);
            constexpr uint32_t idZ = idesc_f16(128, NO, false, false);
            constexpr uint32_t idU = idesc_f16(128, NO, true, false);  // A = A^V^T, MN-major
            int it = 0, ic = 0;
            bool ok = true;
            for (int item = blockIdx.x; item < p.n_items && ok; item += gridDim.x, ++ic) {
                const RaItem w = ra_decode(p, item);
                const int nk16 = ((w.nr / 8 + 1) & ~1) / 2;   // 16-row K steps of the output
                if (!ra_wait(&sh->q_full, ic & 1, sh, p)) { ok = false; break; }
                tcgen05_after();
                const int nsk = p.rk / 128;
                for (int st = 0; st < nsk && ok; ++st, ++it) {
                    const int s = it % RA_STAGES, n = it / RA_STAGES;
                    if (!ra_wait(&sh->full[s], n & 1, sh, p, p.mma_spin)) { ok = false; break; }
                    tcgen05_after();
                    const uint32_t a0 = sbase + s * RA_STAGE;
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk) {      // 16 columns of the stage per step
                        const uint32_t aoff = (kk >> 2) * 1024 + (kk & 3) * 32;
                        const int k0 = st * 128 + kk * 16;
                        const uint64_t bq = smem_desc_sw128(qb + (k0 >> 6) * ATOM + ((k0 & 63) >> 4) * 32,
                                                            16, 1024);
                        const uint32_t acc = (st | kk) ? 1u : 0u;
                        umma_f16(tmem + TM_Z, smem_desc_sw128(a0 + aoff, 16, RA_GROUP), bq, idZ,
                                 acc);
                        if (w.nr > 128)
                            umma_f16(tmem + TM_Z + NO,
                                     smem_desc_sw128(a0 + aoff + 16 * RA_GROUP, 16, RA_GROUP), bq,
                                     idZ, acc);
                    }
                    umma_arrive(&sh->empty[s]);
                }
                if (!ok) break;
                umma_arrive(&sh->z_full);
                if (!ra_wait(&sh->p_full, ic & 1, sh, p)) { ok = false; break; }
                tcgen05_after();
                const int nsv = p.rv / 128;
                for (int st = 0; st < nsv && ok; ++st, ++it) {
                    const int s = it % RA_STAGES, n = it / RA_STAGES;
                    if (!ra_wait(&sh->full[s], n & 1, sh, p, p.mma_spin)) { ok = false; break; }
                    tcgen05_after();
                    const uint32_t a0 = sbase + s * RA_STAGE;
                    for (int kt = 0; kt < nk16; ++kt) {
                        const int k0 = kt * 16;
                        umma_f16(tmem + TM_U + st * NO,
                                 smem_desc_sw128(a0 + kt * 2 * RA_GROUP, 1024, RA_GROUP),
                                 smem_desc_sw128(pb + (k0 >> 6) * ATOM + ((k0 & 63) >> 4) * 32, 16, 1024),
                                 idU, kt ? 1u : 0u);
                    }
                    umma_arrive(&sh->empty[s]);
                }
                if (!ok) break;
                umma_arrive(&sh->o_full);
            }
            umma_arrive(&sh->idle);
            for (uint32_t i = 0; i < RA_SPIN; ++i)
                if (mbar_test(&sh->idle, 0)) break;
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ epilogue
        const int et = threadIdx.x - 32 * W_EPI;   // 0..127
        const int ew = warp - W_EPI;
        const int quad = warp & 3;
        const int lrow = quad * 32 + lane;          // TMEM lane: token of a half / column
        const uint32_t lane_base = (uint32_t)(quad * 32) << 16;
        for (int i = et; i < (RA_QBUF + RA_PBUF) / 16; i += EPI_THREADS)   // pad rows = 0
            reinterpret_cast<uint4 *>(qbuf)[i] = make_uint4(0u, 0u, 0u, 0u);
        ra_epi_bar();
        auto write_q = [&](int item) {             // Q~ rows: hi of the G heads, then lo
            const RaItem w = ra_decode(p, item);
            const size_t base = ((size_t)w.b * p.Hq + (size_t)w.g * G) * p.rk;
            const int per = p.rk / 8;               // 16-byte pieces per row
            for (int e = et; e < 2 * G * per; e += EPI_THREADS) {
                const int n = e / per, c16 = e % per;
                const __nv_bfloat16 *src = (n < G ? p.qt_hi : p.qt_lo) + base +
                                           (size_t)(n % G) * p.rk + c16 * 8;
                const int k = c16 * 8;
                *reinterpret_cast<uint4 *>(qbuf + kmaj_off(n, k, ATOM)) =
                    *reinterpret_cast<const uint4 *>(src);
            }
        };
        // q~ comes from the kernel before (the copies of A started without waiting for it)
        grid_dep_wait();
        if (blockIdx.x < p.n_items) write_q(blockIdx.x);
        fence_async_smem();
        ra_epi_bar();
        if (et == 0) mbar_arrive(&sh->q_full);
        int ic = 0, item = blockIdx.x;
        for (; item < p.n_items; item += gridDim.x, ++ic) {
            const RaItem w = ra_decode(p, item);
            {
                const bool fail = !ra_wait(&sh->z_full, ic & 1, sh, p);
                if (ra_epi_bar_any(fail)) break;
            }
            tcgen05_after();
            float z[2][G];
#pragma unroll
            for (int th = 0; th < 2; ++th) {
                if (th * 128 < w.nr) {
                    float v[NO];
                    if constexpr (NO == 8)
                        tmem_load8(tmem + lane_base + TM_Z + th * NO, v);
                    else
                        tmem_load16(tmem + lane_base + TM_Z + th * NO, v);
                    const bool valid = th * 128 + lrow < w.nr;
#pragma unroll
                    for (int h = 0; h < G; ++h)
                        z[th][h] = valid ? (v[h] + v[G + h]) * p.qscale : -INFINITY;
                } else {
#pragma unroll
                    for (int h = 0; h < G; ++h) z[th][h] = -INFINITY;
                }
            }
            float m[G], l[G];
#pragma unroll
            for (int h = 0; h < G; ++h) {
                m[h] = fmaxf(z[0][h], z[1][h]);
#pragma unroll
                for (int off = 16; off; off >>= 1)
                    m[h] = fmaxf(m[h], __shfl_xor_sync(0xffffffffu, m[h], off));
                if (lane == 0) sh->red[ew][h] = m[h];
            }
            ra_epi_bar();
#pragma unroll
            for (int h = 0; h < G; ++h) {
                m[h] = fmaxf(fmaxf(sh->red[0][h], sh->red[1][h]),
                             fmaxf(sh->red[2][h], sh->red[3][h]));
                l[h] = 0.f;
            }
            ra_epi_bar();
#pragma unroll
            for (int th = 0; th < 2; ++th) {
                const int k = th * 128 + lrow;
#pragma unroll
                for (int h = 0; h < G; ++h) {
                    const float pv = exp2f(z[th][h] - m[h]);   // 0 past the item's rows
                    l[h] += pv;
                    const __nv_bfloat16 hi = __float2bfloat16_rn(pv);
                    const __nv_bfloat16 lo = __float2bfloat16_rn(pv - __bfloat162float(hi));
                    *reinterpret_cast<__nv_bfloat16 *>(pbuf + kmaj_off(h, k, ATOM)) = hi;
                    *reinterpret_cast<__nv_bfloat16 *>(pbuf + kmaj_off(G + h, k, ATOM)) = lo;
                }
            }
#pragma unroll
            for (int h = 0; h < G; ++h) {
#pragma unroll
                for (int off = 16; off; off >>= 1) l[h] += __shfl_xor_sync(0xffffffffu, l[h], off);
                if (lane == 0) sh->red[ew][h] = l[h];
            }
            fence_async_smem();
            tcgen05_before();
            ra_epi_bar();
            if (et == 0) mbar_arrive(&sh->p_full);
            // the logit MMAs of this item are done: Q~ takes the next item's rows while
            // the value MMAs of this one run
            if (item + (int)gridDim.x < p.n_items) {
                write_q(item + gridDim.x);
                fence_async_smem();
                ra_epi_bar();
                if (et == 0) mbar_arrive(&sh->q_full);
            }
#pragma unroll
            for (int h = 0; h < G; ++h)
                l[h] = (sh->red[0][h] + sh->red[1][h]) + (sh->red[2][h] + sh->red[3][h]);
            {
                const bool fail = !ra_wait(&sh->o_full, ic & 1, sh, p);
                if (ra_epi_bar_any(fail)) break;
            }
            tcgen05_after();
            float *dst = p.partials + (((size_t)w.split * p.B + w.b) * p.Hq + (size_t)w.g * G) *
                                          (p.rv + 2);
            for (int sb = 0; sb < p.rv / 128; ++sb) {
                float v[NO];
                if constexpr (NO == 8)
                    tmem_load8(tmem + lane_base + TM_U + sb * NO, v);
                else
                    tmem_load16(tmem + lane_base + TM_U + sb * NO, v);
#pragma unroll
                for (int h = 0; h < G; ++h)
                    dst[(size_t)h * (p.rv + 2) + 2 + sb * 128 + lrow] = v[h] + v[G + h];
            }
            tcgen05_before();
            if (et == 0) {
#pragma unroll
                for (int h = 0; h < G; ++h) {
                    dst[(size_t)h * (p.rv + 2)] = m[h] * 0.6931471805599453f;   // natural log
                    dst[(size_t)h * (p.rv + 2) + 1] = l[h];
                }
            }
            ra_epi_bar();                            // red is rewritten by the next item
        }
    }
    tcgen05_before();
    __syncthreads();
    tcgen05_after();
    if (warp == W_MMA)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 256;" ::"r"(tmem)
                     : "memory");
}

// ------------------------------------------------------------------ dense, all heads
// Dense mode (every head attends every row): the rows of A are the same for all Hq heads
// of a sequence, so the per-(b, g) items above would stream the window once per KV head.
// k_xkv_ra_dense instead gives one CTA a span of the sequence's rows and all of its
// heads, so A^K and A^V each cross HBM once per layer:
//   pass 1, per 128-token tile: D_z[t][n] = A^K[t][:] . Q~[n][:]  (M = 128 tokens,
//           N = NO = the hi and lo rows of the Hq heads), the logits z_h = D_z[t][h] +
//           D_z[t][Hq + h] go to a global scratch (L2-resident: the same thread reads
//           them back in pass 2) and the span's max per head is kept;
//   pass 2, per tile: P[n][t] = exp2(z - m) as hi + lo bf16 rows, then
//           D_u[r][n] += A^V[t][r] P[n][t]  (M = 128 rank columns per block, N = NO,
//           K = tokens), accumulated in tensor memory over the whole span;
//   end:    the span's (m, l, u) partial in rank space, merged across spans by k_merge_project_ra
//           (k_merge_ra and k_project_ra when the spans are few).
// A stage is 128 tokens x 128 rank columns in 16 copies of the 3D view (64, rows, column
// blocks) of A, one per 8-row group, each landing as two consecutive 64-column atoms (the
// layout of k_xkv_ra): logits use A K-major (8-row groups 2 KB apart), the value product
// reads the same stage MN-major (64-column atoms 1 KB apart, 8-token groups 2 KB apart).  TMEM: two logit buffers, then the
// r_V / 128 accumulator blocks, NO columns each.  Warp roles: warp 0 TMEM + MMA issue,
// warp 1 the copies, warps 2-5 the epilogue (thread = TMEM lane = token, or rank column
// at the end).
constexpr int DN_TILE = 128;                     // tokens per tile
constexpr int DN_STAGE = DN_TILE * 128 * 2;      // 128 tokens x 128 rank columns: 32 KB
constexpr int DN_STAGES = 4;
constexpr int DN_SPANS = 148;                    // spans per batch: one per SM of a B200
constexpr int DW_MMA = 0, DW_LOAD = 1, DW_EPI = 2, DN_EPI = 4;
constexpr int DN_THREADS = 32 * (DW_EPI + DN_EPI);   // 192
constexpr int DN_EPI_THREADS = 32 * DN_EPI;           // 128

struct DnShared {
    uint64_t full[DN_STAGES], empty[DN_STAGES];
    uint64_t q_full, zfull[2], zfree[2], pfull[2], pfree[2], ufull, ufree, idle;
    uint32_t tmem_base;
    int abort;
    float red[DN_EPI][32];
};

struct DnParams {
    const __nv_bfloat16 *qt_hi, *qt_lo;   // [B][Hq][r_K]
    float *partials;                      // [n_span][B][Hq][r_V + 2]
    float *z;                             // [B][Hq][tiles * 128] logits, log2 domain
    unsigned *status;
    int64_t L;
    int rk, rv, B;
    int rows_all;                         // B * L: rows of the 3D views
    int tiles, tps, n_span, n_items;
    float qscale;                         // log2(e) / sqrt(hd)
    uint32_t mma_spin;                    // poll limit of the MMA issuer's waits for staged data
};

template <int HQ> struct DnCfg {
    static constexpr int NO = (2 * HQ + 15) / 16 * 16;   // MMA N: hi and lo rows, padded
    static constexpr int ATOM = NO / 8 * 1024;           // bytes per 64-wide K atom
    static constexpr int PBUF = 2 * ATOM;                 // P: NO rows x 128 tokens
};

__device__ __forceinline__ void dn_epi_bar() {
    asm volatile("bar.sync 1, %0;" ::"n"(DN_EPI_THREADS) : "memory");
}
__device__ __forceinline__ bool dn_epi_bar_any(bool flag) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred pin, pout;\n\t"
        "setp.ne.u32 pin, %1, 0;\n\t"
        "bar.red.or.pred pout, 1, %2, pin;\n\t"
        "selp.u32 %0, 1, 0, pout;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)flag), "n"(DN_EPI_THREADS)
        : "memory");
    return r != 0;
}
__device__ __forceinline__ bool dn_wait(uint64_t *b, uint32_t parity, DnShared *sh,
                                        unsigned *status, uint32_t limit = RA_SPIN) {
    if (mbar_wait_bounded(b, parity, &sh->abort, limit)) return true;
    if (!*(volatile int *)&sh->abort) {
        *(volatile int *)&sh->abort = 1;
        grid_dep_wait();    // after q~'s clear of the status word
        if (status) atomicOr(status, 1u << XKV_ERR_TIMEOUT);
    }
    return false;
}
// N consecutive fp32 TMEM columns of this thread's lane, N a multiple of 16
template <int N>
__device__ __forceinline__ void tmem_load_cols(uint32_t taddr, float *v) {
    if constexpr (N >= 32) {
        tmem_load32(taddr, *reinterpret_cast<float(*)[32]>(v));
        tmem_load_cols<N - 32>(taddr + 32, v + 32);
    } else if constexpr (N >= 16) {
        tmem_load16(taddr, *reinterpret_cast<float(*)[16]>(v));
    }
}

struct DnItem {
    int b, span, t0, nt;   // sequence, span, first tile, tiles
};
__device__ __forceinline__ DnItem dn_decode(const DnParams &p, int item) {
    DnItem it;
    it.b = item / p.n_span;
    it.span = item % p.n_span;
    it.t0 = it.span * p.tps;
    it.nt = min(p.tps, p.tiles - it.t0);
    return it;
}

template <int HQ>
__global__ void __launch_bounds__(DN_THREADS, 1)
    k_xkv_ra_dense(const __grid_constant__ CUtensorMap tmAk,
                   const __grid_constant__ CUtensorMap tmAv, const DnParams p) {
    using Cfg = DnCfg<HQ>;
    constexpr int NO = Cfg::NO, ATOM = Cfg::ATOM, PBUF = Cfg::PBUF;
    constexpr uint32_t TM_Z = 0, TM_U = 2 * NO;
    extern __shared__ unsigned char smem_raw[];
    unsigned char *smem = (unsigned char *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    unsigned char *qbuf = smem + DN_STAGES * DN_STAGE;
    unsigned char *pbuf = qbuf + (p.rk / 64) * ATOM;      // two P buffers
    DnShared *sh = reinterpret_cast<DnShared *>(pbuf + 2 * PBUF);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < DN_STAGES; ++s) {
            mbar_init(&sh->full[s], 1);
            mbar_init(&sh->empty[s], 1);
        }
        mbar_init(&sh->q_full, 1);
        for (int i = 0; i < 2; ++i) {
            mbar_init(&sh->zfull[i], 1);
            mbar_init(&sh->zfree[i], 1);
            mbar_init(&sh->pfull[i], 1);
            mbar_init(&sh->pfree[i], 1);
        }
        mbar_init(&sh->ufull, 1);
        mbar_init(&sh->ufree, 1);
        mbar_init(&sh->idle, 1);
        sh->abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        prefetch_tmap(&tmAk);
        prefetch_tmap(&tmAv);
    }
    if (warp == DW_MMA) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 512;" ::"r"(
                         su32(&sh->tmem_base))
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tcgen05_before();
    __syncthreads();
    tcgen05_after();
    const uint32_t tmem = sh->tmem_base;

    if (warp == DW_LOAD) {
        // ------------------------------------------------------------ copies (one thread)
        if (lane == 0) {
            int it = 0;
            bool ok = true;
            for (int item = blockIdx.x; item < p.n_items && ok; item += gridDim.x) {
                const DnItem w = dn_decode(p, item);
                const int row0 = (int)((int64_t)w.b * p.L + (int64_t)w.t0 * DN_TILE);
                for (int phase = 0; phase < 2 && ok; ++phase) {
                    const int nst = (phase == 0 ? p.rk : p.rv) / 128;
                    const CUtensorMap *m = phase == 0 ? &tmAk : &tmAv;
                    for (int i = 0; i < w.nt && ok; ++i)
                        for (int st = 0; st < nst; ++st, ++it) {
                            const int s = it % DN_STAGES, n = it / DN_STAGES;
                            if (!dn_wait(&sh->empty[s], (n & 1) ^ 1, sh, p.status)) {
                                ok = false;
                                break;
                            }
                            mbar_expect_tx(&sh->full[s], (uint32_t)DN_STAGE);
                            // 16 copies of one 8-row group each (both 64-column atoms):
                            // many copies in flight stream faster than one 32 KB box.  A
                            // group past the batch's last row re-reads the last group (its
                            // rows are masked: logit -inf, weight 0)
                            const int base = row0 + i * DN_TILE;
#pragma unroll
                            for (int gr = 0; gr < DN_TILE / 8; ++gr) {
                                int row = base + gr * 8;
                                row = row < p.rows_all - 8 ? row : p.rows_all - 8;
                                tma_load_3d(m, &sh->full[s], smem + s * DN_STAGE + gr * 2048, 0,
                                            row, st * 2);
                            }
                        }
                }
            }
            if (!ok) {
                // the copies issued into the last DN_STAGES stages land before the CTA leaves
                for (int j = it - DN_STAGES > 0 ? it - DN_STAGES : 0; j < it; ++j)
                    for (uint32_t i = 0; i < RA_SPIN; ++i)
                        if (mbar_test(&sh->full[j % DN_STAGES], (uint32_t)(j / DN_STAGES) & 1))
                            break;
            }
        }
        __syncwarp();
    } else if (warp == DW_MMA) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint32_t sbase = su32(smem), qb = su32(qbuf), pb = su32(pbuf);
            constexpr uint32_t idZ = idesc_f16(128, NO, false, false);
            constexpr uint32_t idU = idesc_f16(128, NO, true, false);   // A^V read MN-major
            int it = 0, zt = 0, pt = 0, ic = 0;
            bool ok = true;
            for (int item = blockIdx.x; item < p.n_items && ok; item += gridDim.x, ++ic) {
                const DnItem w = dn_decode(p, item);
                if (!dn_wait(&sh->q_full, ic & 1, sh, p.status)) break;
                tcgen05_after();
                // pass 1: logits of each tile into TMEM buffer zt & 1
                for (int i = 0; i < w.nt && ok; ++i, ++zt) {
                    const int zb = zt & 1;
                    if (!dn_wait(&sh->zfree[zb], ((zt >> 1) & 1) ^ 1, sh, p.status)) {
                        ok = false;
                        break;
                    }
                    tcgen05_after();
                    for (int st = 0; st < p.rk / 128; ++st, ++it) {
                        const int s = it % DN_STAGES, n = it / DN_STAGES;
                        if (!dn_wait(&sh->full[s], n & 1, sh, p.status, p.mma_spin)) {
                            ok = false;
                            break;
                        }
                        tcgen05_after();
                        const uint32_t a0 = sbase + s * DN_STAGE;
#pragma unroll
                        for (int kk = 0; kk < 8; ++kk) {
                            const int k0 = st * 128 + kk * 16;
                            umma_f16(tmem + TM_Z + zb * NO,
                                     smem_desc_sw128(a0 + (kk >> 2) * 1024 + (kk & 3) * 32, 16, 2048),
                                     smem_desc_sw128(qb + (k0 >> 6) * ATOM + ((k0 & 63) >> 4) * 32, 16, 1024),
                                     idZ, (st | kk) ? 1u : 0u);
                        }
                        umma_arrive(&sh->empty[s]);
                    }
                    if (ok) umma_arrive(&sh->zfull[zb]);
                }
                if (!ok) break;
                // pass 2: the span's value products, accumulated over its tiles
                if (!dn_wait(&sh->ufree, (ic & 1) ^ 1, sh, p.status)) break;
                tcgen05_after();
                for (int i = 0; i < w.nt && ok; ++i, ++pt) {
                    const int pbi = pt & 1;
                    if (!dn_wait(&sh->pfull[pbi], (pt >> 1) & 1, sh, p.status)) {
                        ok = false;
                        break;
                    }
                    tcgen05_after();
                    for (int st = 0; st < p.rv / 128; ++st, ++it) {
                        const int s = it % DN_STAGES, n = it / DN_STAGES;
                        if (!dn_wait(&sh->full[s], n & 1, sh, p.status, p.mma_spin)) {
                            ok = false;
                            break;
                        }
                        tcgen05_after();
                        const uint32_t a0 = sbase + s * DN_STAGE;
#pragma unroll
                        for (int kt = 0; kt < 8; ++kt)
                            umma_f16(tmem + TM_U + st * NO,
                                     smem_desc_sw128(a0 + kt * 4096, 1024, 2048),
                                     smem_desc_sw128(pb + pbi * PBUF + (kt >> 2) * ATOM + (kt & 3) * 32, 16, 1024),
                                     idU, (i | kt) ? 1u : 0u);
                        umma_arrive(&sh->empty[s]);
                    }
                    if (ok) umma_arrive(&sh->pfree[pbi]);
                }
                if (!ok) break;
                umma_arrive(&sh->ufull);
            }
            // every MMA this thread issued has completed once `idle` fires
            umma_arrive(&sh->idle);
            for (uint32_t i = 0; i < RA_SPIN; ++i)
                if (mbar_test(&sh->idle, 0)) break;
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ epilogue
        const int et = threadIdx.x - 32 * DW_EPI;   // 0..127
        const int ew = warp - DW_EPI;
        const int quad = warp & 3;                  // TMEM lane quadrant of this warp
        const int lrow = quad * 32 + lane;          // token of a tile / rank column of a block
        const uint32_t lane_base = (uint32_t)(quad * 32) << 16;
        // zero Q~ and both P buffers: the padding rows n >= 2 Hq stay zero
        for (int i = et; i < ((p.rk / 64) * ATOM + 2 * PBUF) / 16; i += DN_EPI_THREADS)
            reinterpret_cast<uint4 *>(qbuf)[i] = make_uint4(0u, 0u, 0u, 0u);
        dn_epi_bar();
        auto write_q = [&](int b) {                 // Q~ rows: hi of the Hq heads, then lo
            const size_t base = (size_t)b * HQ * p.rk;
            const int per = p.rk / 8;               // 16-byte pieces per row
            for (int e = et; e < 2 * HQ * per; e += DN_EPI_THREADS) {
                const int n = e / per, c16 = e % per;
                const __nv_bfloat16 *src =
                    (n < HQ ? p.qt_hi : p.qt_lo) + base + (size_t)(n % HQ) * p.rk + c16 * 8;
                *reinterpret_cast<uint4 *>(qbuf + kmaj_off(n, c16 * 8, ATOM)) =
                    *reinterpret_cast<const uint4 *>(src);
            }
        };
        // q~ comes from the kernel before (the copies of A started without waiting for it)
        grid_dep_wait();
        if (blockIdx.x < p.n_items) write_q(dn_decode(p, blockIdx.x).b);
        fence_async_smem();
        dn_epi_bar();
        if (et == 0) mbar_arrive(&sh->q_full);
        int zt = 0, pt = 0, ic = 0;
        bool dead = false;
        for (int item = blockIdx.x; item < p.n_items && !dead; item += gridDim.x, ++ic) {
            const DnItem w = dn_decode(p, item);
            float m[HQ];
#pragma unroll
            for (int h = 0; h < HQ; ++h) m[h] = -INFINITY;
            // logits of tile (b, t): one contiguous block of HQ x 128 floats, so a tile's
            // stores and loads stay within a few pages
            auto zblk = [&](int i) {
                return p.z + ((size_t)w.b * p.tiles + (size_t)(w.t0 + i)) * HQ * DN_TILE;
            };
            // pass 1: logits to the scratch, running max
            for (int i = 0; i < w.nt; ++i, ++zt) {
                const int zb = zt & 1;
                {
                    const bool fail = !dn_wait(&sh->zfull[zb], (zt >> 1) & 1, sh, p.status);
                    if (dn_epi_bar_any(fail)) { dead = true; break; }
                }
                tcgen05_after();
                float v[NO];
                tmem_load_cols<NO>(tmem + lane_base + TM_Z + zb * NO, v);
                tcgen05_before();
                const int64_t t = (int64_t)(w.t0 + i) * DN_TILE + lrow;
                const bool valid = t < p.L;
#pragma unroll
                for (int h = 0; h < HQ; ++h) {
                    const float zh = valid ? (v[h] + v[HQ + h]) * p.qscale : -INFINITY;
                    m[h] = fmaxf(m[h], zh);
                    zblk(i)[h * DN_TILE + lrow] = zh;
                }
                dn_epi_bar();
                if (et == 0) mbar_arrive(&sh->zfree[zb]);
            }
            if (dead) break;
            // the first tile's logits are loaded before the max reduction, each later
            // tile's right after the previous P is published (same thread, program order)
            float zl[HQ];
            auto load_z = [&](int i) {
                const float *zb = zblk(i);
#pragma unroll
                for (int h = 0; h < HQ; ++h) zl[h] = __ldcg(zb + h * DN_TILE + lrow);
            };
            if (w.nt > 0) load_z(0);
            // the span's max per head
#pragma unroll
            for (int h = 0; h < HQ; ++h) {
#pragma unroll
                for (int off = 16; off; off >>= 1)
                    m[h] = fmaxf(m[h], __shfl_xor_sync(0xffffffffu, m[h], off));
                if (lane == 0) sh->red[ew][h] = m[h];
            }
            dn_epi_bar();
#pragma unroll
            for (int h = 0; h < HQ; ++h)
                m[h] = fmaxf(fmaxf(sh->red[0][h], sh->red[1][h]), fmaxf(sh->red[2][h], sh->red[3][h]));
            dn_epi_bar();
            // every logit MMA of this item has completed: Q~ takes the next item's rows
            if (item + (int)gridDim.x < p.n_items) {
                write_q(dn_decode(p, item + gridDim.x).b);
                fence_async_smem();
                dn_epi_bar();
                if (et == 0) mbar_arrive(&sh->q_full);
            }
            // pass 2: probabilities of each tile into P buffer pt & 1
            float l[HQ];
#pragma unroll
            for (int h = 0; h < HQ; ++h) l[h] = 0.f;
            for (int i = 0; i < w.nt; ++i, ++pt) {
                const int pbi = pt & 1;
                {
                    const bool fail = !dn_wait(&sh->pfree[pbi], ((pt >> 1) & 1) ^ 1, sh, p.status);
                    if (dn_epi_bar_any(fail)) { dead = true; break; }
                }
                unsigned char *pdst = pbuf + pbi * PBUF;
#pragma unroll
                for (int h = 0; h < HQ; ++h) {
                    const float pv = exp2f(zl[h] - m[h]);   // 0 past L
                    l[h] += pv;
                    const __nv_bfloat16 hi = __float2bfloat16_rn(pv);
                    const __nv_bfloat16 lo = __float2bfloat16_rn(pv - __bfloat162float(hi));
                    *reinterpret_cast<__nv_bfloat16 *>(pdst + kmaj_off(h, lrow, ATOM)) = hi;
                    *reinterpret_cast<__nv_bfloat16 *>(pdst + kmaj_off(HQ + h, lrow, ATOM)) = lo;
                }
                fence_async_smem();
                dn_epi_bar();
                if (et == 0) mbar_arrive(&sh->pfull[pbi]);
                if (i + 1 < w.nt) load_z(i + 1);
            }
            if (dead) break;
#pragma unroll
            for (int h = 0; h < HQ; ++h) {
#pragma unroll
                for (int off = 16; off; off >>= 1) l[h] += __shfl_xor_sync(0xffffffffu, l[h], off);
                if (lane == 0) sh->red[ew][h] = l[h];
            }
            {
                const bool fail = !dn_wait(&sh->ufull, ic & 1, sh, p.status);
                if (dn_epi_bar_any(fail)) break;       // also publishes red
            }
#pragma unroll
            for (int h = 0; h < HQ; ++h)
                l[h] = (sh->red[0][h] + sh->red[1][h]) + (sh->red[2][h] + sh->red[3][h]);
            tcgen05_after();
            float *dst = p.partials + ((size_t)w.span * p.B + w.b) * HQ * (p.rv + 2);
            for (int sb = 0; sb < p.rv / 128; ++sb) {
                float v[NO];
                tmem_load_cols<NO>(tmem + lane_base + TM_U + sb * NO, v);
#pragma unroll
                for (int h = 0; h < HQ; ++h)
                    dst[(size_t)h * (p.rv + 2) + 2 + sb * 128 + lrow] = v[h] + v[HQ + h];
            }
            tcgen05_before();
            if (et == 0) {
#pragma unroll
                for (int h = 0; h < HQ; ++h) {
                    dst[(size_t)h * (p.rv + 2)] = m[h] * 0.6931471805599453f;   // natural log
                    dst[(size_t)h * (p.rv + 2) + 1] = l[h];
                }
            }
            dn_epi_bar();                            // red is rewritten by the next item
            if (et == 0) mbar_arrive(&sh->ufree);
        }
    }
    tcgen05_before();
    __syncthreads();
    tcgen05_after();
    if (warp == DW_MMA)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 512;" ::"r"(tmem)
                     : "memory");
}

// q~[b][h][i] = sum_j q[b][h][j] B^K[b][i][g*hd + j]  (Bkt row g*hd + j holds column j of
// the group's slice), fp32, then split into the bf16 nearest and the bf16 of the rest.
// One CTA per (b, g, 32 CPL columns i): warp w takes rows j = w, w + 8, ... of the slice,
// each lane CPL columns (all 16 rows' loads in flight), and the 8 warps' sums meet in
// shared memory.  The host takes CPL = 1 when the CPL = 4 grid would leave SMs idle
// (batch 1: 16 slices per KV head at rank 512), else CPL = 4.
template <int G, int CPL>
__global__ void __launch_bounds__(256) k_qtilde(const __nv_bfloat16 *__restrict__ q,
                                                const __nv_bfloat16 *__restrict__ Bkt,
                                                __nv_bfloat16 *__restrict__ qt_hi,
                                                __nv_bfloat16 *__restrict__ qt_lo, int Hq,
                                                int Hkv, int hd, int rk,
                                                unsigned *__restrict__ status,
                                                unsigned *__restrict__ arrived) {
    __shared__ float qs[G * 128];                  // [G][hd]
    // the attention kernel after this one may start streaming the rows of A at once: it
    // waits for this grid only where it reads q~ or writes the status word
    grid_dep_launch();
    // the call's device-side error word starts clean: this kernel runs first in the call,
    // so the clear is ordered before every kernel that may set it
    if (status && (blockIdx.x | blockIdx.y | blockIdx.z | threadIdx.x) == 0) *status = 0u;
    // so do the per-(b, h) arrival counters of the merge + projection kernel
    if ((blockIdx.x | blockIdx.y | blockIdx.z) == 0)
        for (int e = threadIdx.x; e < Hq * gridDim.y; e += blockDim.x) arrived[e] = 0u;
    constexpr int QT_COLS = 32 * CPL;
    __shared__ float red[8][G][QT_COLS];
    const int g = blockIdx.x, b = blockIdx.y, i0 = blockIdx.z * QT_COLS;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const __nv_bfloat16 *Bg =
        Bkt + ((size_t)b * Hkv * hd + (size_t)g * hd) * rk + i0 + lane * CPL;
    // this warp's rows j = warp, warp + 8, ... (hd <= 128: at most 16) are loaded before
    // the query is staged, so the two loads overlap
    constexpr int RPW = 16;
    float bv[RPW][CPL];
#pragma unroll
    for (int i = 0; i < RPW; ++i) {
        const int j = warp + 8 * i;
        if constexpr (CPL == 4) {
            uint2 w2 = make_uint2(0u, 0u);
            if (j < hd) w2 = *reinterpret_cast<const uint2 *>(Bg + (size_t)j * rk);
            bv[i][0] = bf16lo(w2.x);
            bv[i][1] = bf16hi(w2.x);
            bv[i][2] = bf16lo(w2.y);
            bv[i][3] = bf16hi(w2.y);
        } else {
            bv[i][0] = j < hd ? __bfloat162float(Bg[(size_t)j * rk]) : 0.f;
        }
    }
    for (int e = threadIdx.x; e < G * hd; e += blockDim.x)
        qs[e] = __bfloat162float(q[((size_t)b * Hq + (size_t)g * G) * hd + e]);
    __syncthreads();
    float acc[G][CPL];
#pragma unroll
    for (int h = 0; h < G; ++h)
#pragma unroll
        for (int c = 0; c < CPL; ++c) acc[h][c] = 0.f;
#pragma unroll
    for (int i = 0; i < RPW; ++i) {
        const int j = warp + 8 * i;
        if (j < hd) {
#pragma unroll
            for (int h = 0; h < G; ++h) {
                const float qv = qs[h * hd + j];
#pragma unroll
                for (int c = 0; c < CPL; ++c) acc[h][c] = fmaf(qv, bv[i][c], acc[h][c]);
            }
        }
    }
#pragma unroll
    for (int h = 0; h < G; ++h)
#pragma unroll
        for (int c = 0; c < CPL; ++c) red[warp][h][lane * CPL + c] = acc[h][c];
    __syncthreads();
    for (int e = threadIdx.x; e < G * QT_COLS; e += blockDim.x) {
        const int h = e / QT_COLS, c = e % QT_COLS;
        float v = 0.f;
#pragma unroll
        for (int w = 0; w < 8; ++w) v += red[w][h][c];
        const size_t o = ((size_t)b * Hq + (size_t)g * G + h) * rk + i0 + c;
        const __nv_bfloat16 hi = __float2bfloat16_rn(v);
        qt_hi[o] = hi;
        qt_lo[o] = __float2bfloat16_rn(v - __bfloat162float(hi));
    }
}

// Merge an item's splits in rank space:
//   M = max_s m_s,  U_h[r] = sum_s e^{m_s - M} u_s[r],  L_h = sum_s e^{m_s - M} l_s.
// (A one-pass form with a running max per warp was measured slower at the 147 spans of a
// dense batch-1 call.)
// One CTA per (b, h, 32 CPL columns of r): warp w takes the splits s = w, w + 8, ..., each
// lane CPL columns (coalesced 128-byte rows; the loop is unrolled so that several splits'
// loads are in flight); the 8 warps' sums meet in shared memory.  The host takes CPL = 2
// when the CPL = 8 grid would leave SMs idle (the 147 spans of a dense batch-1 call), else
// CPL = 8.
constexpr int MG_THREADS = 256;
template <int CPL>
__global__ void __launch_bounds__(MG_THREADS) k_merge_ra(const float *__restrict__ partials,
                                                         float *__restrict__ U,
                                                         float *__restrict__ Lsum, int n_split,
                                                         int BH, int rv,
                                                         const unsigned *__restrict__ status) {
    constexpr int MG_COLS = 32 * CPL;
    __shared__ float red[MG_THREADS / 32][MG_COLS];
    __shared__ float s_m[MG_THREADS / 32];
    __shared__ float s_l[MG_THREADS / 32];
    const int bh = blockIdx.x, r0 = blockIdx.y * MG_COLS;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    constexpr int NW = MG_THREADS / 32;
    if (status && *(volatile const unsigned *)status) return;   // outputs become NaN anyway
    const size_t stride = (size_t)BH * (rv + 2);
    const float *p = partials + (size_t)bh * (rv + 2);
    float M = -INFINITY;
    for (int sp = threadIdx.x; sp < n_split; sp += MG_THREADS) M = fmaxf(M, p[sp * stride]);
#pragma unroll
    for (int off = 16; off; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
    if (lane == 0) s_m[warp] = M;
    __syncthreads();
    M = s_m[0];
#pragma unroll
    for (int w = 1; w < NW; ++w) M = fmaxf(M, s_m[w]);
    float acc[CPL], l = 0.f;
#pragma unroll
    for (int k = 0; k < CPL; ++k) acc[k] = 0.f;
#pragma unroll 8
    for (int sp = warp; sp < n_split; sp += NW) {
        const float *ps = p + sp * stride;
        const float wgt = expf(ps[0] - M);
        l = fmaf(wgt, ps[1], l);
#pragma unroll
        for (int k = 0; k < CPL; ++k) {
            const int r = r0 + lane + 32 * k;
            if (r < rv) acc[k] = fmaf(wgt, ps[2 + r], acc[k]);
        }
    }
#pragma unroll
    for (int k = 0; k < CPL; ++k) red[warp][lane + 32 * k] = acc[k];
    if (lane == 0) s_l[warp] = l;
    __syncthreads();
    const int r = r0 + threadIdx.x;
    if (threadIdx.x < MG_COLS && r < rv) {
        float sum = 0.f;
#pragma unroll
        for (int w = 0; w < NW; ++w) sum += red[w][threadIdx.x];
        U[(size_t)bh * rv + r] = sum;
    }
    if (blockIdx.y == 0 && threadIdx.x == 0) {
        float ls = 0.f;
#pragma unroll
        for (int w = 0; w < NW; ++w) ls += s_l[w];
        Lsum[bh] = ls;
    }
}

// out[b][h][j] = (U_h . B^V[:, g*hd + j]) / L_h.  One CTA per (b, g, 8 RPW columns j): each
// warp takes RPW rows j of Bvt, so the group's B^V slice is read once for its G heads; the
// 32 / RPW lanes of a row take its 16-byte pieces in turn (all in flight) and sum their
// partial dot products with shuffles.  The host takes RPW = 1 (more, smaller CTAs) when
// the RPW = 4 grid would leave SMs idle, else RPW = 4.
template <int G, int RPW>
__global__ void __launch_bounds__(256) k_project_ra(const float *__restrict__ U,
                                                    const float *__restrict__ Lsum,
                                                    const __nv_bfloat16 *__restrict__ Bvt,
                                                    float *__restrict__ out, int Hq, int Hkv,
                                                    int hd, int rv,
                                                    const unsigned *__restrict__ status) {
    constexpr int PJ_ROWS = 8 * RPW, LPR = 32 / RPW;   // rows per CTA, lanes per row
    extern __shared__ float Us[];                 // [G][rv]
    const int g = blockIdx.x, b = blockIdx.y, j0 = blockIdx.z * PJ_ROWS;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const size_t bh0 = (size_t)b * Hq + (size_t)g * G;
    const int c = lane % LPR;
    const int j = j0 + warp * RPW + lane / LPR;
    const __nv_bfloat16 *row = Bvt + ((size_t)b * Hkv * hd + (size_t)g * hd + j) * rv;
    // the first pieces of the row are loaded before U is staged, so the two loads overlap
    constexpr int PRE = 4;
    uint4 pre[PRE];
#pragma unroll
    for (int i = 0; i < PRE; ++i) {
        const int pc = c + i * LPR;
        pre[i] = pc < rv / 8 ? *reinterpret_cast<const uint4 *>(row + pc * 8)
                             : make_uint4(0u, 0u, 0u, 0u);
    }
    if (status && *(volatile const unsigned *)status) {   // a device-side failure: NaN out
        for (int e = threadIdx.x; e < G * PJ_ROWS; e += blockDim.x)
            out[(bh0 + e / PJ_ROWS) * hd + j0 + e % PJ_ROWS] = __int_as_float(0x7fc00000);
        return;
    }
    for (int e = threadIdx.x; e < G * rv; e += blockDim.x) Us[e] = U[bh0 * rv + e];
    __syncthreads();
    float acc[G];
#pragma unroll
    for (int h = 0; h < G; ++h) acc[h] = 0.f;
    // 16-byte piece pc holds columns 8 pc .. 8 pc + 7 of the row
    auto piece = [&](int pc, const uint4 &w4) {
        const float bv[8] = {bf16lo(w4.x), bf16hi(w4.x), bf16lo(w4.y), bf16hi(w4.y),
                             bf16lo(w4.z), bf16hi(w4.z), bf16lo(w4.w), bf16hi(w4.w)};
#pragma unroll
        for (int h = 0; h < G; ++h)
#pragma unroll
            for (int k = 0; k < 8; ++k) acc[h] = fmaf(Us[h * rv + pc * 8 + k], bv[k], acc[h]);
    };
#pragma unroll
    for (int i = 0; i < PRE; ++i)
        if (c + i * LPR < rv / 8) piece(c + i * LPR, pre[i]);
#pragma unroll 4
    for (int pc = c + PRE * LPR; pc < rv / 8; pc += LPR)
        piece(pc, *reinterpret_cast<const uint4 *>(row + pc * 8));
#pragma unroll
    for (int h = 0; h < G; ++h) {
#pragma unroll
        for (int off = LPR / 2; off; off >>= 1) acc[h] += __shfl_xor_sync(0xffffffffu, acc[h], off);
        if (c == 0) out[(bh0 + h) * hd + j] = acc[h] / Lsum[bh0 + h];
    }
}

// Merge of an item's splits in rank space fused with the projection, for calls with many
// splits (dense calls at small batch: one span per SM, so ~148 / B splits per head).  For
// a query head h of group g and a slice of W = 32 CPL rank columns r:
//   M = max_s m_s,  w_s = e^{m_s - M},  L = sum_s w_s l_s,  U[r] = sum_s w_s u_s[r],
//   y[j] = sum_{r in the slice} U[r] B^V[g*hd + j][r],
// and the CTA of h that finishes last sums y over the slices in slice order and writes
// o_h[j] = y[j] / L.  Every CTA of a head forms M and L from all splits in the same
// order, so they agree bit for bit, and the order of the final sum does not depend on
// which CTA is last: the output is reproducible.  The CTA's rows of B^V (128 rows x W
// columns, two threads per row) are loaded first, since they do not depend on the merge.
// Warp w takes the splits s = w, w + 8, ..., each lane CPL columns (coalesced 128-byte
// rows).  The arrival counters are zeroed by k_qtilde, which runs first in every call.
// Each head re-reads its group's B^V slice (from L2), so with few splits the two
// separate kernels above, which read it once per group, are faster; the host takes this
// kernel from MP_MIN_SPLITS splits on.
constexpr int MP_THREADS = 256;
constexpr int MP_HD = 128;
constexpr int MP_MIN_CTAS = 296;   // about two CTAs per SM: the widest slices that keep this
constexpr int MP_MIN_SPLITS = 32;
template <int CPL>
__global__ void __launch_bounds__(MP_THREADS) k_merge_project_ra(
    const float *__restrict__ partials, const __nv_bfloat16 *__restrict__ Bvt,
    float *__restrict__ yparts, unsigned *__restrict__ arrived, float *__restrict__ out,
    int n_split, int BH, int Hq, int Hkv, int rv, const unsigned *__restrict__ status) {
    constexpr int W = 32 * CPL, NW = MP_THREADS / 32, HALF = W / 2, NV = HALF / 8;
    static_assert(MP_THREADS == 2 * MP_HD, "two threads per row of the B^V slice");
    __shared__ float red[NW][W];
    __shared__ float Us[W];
    __shared__ float s_m[NW], s_l[NW];
    __shared__ int s_last;
    const int bh = blockIdx.x, sl = blockIdx.y, n_sl = gridDim.y, r0 = sl * W;
    const int G = Hq / Hkv;
    const int b = bh / Hq, g = (bh % Hq) / G;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int j = threadIdx.x >> 1, half = threadIdx.x & 1;
    const uint4 *brow = reinterpret_cast<const uint4 *>(
        Bvt + ((size_t)b * Hkv * MP_HD + (size_t)g * MP_HD + j) * rv + r0 + half * HALF);
    uint4 bw[NV];
#pragma unroll
    for (int i = 0; i < NV; ++i) bw[i] = brow[i];
    if (status && *(volatile const unsigned *)status) {
        if (sl == 0 && threadIdx.x < MP_HD) out[(size_t)bh * MP_HD + threadIdx.x] = __int_as_float(0x7fc00000);
        return;
    }
    const size_t stride = (size_t)BH * (rv + 2);
    const float *p = partials + (size_t)bh * (rv + 2);
    float M = -INFINITY;
    for (int sp = threadIdx.x; sp < n_split; sp += MP_THREADS) M = fmaxf(M, p[sp * stride]);
#pragma unroll
    for (int off = 16; off; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
    if (lane == 0) s_m[warp] = M;
    __syncthreads();
    M = s_m[0];
#pragma unroll
    for (int w = 1; w < NW; ++w) M = fmaxf(M, s_m[w]);
    float acc[CPL], l = 0.f;
#pragma unroll
    for (int k = 0; k < CPL; ++k) acc[k] = 0.f;
#pragma unroll 8
    for (int sp = warp; sp < n_split; sp += NW) {
        const float *ps = p + sp * stride;
        const float wgt = expf(ps[0] - M);
        l = fmaf(wgt, ps[1], l);
#pragma unroll
        for (int k = 0; k < CPL; ++k) acc[k] = fmaf(wgt, ps[2 + r0 + lane + 32 * k], acc[k]);
    }
#pragma unroll
    for (int k = 0; k < CPL; ++k) red[warp][lane + 32 * k] = acc[k];
    if (lane == 0) s_l[warp] = l;
    __syncthreads();
    if (threadIdx.x < W) {
        float sum = 0.f;
#pragma unroll
        for (int w = 0; w < NW; ++w) sum += red[w][threadIdx.x];
        Us[threadIdx.x] = sum;
    }
    __syncthreads();
    float y = 0.f;
#pragma unroll
    for (int i = 0; i < NV; ++i) {
        const float bv[8] = {bf16lo(bw[i].x), bf16hi(bw[i].x), bf16lo(bw[i].y), bf16hi(bw[i].y),
                             bf16lo(bw[i].z), bf16hi(bw[i].z), bf16lo(bw[i].w), bf16hi(bw[i].w)};
#pragma unroll
        for (int k = 0; k < 8; ++k) y = fmaf(Us[half * HALF + i * 8 + k], bv[k], y);
    }
    y += __shfl_xor_sync(0xffffffffu, y, 1);
    if (half == 0) yparts[((size_t)bh * n_sl + sl) * MP_HD + j] = y;
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) s_last = atomicAdd(&arrived[bh], 1u) == (unsigned)(n_sl - 1);
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    if (threadIdx.x < MP_HD) {
        const float *yu = yparts + (size_t)bh * n_sl * MP_HD + threadIdx.x;
        float sum = 0.f;
        for (int t0 = 0; t0 < n_sl; t0 += 8) {
            float v[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) v[i] = t0 + i < n_sl ? __ldcg(yu + (size_t)(t0 + i) * MP_HD) : 0.f;
#pragma unroll
            for (int i = 0; i < 8; ++i)
                if (t0 + i < n_sl) sum += v[i];
        }
        float L = 0.f;
#pragma unroll
        for (int w = 0; w < NW; ++w) L += s_l[w];
        out[(size_t)bh * MP_HD + threadIdx.x] = sum / L;
    }
}
int mp_cpl(const xkv_dims &d) {
    const int64_t bh = (int64_t)d.batch * d.n_q_heads;
    for (int c = 4; c > 1; c /= 2)
        if (bh * (d.rank_v / (32 * c)) >= MP_MIN_CTAS) return c;
    return 1;
}
// Dense-mode plan: spans of whole 128-token tiles, about one span per SM over the batch.
struct DnPlan {
    int tiles, tps, n_span;
};
DnPlan dense_plan(const xkv_dims &d) {
    DnPlan q;
    q.tiles = (int)((d.ctx_len + DN_TILE - 1) / DN_TILE);
    int ns = DN_SPANS / d.batch;
    ns = ns < 1 ? 1 : (ns > q.tiles ? q.tiles : ns);
    q.tps = (q.tiles + ns - 1) / ns;
    q.n_span = (q.tiles + q.tps - 1) / q.tps;
    return q;
}
template <int HQ>
size_t dn_smem(const xkv_dims &d) {
    return 1024 + (size_t)DN_STAGES * DN_STAGE + (size_t)(d.rank_k / 64) * DnCfg<HQ>::ATOM +
           2 * (size_t)DnCfg<HQ>::PBUF + sizeof(DnShared);
}
template <int HQ>
bool dn_fits(const xkv_dims &d) {
    return (2 + d.rank_v / 128) * DnCfg<HQ>::NO <= 512 && dn_smem<HQ>(d) <= 232448;
}
bool dense_heads_ok(const xkv_dims &d) {
    if ((int64_t)d.batch * d.ctx_len < DN_TILE) return false;   // a copy box fits the rows
    switch (d.n_q_heads) {
        case 8: return dn_fits<8>(d);
        case 16: return dn_fits<16>(d);
        case 24: return dn_fits<24>(d);
        case 32: return dn_fits<32>(d);
        default: return false;
    }
}
template <int HQ>
cudaError_t launch_dense_hq(const xkv_dims &d, const CUtensorMap *maps, const DnParams &dp,
                            cudaStream_t s) {
    const size_t smem = dn_smem<HQ>(d);
    auto k = k_xkv_ra_dense<HQ>;
    cudaError_t e = set_smem_limit((const void *)k, smem);
    if (e != cudaSuccess) return e;
    const int grid = dp.n_items < sm_count() ? dp.n_items : sm_count();
    return launch_chained(k, dim3(grid), dim3(DN_THREADS), smem, s, maps[0], maps[1], dp);
}
cudaError_t launch_dense(const xkv_dims &d, const CUtensorMap *maps, const DnParams &dp,
                         cudaStream_t s) {
    switch (d.n_q_heads) {
        case 8: return launch_dense_hq<8>(d, maps, dp, s);
        case 16: return launch_dense_hq<16>(d, maps, dp, s);
        case 24: return launch_dense_hq<24>(d, maps, dp, s);
        case 32: return launch_dense_hq<32>(d, maps, dp, s);
        default: return cudaErrorInvalidValue;
    }
}

template <int G>
cudaError_t launch_g(const xkv_dims &d, const CUtensorMap *maps, const RaParams &p,
                     const DnParams *dp, const void *q, const void *Bkt, const void *Bvt,
                     __nv_bfloat16 *qt_hi, __nv_bfloat16 *qt_lo, float *yparts,
                     unsigned *arrived, float *out, cudaStream_t s) {
    // narrow slices only where the wide ones leave SMs without a CTA
    const bool few = (int64_t)d.batch * d.n_kv_heads * (d.rank_k / 128) < sm_count();
    if (few)
        k_qtilde<G, 1><<<dim3(d.n_kv_heads, d.batch, d.rank_k / 32), 256, 0, s>>>(
            (const __nv_bfloat16 *)q, (const __nv_bfloat16 *)Bkt, qt_hi, qt_lo, d.n_q_heads,
            d.n_kv_heads, d.head_dim, d.rank_k, p.status, arrived);
    else
        k_qtilde<G, 4><<<dim3(d.n_kv_heads, d.batch, d.rank_k / 128), 256, 0, s>>>(
            (const __nv_bfloat16 *)q, (const __nv_bfloat16 *)Bkt, qt_hi, qt_lo, d.n_q_heads,
            d.n_kv_heads, d.head_dim, d.rank_k, p.status, arrived);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    int n_split = p.n_split;
    if (dp) {
        if ((e = launch_dense(d, maps, *dp, s)) != cudaSuccess) return e;
        n_split = dp->n_span;
    } else {
        const size_t smem =
            1024 + (size_t)RA_STAGES * RA_STAGE + RA_QBUF + RA_PBUF + sizeof(RaShared);
        auto k = k_xkv_ra<G>;
        if ((e = set_smem_limit((const void *)k, smem)) != cudaSuccess) return e;
        const int grid = p.n_items < sm_count() ? p.n_items : sm_count();
        if ((e = launch_chained(k, dim3(grid), dim3(RA_THREADS), smem, s, maps[0], maps[1], p)) !=
            cudaSuccess)
            return e;
    }
    const int BH = d.batch * d.n_q_heads;
    if (n_split >= MP_MIN_SPLITS) {
        const dim3 mgrid(BH, d.rank_v / (32 * mp_cpl(d)));
        switch (mp_cpl(d)) {
#define XKV_MP(C)                                                                              \
    case C:                                                                                    \
        k_merge_project_ra<C><<<mgrid, MP_THREADS, 0, s>>>(p.partials, (const __nv_bfloat16 *)Bvt, \
                                                           yparts, arrived, out, n_split, BH,  \
                                                           d.n_q_heads, d.n_kv_heads, d.rank_v, \
                                                           p.status);                          \
        break;
            XKV_MP(1) XKV_MP(2) XKV_MP(4)
#undef XKV_MP
            default: return cudaErrorInvalidValue;
        }
        return cudaGetLastError();
    }
    // few splits: merge, then project (U and L take the y and counter regions)
    float *U = yparts, *Lsum = (float *)arrived;
    if ((int64_t)BH * ((d.rank_v + 255) / 256) < sm_count())
        k_merge_ra<2><<<dim3(BH, (d.rank_v + 63) / 64), MG_THREADS, 0, s>>>(
            p.partials, U, Lsum, n_split, BH, d.rank_v, p.status);
    else
        k_merge_ra<8><<<dim3(BH, (d.rank_v + 255) / 256), MG_THREADS, 0, s>>>(
            p.partials, U, Lsum, n_split, BH, d.rank_v, p.status);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    const size_t psmem = sizeof(float) * (size_t)G * d.rank_v;
    const bool pj_few = (int64_t)d.n_kv_heads * d.batch * (d.head_dim / 32) < sm_count();
    auto kp = pj_few ? k_project_ra<G, 1> : k_project_ra<G, 4>;
    if ((e = set_smem_limit((const void *)kp, psmem)) != cudaSuccess) return e;
    kp<<<dim3(d.n_kv_heads, d.batch, d.head_dim / (pj_few ? 8 : 32)), 256, psmem, s>>>(
        U, Lsum, (const __nv_bfloat16 *)Bvt, out, d.n_q_heads, d.n_kv_heads, d.head_dim,
        d.rank_v, p.status);
    return cudaGetLastError();
}

}  // namespace

bool attend_ra_shape_ok(const xkv_dims &d) {
    const int G = d.n_q_heads / d.n_kv_heads;
    const int max_rk = G > 4 ? RaCfg<8>::MAXR : RaCfg<4>::MAXR;
    return d.dtype == XKV_BF16 && d.head_dim == 128 &&
           (G == 1 || G == 2 || G == 4 || G == 5 || G == 8) && d.rank_k % 128 == 0 &&
           d.rank_v % 128 == 0 && d.rank_k <= max_rk && d.rank_v <= 1024 &&
           RA_ROWS % d.chunk == 0;
}

int ra_splits(const xkv_dims &d, int n_sel) {
    const int64_t rows = (int64_t)n_sel * d.chunk;
    return (int)((rows + RA_ROWS - 1) / RA_ROWS);
}

// scratch: q~ hi and lo [B][Hq][r_K] bf16, the projected slices y [B][Hq][r_V / W][hd]
// fp32 (W the merge + projection kernel's slice width; with few splits U [B][Hq][r_V]
// instead, which fits), the arrival counters (or L) [B][Hq] 32-bit, then the partials
// [n_split][B][Hq][r_V + 2] fp32; each region starts on a 256-byte boundary
static size_t al256(size_t n) { return (n + 255) / 256 * 256; }
static size_t y_bytes(const xkv_dims &d) {
    return al256((size_t)d.batch * d.n_q_heads * (d.rank_v / (32 * mp_cpl(d))) * MP_HD *
                 sizeof(float));
}
static size_t arrived_bytes(const xkv_dims &d) {
    return al256((size_t)d.batch * d.n_q_heads * sizeof(unsigned));
}
size_t ra_scratch_bytes(const xkv_dims &d, int n_split) {
    const size_t bh = (size_t)d.batch * d.n_q_heads;
    return 2 * al256(bh * d.rank_k * sizeof(__nv_bfloat16)) + y_bytes(d) + arrived_bytes(d) +
           (size_t)n_split * bh * (d.rank_v + 2) * sizeof(float);
}

// Dense calls with a supported head count run the head-batched kernel: partials per span,
// then the logit scratch [B][Hq][tiles * 128] fp32 on a 256-byte boundary.
bool attend_ra_dense_heads(const xkv_dims &d) { return attend_ra_shape_ok(d) && dense_heads_ok(d); }

size_t ra_call_scratch_bytes(const xkv_dims &d, bool dense, int n_sel) {
    if (dense && attend_ra_dense_heads(d)) {
        const DnPlan pl = dense_plan(d);
        const size_t bh = (size_t)d.batch * d.n_q_heads;
        return al256(ra_scratch_bytes(d, pl.n_span)) +
               bh * (size_t)pl.tiles * DN_TILE * sizeof(float);
    }
    return ra_scratch_bytes(d, ra_splits(d, n_sel));
}

cudaError_t launch_attend_ra(const xkv_dims &d, const void *Ak, const void *Av, const void *Bkt,
                             const void *Bvt, const void *q, const int32_t *sel, int n_sel,
                             void *scratch, unsigned *status, float *out, cudaStream_t s) {
    CUtensorMap maps[2];
    if (!make_map_bf16_sw128_cb(&maps[0], Ak, (uint64_t)d.batch * d.ctx_len, d.rank_k, 8, 2) ||
        !make_map_bf16_sw128_cb(&maps[1], Av, (uint64_t)d.batch * d.ctx_len, d.rank_v, 8, 2))
        return cudaErrorInvalidValue;
    const size_t bh = (size_t)d.batch * d.n_q_heads;
    const size_t qt_al = al256(bh * d.rank_k * sizeof(__nv_bfloat16));
    char *sc = (char *)scratch;
    __nv_bfloat16 *qt_hi = (__nv_bfloat16 *)sc;
    __nv_bfloat16 *qt_lo = (__nv_bfloat16 *)(sc + qt_al);
    float *yparts = (float *)(sc + 2 * qt_al);
    unsigned *arrived = (unsigned *)(sc + 2 * qt_al + y_bytes(d));
    RaParams p;
    p.qt_hi = qt_hi;
    p.qt_lo = qt_lo;
    p.sel = sel;
    p.partials = (float *)(sc + 2 * qt_al + y_bytes(d) + arrived_bytes(d));
    p.status = status;
    p.L = d.ctx_len;
    p.n_sel = n_sel;
    p.C = d.chunk;
    p.rk = d.rank_k;
    p.rv = d.rank_v;
    p.Hq = d.n_q_heads;
    p.Hkv = d.n_kv_heads;
    p.B = d.batch;
    const int n_split = ra_splits(d, n_sel);
    p.chunks_per_item = (n_sel + n_split - 1) / n_split;
    p.n_split = (n_sel + p.chunks_per_item - 1) / p.chunks_per_item;
    p.n_items = d.batch * d.n_kv_heads * p.n_split;
    p.qscale = 1.4426950408889634f / sqrtf((float)d.head_dim);
    // XKV_TEST_MMA_SPIN (tests only, read on every call): a shorter poll limit for the MMA
    // issuer's waits on staged data, so a test can make them give up; every other wait,
    // and the drain that follows, keeps its full bound
    p.mma_spin = test_poll_limit("XKV_TEST_MMA_SPIN", RA_SPIN);
    DnParams dp;
    const DnParams *dpp = nullptr;
    if (!sel && attend_ra_dense_heads(d)) {
        const DnPlan pl = dense_plan(d);
        dp.qt_hi = qt_hi;
        dp.qt_lo = qt_lo;
        dp.partials = p.partials;
        dp.z = (float *)((char *)p.partials + al256((size_t)pl.n_span * bh * (d.rank_v + 2) *
                                                    sizeof(float)));
        dp.status = status;
        dp.L = d.ctx_len;
        dp.rk = d.rank_k;
        dp.rv = d.rank_v;
        dp.B = d.batch;
        dp.tiles = pl.tiles;
        dp.tps = pl.tps;
        dp.n_span = pl.n_span;
        dp.n_items = d.batch * pl.n_span;
        dp.qscale = p.qscale;
        dp.mma_spin = p.mma_spin;
        dpp = &dp;
        dp.rows_all = (int)((int64_t)d.batch * d.ctx_len);
    }
    switch (d.n_q_heads / d.n_kv_heads) {
#define XKV_RA_G(GG) \
    case GG: return launch_g<GG>(d, maps, p, dpp, q, Bkt, Bvt, qt_hi, qt_lo, yparts, arrived, out, s);
        XKV_RA_G(1) XKV_RA_G(2) XKV_RA_G(4) XKV_RA_G(5) XKV_RA_G(8)
#undef XKV_RA_G
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace xkv
