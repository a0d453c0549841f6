// R-CLA decode attention over a leader's cache on the 5th-generation tensor cores.
//
// Stochastic KV Routing page, inference paragraph: a layer attends over the K/V cache of
// its nearest previous leader; a leader first appends this step's row.  Per (sequence b,
// KV head g) the G query heads of the group attend over the leader's rows [0, n_rows):
//   z_h[t] = q_h . K[t] / sqrt(hd),  p_h = softmax_t(z_h),  o_h = sum_t p_h[t] V[t].
// Both contractions run as tcgen05.mma (bf16 in, fp32 accumulate in tensor memory):
//   logits   D_z[t][n] = K[t][:] . Q[n][:]       (M = 128 rows, N = 8: Q = the G heads)
//   output   D_o[j][n] = sum_t V[t][j] P[n][t]    (M = hd = 128, N = 8 or 16)
// V is read straight from its TMA tile as an MN-major operand; P holds each head's
// probabilities twice, as the bf16 nearest to p and the bf16 nearest to the rest
// (p - hi), so the product keeps ~16 bits of p; the epilogue adds the two columns.
//
// Work item = (b, g, a split of <= 1024 rows).  Persistent kernel, one CTA per SM:
//   warp 0      allocates TMEM; one thread issues the MMAs.  The whole warp patches a
//               tile that holds the appended row (copied from the input, never read
//               back from the cache another CTA is writing) or rows past the end of
//               the split (zeroed, so that stale cache bytes never meet a zero weight).
//   warp 1      TMA producer: an item's key tiles, then its value tiles (128 rows x
//               256 B = two 128-byte-swizzled boxes), through a ring of stages.
//   warps 2-5   epilogue: thread = row of a tile (logits) or output column j.  Exact
//               max / sum of the item's logits, P into shared memory, partials (m, l, o)
//               to the workspace; the combine kernel merges an item's splits.
// Every mbarrier wait is bounded; on expiry the CTA poisons the partials it still owes
// (NaN running max, so the combine writes NaN outputs), drains its own copies and MMAs
// (bounded), frees TMEM and returns.
#include "sm100_util.cuh"

namespace xkv {
namespace {

constexpr int RT_ROWS = 128;                   // rows per tile = MMA M
constexpr int RT_HALF = RT_ROWS * 128;         // one 64-column box: 16 KB
constexpr int RT_TILE = 2 * RT_HALF;           // 32 KB
constexpr int RT_MAX_TILES = 8;                // rows per item <= 1024
constexpr int RT_HD = 128;
constexpr int RT_NZ = 8;                       // logit columns (G <= 8)
constexpr uint32_t TM_Z = 0;                   // TMEM columns [0, 64): logits of 8 tiles
constexpr uint32_t TM_O = 128;                 // TMEM columns [128, 144): output
constexpr int W_MMA = 0, W_LOAD = 1, W_EPI = 2, N_EPI = 4;
constexpr int RT_THREADS = 32 * (W_EPI + N_EPI);  // 192
constexpr int EPI_THREADS = 32 * N_EPI;           // 128
constexpr uint32_t RT_SPIN = 1u << 24;

template <int G> struct RtCfg {
    static constexpr int NO = (2 * G + 7) / 8 * 8;                 // P rows: hi and lo
    static constexpr int STAGES = NO == 8 ? 6 : 5;
    static constexpr int PBUF = RT_MAX_TILES * RT_ROWS / 64 * (NO / 8) * 1024;
    static constexpr int QBUF = 2 * 1024;                           // 8 rows x 128
};

struct RtShared {
    uint64_t full[6], empty[6];
    uint64_t q_full, z_full, p_full, o_full, idle;
    uint32_t tmem_base;
    int abort;
    float red[N_EPI][8];
};

struct RtParams {
    __nv_bfloat16 *K, *V;                      // caches (the appended row is written here)
    const __nv_bfloat16 *k_new, *v_new, *q;
    float *partials;                           // [n_split][B][Hq][hd + 2]
    int slot, B, Hq, Hkv;
    int64_t L_max, n_rows, update_row;
    int rows_per_split, n_split, n_items;
    float qscale;                              // log2(e) / sqrt(hd)
    uint32_t mma_spin;                         // poll limit of the MMA warp's waits for staged data
};

struct RtItem {
    int b, g, split, nr, tiles;
    int64_t r0, row_base;                      // first row: in the unit, in the tensor map
};
__device__ __forceinline__ RtItem rt_decode(const RtParams &p, int item) {
    RtItem w;
    const int u = item / p.n_split;
    w.split = item % p.n_split;
    w.b = u / p.Hkv;
    w.g = u % p.Hkv;
    w.r0 = (int64_t)w.split * p.rows_per_split;
    w.nr = (int)min64(p.rows_per_split, p.n_rows - w.r0);
    w.tiles = (w.nr + RT_ROWS - 1) / RT_ROWS;
    w.row_base = (((int64_t)p.slot * p.B + w.b) * p.Hkv + w.g) * p.L_max + w.r0;
    return w;
}

// byte offset of element (n, k) in a K-major 128-byte-swizzled operand whose 8-row
// groups are 1024 B apart and whose 64-wide K atoms are `atom` bytes apart
__device__ __forceinline__ uint32_t kmaj_off(int n, int k, int atom) {
    const int kin = k & 63;
    return (uint32_t)((k >> 6) * atom + (n >> 3) * 1024 + (n & 7) * 128 +
                      ((((kin >> 3) ^ (n & 7)) & 7) << 4) + (kin & 7) * 2);
}

__device__ __forceinline__ void rt_epi_bar() {
    asm volatile("bar.sync 1, %0;" ::"n"(EPI_THREADS) : "memory");
}
__device__ __forceinline__ bool rt_epi_bar_any(bool flag) {
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
__device__ __forceinline__ bool rt_wait(uint64_t *b, uint32_t parity, RtShared *sh,
                                        uint32_t limit = RT_SPIN) {
    const bool ok = mbar_wait_bounded(b, parity, &sh->abort, limit);
    if (!ok) *(volatile int *)&sh->abort = 1;
    return ok;
}
// warp-uniform bounded wait: lane 0 polls
__device__ __forceinline__ bool rt_warp_wait(uint64_t *b, uint32_t parity, RtShared *sh,
                                             int lane, uint32_t limit = RT_SPIN) {
    int got = 0;
    if (lane == 0) got = rt_wait(b, parity, sh, limit) ? 1 : 0;
    return __shfl_sync(0xffffffffu, got, 0) != 0;
}

// Patch a staged tile (warp-collective): row `new_r` (or -1) becomes `src` (128 bf16),
// rows [z0, z1) become zero.  Rows are 128-byte-swizzled in two 64-column halves.
__device__ __forceinline__ void patch_tile(unsigned char *st, int new_r, const __nv_bfloat16 *src,
                                           int z0, int z1, int lane) {
    const int half = (lane >> 3) & 1, c16 = lane & 7;
    if (new_r >= 0 && lane < 16) {
        const uint4 v = reinterpret_cast<const uint4 *>(src)[half * 8 + c16];
        *reinterpret_cast<uint4 *>(st + half * RT_HALF + new_r * 128 + ((c16 ^ (new_r & 7)) << 4)) = v;
    }
    for (int r = z0 + (lane >> 4); r < z1; r += 2)
        *reinterpret_cast<uint4 *>(st + half * RT_HALF + r * 128 + ((c16 ^ (r & 7)) << 4)) =
            make_uint4(0u, 0u, 0u, 0u);
    fence_async_smem();
    __syncwarp();
}

template <int G>
__global__ void __launch_bounds__(RT_THREADS, 1)
    k_rcla_tc(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
              const RtParams p) {
    using Cfg = RtCfg<G>;
    constexpr int S = Cfg::STAGES, NO = Cfg::NO;
    constexpr int PATOM = (NO / 8) * 1024;     // bytes per 64-row K atom of P
    extern __shared__ unsigned char smem_raw[];
    unsigned char *smem = (unsigned char *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    unsigned char *pbuf = smem + S * RT_TILE;
    unsigned char *qbuf = pbuf + Cfg::PBUF;
    RtShared *sh = reinterpret_cast<RtShared *>(qbuf + Cfg::QBUF);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
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
        prefetch_tmap(&tmK);
        prefetch_tmap(&tmV);
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
    grid_dep_launch();  // the split merge after this kernel may be scheduled

    if (warp == W_LOAD) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            int it = 0;
            bool ok = true;
            // ring order K(0), K(1), V(0), K(2), V(1), ...: the next item's logits are
            // computed while the epilogue turns this item's logits into probabilities
            for (int step = 0; ok; ++step) {
                const int kitem = blockIdx.x + step * gridDim.x;
                const int vitem = kitem - gridDim.x;
                if (vitem >= p.n_items) break;
                for (int ph = 0; ph < 2 && ok; ++ph) {
                    const int item = ph == 0 ? kitem : vitem;
                    if (item < (int)blockIdx.x || item >= p.n_items) continue;
                    const RtItem w = rt_decode(p, item);
                    const CUtensorMap *m = ph == 0 ? &tmK : &tmV;
                    for (int t = 0; t < w.tiles; ++t, ++it) {
                        const int s = it % S, n = it / S;
                        if (!rt_wait(&sh->empty[s], (n & 1) ^ 1, sh)) { ok = false; break; }
                        unsigned char *st = smem + s * RT_TILE;
                        const int row = (int)(w.row_base + (int64_t)t * RT_ROWS);
                        mbar_expect_tx(&sh->full[s], (uint32_t)RT_TILE);
                        tma_load_2d(m, &sh->full[s], st, 0, row);
                        tma_load_2d(m, &sh->full[s], st + RT_HALF, 64, row);
                    }
                }
            }
            if (!ok) {
                // let this CTA's copies land: the last S fills issued complete their phase
                for (int j = it - S > 0 ? it - S : 0; j < it; ++j)
                    for (uint32_t i = 0; i < RT_SPIN; ++i)
                        if (mbar_test(&sh->full[j % S], (uint32_t)(j / S) & 1)) break;
            }
        }
        __syncwarp();
    } else if (warp == W_MMA) {
        // ------------------------------------------------------------ MMA issuer
        const uint32_t sbase = su32(smem), pb = su32(pbuf), qb = su32(qbuf);
        constexpr uint32_t idZ = idesc_f16(128, RT_NZ, false, false);
        constexpr uint32_t idO = idesc_f16(128, NO, true, false);    // A = V^T, MN-major
        int it = 0;
        bool ok = true;
        for (int step = 0; ok; ++step) {
            const int kitem = blockIdx.x + step * gridDim.x;
            const int vitem = kitem - gridDim.x;
            if (vitem >= p.n_items) break;
            if (kitem < p.n_items) {
                // logits of item kitem (its ordinal among this CTA's items is `step`)
                const RtItem w = rt_decode(p, kitem);
                const int64_t new_local = p.update_row >= 0 ? p.update_row - w.r0 : -1;
                const size_t new_off = ((size_t)w.b * p.Hkv + w.g) * RT_HD;
                if (!rt_warp_wait(&sh->q_full, step & 1, sh, lane)) { ok = false; break; }
                tcgen05_after();
                for (int t = 0; t < w.tiles && ok; ++t, ++it) {
                    const int s = it % S, n = it / S;
                    if (!rt_warp_wait(&sh->full[s], n & 1, sh, lane, p.mma_spin)) { ok = false; break; }
                    tcgen05_after();
                    const int64_t nl = new_local - (int64_t)t * RT_ROWS;
                    if (nl >= 0 && nl < RT_ROWS)
                        patch_tile(smem + s * RT_TILE, (int)nl, p.k_new + new_off, 0, 0, lane);
                    if (lane == 0) {
                        const uint32_t a0 = sbase + s * RT_TILE;
#pragma unroll
                        for (int kk = 0; kk < RT_HD / 16; ++kk)
                            umma_f16(tmem + TM_Z + t * RT_NZ,
                                     smem_desc_sw128(a0 + (kk >> 2) * RT_HALF + (kk & 3) * 32, 16, 1024),
                                     smem_desc_sw128(qb + (kk >> 2) * 1024 + (kk & 3) * 32, 16, 1024),
                                     idZ, kk ? 1u : 0u);
                        umma_arrive(&sh->empty[s]);
                    }
                    __syncwarp();
                }
                if (!ok) break;
                if (lane == 0) umma_arrive(&sh->z_full);
            }
            if (vitem >= (int)blockIdx.x) {
                // output of item vitem (ordinal step - 1)
                const RtItem w = rt_decode(p, vitem);
                const int64_t new_local = p.update_row >= 0 ? p.update_row - w.r0 : -1;
                const size_t new_off = ((size_t)w.b * p.Hkv + w.g) * RT_HD;
                if (!rt_warp_wait(&sh->p_full, (step - 1) & 1, sh, lane)) { ok = false; break; }
                tcgen05_after();
                for (int t = 0; t < w.tiles && ok; ++t, ++it) {
                    const int s = it % S, n = it / S;
                    if (!rt_warp_wait(&sh->full[s], n & 1, sh, lane, p.mma_spin)) { ok = false; break; }
                    tcgen05_after();
                    const int rows = min(RT_ROWS, w.nr - t * RT_ROWS);
                    const int nks = (rows + 15) / 16;
                    const int64_t nl = new_local - (int64_t)t * RT_ROWS;
                    const bool has_new = nl >= 0 && nl < RT_ROWS;
                    if (has_new || rows < nks * 16)
                        patch_tile(smem + s * RT_TILE, has_new ? (int)nl : -1, p.v_new + new_off,
                                   rows, nks * 16, lane);
                    if (lane == 0) {
                        const uint32_t a0 = sbase + s * RT_TILE;
                        for (int kk = 0; kk < nks; ++kk) {
                            const int k0 = t * RT_ROWS + kk * 16;
                            umma_f16(tmem + TM_O,
                                     smem_desc_sw128(a0 + kk * 2048, RT_HALF, 1024),
                                     smem_desc_sw128(pb + (k0 >> 6) * PATOM + ((k0 & 63) >> 4) * 32,
                                                     16, 1024),
                                     idO, (t | kk) ? 1u : 0u);
                        }
                        umma_arrive(&sh->empty[s]);
                    }
                    __syncwarp();
                }
                if (!ok) break;
                if (lane == 0) umma_arrive(&sh->o_full);
            }
        }
        if (lane == 0) {                            // every MMA issued here has completed
            umma_arrive(&sh->idle);
            for (uint32_t i = 0; i < RT_SPIN; ++i)
                if (mbar_test(&sh->idle, 0)) break;
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ epilogue
        const int et = threadIdx.x - 32 * W_EPI;    // 0..127
        const int ew = warp - W_EPI;
        const int quad = warp & 3;                  // TMEM lane quadrant of this warp
        const int row = quad * 32 + lane;           // tile row (logits) / column j (output)
        const uint32_t lane_base = (uint32_t)(quad * 32) << 16;
        // P rows >= 2G and Q rows >= G stay zero
        for (int i = et; i < (Cfg::PBUF + Cfg::QBUF) / 16; i += EPI_THREADS)
            reinterpret_cast<uint4 *>(pbuf)[i] = make_uint4(0u, 0u, 0u, 0u);
        auto write_q = [&](int item) {
            const RtItem w = rt_decode(p, item);
            const __nv_bfloat16 *qg = p.q + ((size_t)w.b * p.Hq + (size_t)w.g * G) * RT_HD;
            for (int e = et; e < G * 16; e += EPI_THREADS) {
                const int n = e >> 4, c16 = e & 15;
                const uint4 v = reinterpret_cast<const uint4 *>(qg + (size_t)n * RT_HD)[c16];
                *reinterpret_cast<uint4 *>(qbuf + (c16 >> 3) * 1024 + n * 128 +
                                           (((c16 & 7) ^ n) << 4)) = v;
            }
        };
        rt_epi_bar();
        if (blockIdx.x < p.n_items) write_q(blockIdx.x);
        fence_async_smem();
        rt_epi_bar();
        if (et == 0) mbar_arrive(&sh->q_full);
        int ic = 0, item = blockIdx.x;
        bool ok = true;
        for (; item < p.n_items; item += gridDim.x, ++ic) {
            const RtItem w = rt_decode(p, item);
            if (p.update_row >= 0 && w.split == 0) {   // the leader's append
                const size_t dst = ((((size_t)p.slot * p.B + w.b) * p.Hkv + w.g) * p.L_max +
                                    (size_t)p.update_row) * RT_HD;
                const size_t src = ((size_t)w.b * p.Hkv + w.g) * RT_HD;
                p.K[dst + et] = p.k_new[src + et];
                p.V[dst + et] = p.v_new[src + et];
            }
            {
                const bool fail = !rt_wait(&sh->z_full, ic & 1, sh);
                if (rt_epi_bar_any(fail)) { ok = false; break; }
            }
            tcgen05_after();
            float z[RT_MAX_TILES][G];
#pragma unroll
            for (int t = 0; t < RT_MAX_TILES; ++t) {
                if (t < w.tiles) {
                    float v[8];
                    tmem_load8(tmem + lane_base + TM_Z + t * RT_NZ, v);
                    const bool valid = t * RT_ROWS + row < w.nr;
#pragma unroll
                    for (int h = 0; h < G; ++h) z[t][h] = valid ? v[h] * p.qscale : -INFINITY;
                } else {
#pragma unroll
                    for (int h = 0; h < G; ++h) z[t][h] = -INFINITY;
                }
            }
            // the logits are read: Q takes the next item's heads and the next item's logit
            // MMAs may overwrite D_z while this item's softmax runs
            const bool has_next = item + (int)gridDim.x < p.n_items;
            if (has_next) write_q(item + gridDim.x);
            fence_async_smem();
            tcgen05_before();
            float m[G], l[G];
#pragma unroll
            for (int h = 0; h < G; ++h) {
                m[h] = z[0][h];
#pragma unroll
                for (int t = 1; t < RT_MAX_TILES; ++t) m[h] = fmaxf(m[h], z[t][h]);
#pragma unroll
                for (int off = 16; off; off >>= 1)
                    m[h] = fmaxf(m[h], __shfl_xor_sync(0xffffffffu, m[h], off));
                if (lane == 0) sh->red[ew][h] = m[h];
            }
            rt_epi_bar();
            if (et == 0 && has_next) mbar_arrive(&sh->q_full);
#pragma unroll
            for (int h = 0; h < G; ++h) {
                m[h] = fmaxf(fmaxf(sh->red[0][h], sh->red[1][h]),
                             fmaxf(sh->red[2][h], sh->red[3][h]));
                l[h] = 0.f;
            }
            rt_epi_bar();                           // red is reused for the sums
#pragma unroll
            for (int t = 0; t < RT_MAX_TILES; ++t) {
                if (t < w.tiles) {
                    const int k = t * RT_ROWS + row;
#pragma unroll
                    for (int h = 0; h < G; ++h) {
                        const float pv = exp2f(z[t][h] - m[h]);
                        l[h] += pv;
                        const __nv_bfloat16 hi = __float2bfloat16_rn(pv);
                        const __nv_bfloat16 lo = __float2bfloat16_rn(pv - __bfloat162float(hi));
                        *reinterpret_cast<__nv_bfloat16 *>(pbuf + kmaj_off(h, k, PATOM)) = hi;
                        *reinterpret_cast<__nv_bfloat16 *>(pbuf + kmaj_off(G + h, k, PATOM)) = lo;
                    }
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
            rt_epi_bar();
            if (et == 0) {
                mbar_arrive(&sh->p_full);
            }
#pragma unroll
            for (int h = 0; h < G; ++h)
                l[h] = (sh->red[0][h] + sh->red[1][h]) + (sh->red[2][h] + sh->red[3][h]);
            {
                const bool fail = !rt_wait(&sh->o_full, ic & 1, sh);
                if (rt_epi_bar_any(fail)) { ok = false; break; }
            }
            tcgen05_after();
            float o[G];
            if constexpr (NO == 8) {
                float v[8];
                tmem_load8(tmem + lane_base + TM_O, v);
#pragma unroll
                for (int h = 0; h < G; ++h) o[h] = v[h] + v[G + h];
            } else {
                float v[16];
                tmem_load16(tmem + lane_base + TM_O, v);
#pragma unroll
                for (int h = 0; h < G; ++h) o[h] = v[h] + v[G + h];
            }
            tcgen05_before();
            float *dst = p.partials + (((size_t)w.split * p.B + w.b) * p.Hq + (size_t)w.g * G) *
                                          (RT_HD + 2);
#pragma unroll
            for (int h = 0; h < G; ++h) {
                dst[h * (RT_HD + 2) + 2 + row] = o[h];
                if (et == 0) {
                    dst[h * (RT_HD + 2)] = m[h] * 0.6931471805599453f;   // natural log
                    dst[h * (RT_HD + 2) + 1] = l[h];
                }
            }
            rt_epi_bar();                           // red is rewritten by the next item
        }
        if (!ok) {
            // poison every item this CTA still owed: NaN running max -> NaN outputs
            for (int it2 = item; it2 < p.n_items; it2 += gridDim.x) {
                const RtItem w = rt_decode(p, it2);
                if (et < G)
                    p.partials[(((size_t)w.split * p.B + w.b) * p.Hq + (size_t)w.g * G + et) *
                               (RT_HD + 2)] = __int_as_float(0x7fc00000);
            }
        }
    }
    tcgen05_before();
    __syncthreads();
    tcgen05_after();
    if (warp == W_MMA)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 256;" ::"r"(tmem)
                     : "memory");
}

template <int G>
cudaError_t launch_g(const CUtensorMap *tm, const RtParams &p, cudaStream_t s) {
    using Cfg = RtCfg<G>;
    const size_t smem = 1024 + (size_t)Cfg::STAGES * RT_TILE + Cfg::PBUF + Cfg::QBUF +
                        sizeof(RtShared);
    auto k = k_rcla_tc<G>;
    cudaError_t e = set_smem_limit((const void *)k, smem);
    if (e != cudaSuccess) return e;
    const int grid = p.n_items < sm_count() ? p.n_items : sm_count();
    k<<<grid, RT_THREADS, smem, s>>>(tm[0], tm[1], p);
    return cudaGetLastError();
}

}  // namespace

bool rcla_tc_ok(const xkv_dims &d, int slot, int64_t L_max, const SplitPlan &plan) {
    const int G = d.n_q_heads / d.n_kv_heads;
    const int64_t rows = (int64_t)(slot + 1) * d.batch * d.n_kv_heads * L_max;
    return d.dtype == XKV_BF16 && d.head_dim == RT_HD &&
           (G == 1 || G == 2 || G == 4 || G == 5 || G == 8) &&
           plan.rows_per_split <= RT_MAX_TILES * RT_ROWS &&
           rows + RT_ROWS < ((int64_t)1 << 31) && tma_available() && !env_flag(ENV_FORCE_SIMT) &&
           !env_flag(ENV_NO_TC);
}

cudaError_t launch_rcla_tc(const xkv_dims &d, int slot, int64_t L_max, int64_t n_rows,
                           int64_t update_row, void *K, void *V, const void *k_new,
                           const void *v_new, const void *q, const SplitPlan &plan,
                           float *partials, cudaStream_t s) {
    const uint64_t rows = (uint64_t)(slot + 1) * d.batch * d.n_kv_heads * (uint64_t)L_max;
    CUtensorMap tm[2];
    if (!make_map_bf16_sw128(&tm[0], K, rows, RT_HD, RT_ROWS) ||
        !make_map_bf16_sw128(&tm[1], V, rows, RT_HD, RT_ROWS))
        return cudaErrorInvalidValue;
    RtParams p;
    p.K = (__nv_bfloat16 *)K;
    p.V = (__nv_bfloat16 *)V;
    p.k_new = (const __nv_bfloat16 *)k_new;
    p.v_new = (const __nv_bfloat16 *)v_new;
    p.q = (const __nv_bfloat16 *)q;
    p.partials = partials;
    p.slot = slot;
    p.B = d.batch;
    p.Hq = d.n_q_heads;
    p.Hkv = d.n_kv_heads;
    p.L_max = L_max;
    p.n_rows = n_rows;
    p.update_row = update_row;
    p.rows_per_split = (int)plan.rows_per_split;
    p.n_split = plan.n_split;
    p.n_items = d.batch * d.n_kv_heads * plan.n_split;
    p.qscale = 1.4426950408889634f / sqrtf((float)RT_HD);
    // XKV_TEST_MMA_SPIN (tests only, read on every call): a shorter poll limit for the MMA
    // warp's waits on staged data, so a test can make them give up; every other wait, and
    // the drain that follows, keeps its full bound
    p.mma_spin = test_poll_limit("XKV_TEST_MMA_SPIN", RT_SPIN);
    switch (d.n_q_heads / d.n_kv_heads) {
        case 1: return launch_g<1>(tm, p, s);
        case 2: return launch_g<2>(tm, p, s);
        case 4: return launch_g<4>(tm, p, s);
        case 5: return launch_g<5>(tm, p, s);
        case 8: return launch_g<8>(tm, p, s);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace xkv
