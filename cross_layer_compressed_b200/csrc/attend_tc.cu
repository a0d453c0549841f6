// Selective / dense reconstruction + GQA attention on the 5th-generation tensor cores.
//
// xKV page, section 2.3 (selective reconstruction) and section 4 (dense): for each
// (sequence b, KV head g) only the rows T of the selected chunks are rebuilt,
//   K_hat = A^K[T] B^K_l[:, g],  V_hat = A^V[T] B^V_l[:, g],
// and the G query heads of the group attend over them.  The two rebuilds are dense
// GEMMs (rank 512 / 768 deep) and run as tcgen05.mma (bf16 in, fp32 accumulate in
// tensor memory); K_hat and V_hat never leave the SM.
//
// Work item = (b, g, a run of <= 256 selected rows).  Persistent kernel: one CTA per SM
// walks the items.  The pipeline streams 64-wide rank slices: a stage holds the item's
// rows of A for that slice (256 x 128 B, 128-byte-swizzled 8-row atoms) and the 128 x 64
// slice of B_l's group-g columns.  Roles (warp-specialised):
//   warp 0        allocates the 512 TMEM columns; one thread issues the MMAs.
//                 Key phase:   D_K[tok][j]  (cols   0..255) += A^K[tok][k] . B^K[j][k]
//                              (M = 128 tokens per MMA, N = hd = 128)
//                 Value phase: D_V[j][tok]  (cols 256..511) += B^V[j][k] . A^V[tok][k]
//                              (M = hd = 128, N = tokens rounded up to 16)
//                 so keys come out one token per TMEM lane and values one head-dim per
//                 lane: neither epilogue needs a cross-thread reduction.
//   warps 1-8     TMA producers (warps 1-4 when G > 6).  Each 8-row group of the item's A
//                 rows is one 8 x 64 box (a selected chunk is 8 contiguous rows, so a
//                 group is one 128-byte swizzle atom); the groups are spread over the
//                 warps (four boxes each) because the cost of issuing the boxes, not
//                 bandwidth, bounds how fast one warp can feed a stage.  Warp 1 also loads
//                 the 16 KB B slice.
//   next 8 warps  epilogue in two groups of four (group 1 takes rows / tokens 128..255).
//                 Key epilogue: thread = token, logits z_h = q_h . K_hat (fp32); then the
//                 exact max / sum of the item's rows.  Value epilogue: thread = output
//                 column j, o_h[j] = sum_t p_h[t] V_hat[t][j]; the groups' halves are
//                 summed in shared memory.  Partials (m, l, o) go to the workspace and
//                 the combine kernel merges an item's splits.
// The key MMAs of item i+1 overlap the value epilogue of item i (separate TMEM columns);
// the producers run ahead across items, so the HBM stream does not stop between items.
//
// Every wait on an mbarrier is bounded; on expiry the CTA records XKV_ERR_TIMEOUT in the
// workspace status word, drains its own copies and MMAs (again bounded), frees TMEM and
// returns; the combine kernel then writes NaN outputs.
#include "sm100_util.cuh"

namespace xkv {
namespace {

constexpr int TC_STAGES = 4;
constexpr int TC_ROWS = 256;                 // rows per work item
constexpr int TC_KS = 64;                    // rank slice per stage: 128 bytes of bf16
constexpr int TC_HD = 128;
constexpr int A_TILE = TC_ROWS * TC_KS * 2;  // 32 KB: 32 row groups of 8 x 128 B
constexpr int B_TILE = TC_HD * TC_KS * 2;    // 16 KB
constexpr int STAGE_BYTES = A_TILE + B_TILE;
constexpr int W_MMA = 0, W_LOAD = 1, N_EPI = 8;
constexpr int EPI_THREADS = 32 * N_EPI;                // 256
// Producer warps: eight for groups of up to 6 query heads (544 threads, 96 registers
// each, no spills); the larger groups' epilogue needs the 128 registers a 416-thread CTA
// of four producer warps leaves it.
template <int G>
struct TcRoles {
    static constexpr int N_LOAD = G <= 6 ? 8 : 4;
    static constexpr int W_EPI = W_LOAD + N_LOAD;
    static constexpr int THREADS = 32 * (W_EPI + N_EPI);
};
constexpr uint32_t SPIN_LIMIT = 1u << 24;

struct TcShared {
    uint64_t full[TC_STAGES];     // one arrival + the stage's bytes
    uint64_t empty[TC_STAGES];    // MMA commit
    uint64_t kdone, vdone, kfree, vfree, idle;
    uint32_t tmem_base;
    int abort;
    float red[N_EPI][16];
};

struct TcParams {
    const __nv_bfloat16 *q;   // [B][Hq][hd]
    const int32_t *sel;       // [B][Hkv][n_sel] or null (dense)
    float *partials;          // [n_split][B][Hq][hd + 2]
    unsigned *status;         // workspace status word
    int64_t L;
    int n_sel;                // chunks per unit
    int C;
    int rk, rv;
    int Hq, Hkv, B;
    int chunks_per_item;
    int n_split;
    int n_items;
    float qscale;             // log2(e) / sqrt(hd)
    uint32_t mma_spin;        // poll limit of the MMA issuer's waits for staged data
};

// ----------------------------------------------------------------- PTX wrappers
// Bounded wait for the phase of parity `parity`; false on timeout or abort.
__device__ __forceinline__ bool mbar_wait(uint64_t *b, uint32_t parity, TcShared *sh,
                                          uint32_t limit = SPIN_LIMIT) {
    for (uint32_t i = 0; i < limit; ++i) {
        if (mbar_test(b, parity)) return true;
        if (*(volatile int *)&sh->abort) return false;
    }
    return false;
}
// Shared-memory descriptor of a K-major 128-byte-swizzled operand: 8-row groups 1 KB apart.
__device__ __forceinline__ uint64_t sdesc(uint32_t saddr) { return smem_desc_sw128(saddr, 16, 1024); }
// Named barrier 1: the epilogue threads.
__device__ __forceinline__ void epi_bar() {
    asm volatile("bar.sync 1, %0;" ::"n"(EPI_THREADS) : "memory");
}
// Epilogue barrier that also ORs `flag` over the epilogue threads, so that a decision
// taken after a bounded wait is the same in every epilogue thread.
__device__ __forceinline__ bool epi_bar_any(bool flag) {
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

struct Item {
    int b, g, split, c0, nch, nr;
};
// Items run split-major: the B * Hkv units of one row range are consecutive, so the KV
// heads that read the same rows of A (every row, in dense mode) run side by side and
// share them through L2 instead of each streaming the window from DRAM.
__device__ __forceinline__ Item decode(const TcParams &p, int item) {
    Item it;
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

__device__ void abort_cta(TcShared *sh, const TcParams &p) {
    *(volatile int *)&sh->abort = 1;
    if (p.status) atomicOr(p.status, 1u << XKV_ERR_TIMEOUT);
}

// One warp-uniform bounded wait: lane 0 polls, every lane gets the outcome.
__device__ __forceinline__ bool warp_wait(uint64_t *b, uint32_t parity, TcShared *sh,
                                          const TcParams &p, int lane) {
    int got = 0;
    if (lane == 0) {
        got = mbar_wait(b, parity, sh) ? 1 : 0;
        if (!got) abort_cta(sh, p);
    }
    return __shfl_sync(0xffffffffu, got, 0) != 0;
}

template <int G>
__global__ void __launch_bounds__(TcRoles<G>::THREADS, 1)
    k_xkv_tc(const __grid_constant__ CUtensorMap tmAk, const __grid_constant__ CUtensorMap tmAv,
             const __grid_constant__ CUtensorMap tmBk, const __grid_constant__ CUtensorMap tmBv,
             const TcParams p) {
    extern __shared__ unsigned char smem_raw[];
    unsigned char *smem = (unsigned char *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    TcShared *sh = reinterpret_cast<TcShared *>(smem + TC_STAGES * STAGE_BYTES);
    float *qs = reinterpret_cast<float *>(sh + 1);       // [hd][G]
    float *zs = qs + TC_HD * G;                          // [TC_ROWS][G]
    float *os = zs + TC_ROWS * G;                        // [G][hd]: group 1's value partials
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t nC = p.L / p.C;
    const int gpc = p.C / 8;                             // 8-row groups per chunk

    if (threadIdx.x == 0) {
        for (int s = 0; s < TC_STAGES; ++s) {
            mbar_init(&sh->full[s], 1);
            mbar_init(&sh->empty[s], 1);
        }
        mbar_init(&sh->kdone, 1);
        mbar_init(&sh->vdone, 1);
        mbar_init(&sh->kfree, 1);
        mbar_init(&sh->vfree, 1);
        mbar_init(&sh->idle, 1);
        sh->abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        prefetch_tmap(&tmAk);
        prefetch_tmap(&tmAv);
        prefetch_tmap(&tmBk);
        prefetch_tmap(&tmBv);
    }
    if (warp == W_MMA) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 512;" ::"r"(
                         su32(&sh->tmem_base))
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tcgen05_before();
    __syncthreads();
    tcgen05_after();
    const uint32_t tmem = sh->tmem_base;
    grid_dep_wait();    // selection, query and status come from the kernels before
    grid_dep_launch();

    constexpr int N_LOAD = TcRoles<G>::N_LOAD, W_EPI = TcRoles<G>::W_EPI;
    if (warp >= W_LOAD && warp < W_LOAD + N_LOAD) {
        // ------------------------------------------------------------ TMA producers
        const int pi = warp - W_LOAD;              // row groups pi, pi + 4, ... of an item
        const int gi = pi + N_LOAD * lane;
        // global row of this lane's 8-row group in an item (-1: none)
        auto group_row = [&](const Item &w) -> int64_t {
            if (gi >= w.nr / 8) return -1;
            const int ci = gi / gpc, sub = gi % gpc;
            int64_t c = w.c0 + ci;
            if (p.sel) c = p.sel[((int64_t)w.b * p.Hkv + w.g) * p.n_sel + c];
            if ((c < 0 || c >= nC) && p.status)             // the call fails: NaN outputs
                atomicOr(p.status, 1u << XKV_ERR_INVALID_ARG);
            c = min64(max64(c, 0), nC - 1);                 // and the copy stays in bounds
            return (int64_t)w.b * p.L + c * p.C + sub * 8;
        };
        int it = 0;
        bool ok = true;
        for (int item = blockIdx.x; item < p.n_items && ok; item += gridDim.x) {
            const Item w = decode(p, item);
            const int ng = w.nr / 8;
            const int64_t grow = group_row(w);
            const int row = grow < 0 ? 0 : (int)grow;
            const int brow = (w.b * p.Hkv + w.g) * TC_HD;
            for (int phase = 0; phase < 2 && ok; ++phase) {
                const int nks = (phase == 0 ? p.rk : p.rv) / TC_KS;
                const CUtensorMap *mA = phase == 0 ? &tmAk : &tmAv;
                const CUtensorMap *mB = phase == 0 ? &tmBk : &tmBv;
                for (int ks = 0; ks < nks; ++ks, ++it) {
                    const int s = it % TC_STAGES, n = it / TC_STAGES;
                    if (!warp_wait(&sh->empty[s], (n & 1) ^ 1, sh, p, lane)) {
                        ok = false;
                        break;
                    }
                    unsigned char *st = smem + s * STAGE_BYTES;
                    if (pi == 0 && lane == 0) {
                        // the stage's one arrival, with every byte the producer warps will load
                        mbar_expect_tx(&sh->full[s], (uint32_t)(ng * 1024 + B_TILE));
                        tma_load_2d(mB, &sh->full[s], st + A_TILE, ks * TC_KS, brow);
                    }
                    if (gi < ng) tma_load_2d(mA, &sh->full[s], st + gi * 1024, ks * TC_KS, row);
                    __syncwarp();
                }
            }
        }
        if (!ok && pi == 0 && lane == 0) {
            // Every stage the producer warps issued lands before the CTA may leave: the last
            // TC_STAGES fills (each issued whole: a warp checks for abort only in its wait
            // on `empty`, which completes for all of them alike) complete their phase.
            for (int j = it - TC_STAGES > 0 ? it - TC_STAGES : 0; j < it; ++j)
                for (uint32_t i = 0; i < SPIN_LIMIT; ++i)
                    if (mbar_test(&sh->full[j % TC_STAGES], (uint32_t)(j / TC_STAGES) & 1)) break;
        }
    } else if (warp == W_MMA) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint32_t smem_base = su32(smem);
            int it = 0, ic = 0;
            bool ok = true;
            for (int item = blockIdx.x; item < p.n_items && ok; item += gridDim.x, ++ic) {
                const Item w = decode(p, item);
                const int nr16 = (w.nr + 15) & ~15;
                const uint32_t idK = idesc_f16(128, TC_HD, false, false);
                const uint32_t idV = idesc_f16(128, nr16, false, false);
                // key phase into columns [0, 256)
                if (!mbar_wait(&sh->kfree, (ic & 1) ^ 1, sh)) { abort_cta(sh, p); ok = false; break; }
                tcgen05_after();
                const int nk = p.rk / TC_KS;
                for (int ks = 0; ks < nk && ok; ++ks, ++it) {
                    const int s = it % TC_STAGES, n = it / TC_STAGES;
                    if (!mbar_wait(&sh->full[s], n & 1, sh, p.mma_spin)) { abort_cta(sh, p); ok = false; break; }
                    tcgen05_after();
                    const uint32_t a0 = smem_base + s * STAGE_BYTES, b0 = a0 + A_TILE;
#pragma unroll
                    for (int kk = 0; kk < TC_KS / 16; ++kk) {
                        const uint32_t acc = (ks | kk) ? 1u : 0u;
                        umma_f16(tmem, sdesc(a0 + kk * 32), sdesc(b0 + kk * 32), idK, acc);
                        if (w.nr > 128)
                            umma_f16(tmem + 128, sdesc(a0 + 16384 + kk * 32), sdesc(b0 + kk * 32), idK,
                                 acc);
                    }
                    umma_arrive(&sh->empty[s]);
                }
                if (!ok) break;
                umma_arrive(&sh->kdone);
                // value phase into columns [256, 512)
                if (!mbar_wait(&sh->vfree, (ic & 1) ^ 1, sh)) { abort_cta(sh, p); ok = false; break; }
                tcgen05_after();
                const int nv = p.rv / TC_KS;
                for (int ks = 0; ks < nv && ok; ++ks, ++it) {
                    const int s = it % TC_STAGES, n = it / TC_STAGES;
                    if (!mbar_wait(&sh->full[s], n & 1, sh, p.mma_spin)) { abort_cta(sh, p); ok = false; break; }
                    tcgen05_after();
                    const uint32_t a0 = smem_base + s * STAGE_BYTES, b0 = a0 + A_TILE;
#pragma unroll
                    for (int kk = 0; kk < TC_KS / 16; ++kk)
                        umma_f16(tmem + 256, sdesc(b0 + kk * 32), sdesc(a0 + kk * 32), idV,
                             (ks | kk) ? 1u : 0u);
                    umma_arrive(&sh->empty[s]);
                }
                if (!ok) break;
                umma_arrive(&sh->vdone);
            }
            // all MMAs issued by this thread have completed once `idle` fires
            umma_arrive(&sh->idle);
            for (uint32_t i = 0; i < SPIN_LIMIT; ++i)
                if (mbar_test(&sh->idle, 0)) break;
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ epilogue
        const int et = threadIdx.x - 32 * W_EPI;  // 0..255
        const int ew = warp - W_EPI;              // 0..7 (each group of four covers the
                                                  // four TMEM lane quadrants, warp & 3)
        const int grp = ew >> 2;                  // rows / tokens [128 grp, 128 grp + 128)
        const int quad = warp & 3;                // TMEM lane quadrant of this warp
        const uint32_t lane_base = (uint32_t)(quad * 32) << 16;
        int ic = 0;
        for (int item = blockIdx.x; item < p.n_items; item += gridDim.x, ++ic) {
            const Item w = decode(p, item);
            epi_bar();
            const __nv_bfloat16 *qg = p.q + ((size_t)w.b * p.Hq + (size_t)w.g * G) * TC_HD;
            for (int e = et; e < G * TC_HD; e += EPI_THREADS) {
                const int h = e / TC_HD, j = e % TC_HD;
                qs[j * G + h] = __bfloat162float(qg[e]) * p.qscale;
            }
            {
                const bool fail = !mbar_wait(&sh->kdone, ic & 1, sh);
                if (fail) abort_cta(sh, p);
                if (epi_bar_any(fail)) break;     // also publishes qs
            }
            tcgen05_after();
            // key epilogue: thread = token grp*128 + quad*32 + lane
            if (grp * 128 < w.nr) {
                float acc[G];
#pragma unroll
                for (int h = 0; h < G; ++h) acc[h] = 0.f;
#pragma unroll 1
                for (int c0 = 0; c0 < TC_HD; c0 += 32) {
                    float v[32];
                    tmem_load32(tmem + lane_base + grp * 128 + c0, v);
#pragma unroll
                    for (int c = 0; c < 32; ++c) {
                        const float *qd = qs + (c0 + c) * G;
#pragma unroll
                        for (int h = 0; h < G; ++h) acc[h] = fmaf(v[c], qd[h], acc[h]);
                    }
                }
                const int t = grp * 128 + quad * 32 + lane;
                if (t < w.nr) {
#pragma unroll
                    for (int h = 0; h < G; ++h) zs[t * G + h] = acc[h];
                }
            }
            tcgen05_before();
            epi_bar();
            if (et == 0) mbar_arrive(&sh->kfree);
            // exact softmax statistics of the item's rows (log2 domain)
            float m[G], l[G];
#pragma unroll
            for (int h = 0; h < G; ++h) m[h] = -INFINITY;
            for (int t = et; t < w.nr; t += EPI_THREADS)
#pragma unroll
                for (int h = 0; h < G; ++h) m[h] = fmaxf(m[h], zs[t * G + h]);
#pragma unroll
            for (int h = 0; h < G; ++h) {
#pragma unroll
                for (int off = 16; off; off >>= 1)
                    m[h] = fmaxf(m[h], __shfl_xor_sync(0xffffffffu, m[h], off));
                if (lane == 0) sh->red[ew][h] = m[h];
            }
            epi_bar();
#pragma unroll
            for (int h = 0; h < G; ++h) {
                float mm = sh->red[0][h];
#pragma unroll
                for (int k = 1; k < N_EPI; ++k) mm = fmaxf(mm, sh->red[k][h]);
                m[h] = mm;
            }
            epi_bar();
#pragma unroll
            for (int h = 0; h < G; ++h) l[h] = 0.f;
            for (int t = et; t < w.nr; t += EPI_THREADS)
#pragma unroll
                for (int h = 0; h < G; ++h) {
                    const float pv = exp2f(zs[t * G + h] - m[h]);
                    zs[t * G + h] = pv;
                    l[h] += pv;
                }
#pragma unroll
            for (int h = 0; h < G; ++h) {
#pragma unroll
                for (int off = 16; off; off >>= 1) l[h] += __shfl_xor_sync(0xffffffffu, l[h], off);
                if (lane == 0) sh->red[ew][h] = l[h];
            }
            {
                const bool fail = !mbar_wait(&sh->vdone, ic & 1, sh);
                if (fail) abort_cta(sh, p);
                if (epi_bar_any(fail)) break;     // also publishes p (zs) and red
            }
#pragma unroll
            for (int h = 0; h < G; ++h) {
                float ll = 0.f;
#pragma unroll
                for (int k = 0; k < N_EPI; ++k) ll += sh->red[k][h];
                l[h] = ll;
            }
            tcgen05_after();
            // value epilogue: thread = output column j; tokens [128 grp, 128 grp + 128)
            float o[G];
#pragma unroll
            for (int h = 0; h < G; ++h) o[h] = 0.f;
            const int tend = min(w.nr, grp * 128 + 128);
#pragma unroll 1
            for (int c0 = grp * 128; c0 < tend; c0 += 32) {
                float v[32];
                tmem_load32(tmem + lane_base + 256 + c0, v);
                const int nc = tend - c0;      // >= 1; columns past it are not attended
#pragma unroll
                for (int c = 0; c < 32; ++c) {
                    if (c < nc) {
                        const float *pz = zs + (c0 + c) * G;
#pragma unroll
                        for (int h = 0; h < G; ++h) o[h] = fmaf(pz[h], v[c], o[h]);
                    }
                }
            }
            tcgen05_before();
            const int j = quad * 32 + lane;
            if (grp == 1) {
#pragma unroll
                for (int h = 0; h < G; ++h) os[h * TC_HD + j] = o[h];
            }
            epi_bar();
            if (et == 0) mbar_arrive(&sh->vfree);
            if (grp == 0) {
                float *dst = p.partials + (((size_t)w.split * p.B + w.b) * p.Hq + (size_t)w.g * G) *
                                              (TC_HD + 2);
                const bool two = w.nr > 128;
#pragma unroll
                for (int h = 0; h < G; ++h) {
                    dst[h * (TC_HD + 2) + 2 + j] = two ? o[h] + os[h * TC_HD + j] : o[h];
                    if (et == 0) {
                        dst[h * (TC_HD + 2)] = m[h] * 0.6931471805599453f;  // natural log
                        dst[h * (TC_HD + 2) + 1] = l[h];
                    }
                }
            }
        }
    }
    tcgen05_before();
    __syncthreads();
    tcgen05_after();
    if (warp == W_MMA)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 512;" ::"r"(tmem)
                     : "memory");
}

// ----------------------------------------------------------------- host side
template <int G>
cudaError_t launch_g(const CUtensorMap *maps, const TcParams &p, cudaStream_t s) {
    const size_t smem = 1024 + (size_t)TC_STAGES * STAGE_BYTES + sizeof(TcShared) +
                        sizeof(float) * ((size_t)TC_HD * G + (size_t)TC_ROWS * G +
                                         (size_t)G * TC_HD);
    auto k = k_xkv_tc<G>;
    cudaError_t e = set_smem_limit((const void *)k, smem);
    if (e != cudaSuccess) return e;
    const int grid = p.n_items < sm_count() ? p.n_items : sm_count();
    return launch_chained(k, dim3(grid), dim3(TcRoles<G>::THREADS), smem, s, maps[0], maps[1], maps[2],
                          maps[3], p);
}

}  // namespace

bool attend_tc_shape_ok(const xkv_dims &d) {
    return d.dtype == XKV_BF16 && d.head_dim == TC_HD && d.rank_k % TC_KS == 0 &&
           d.rank_v % TC_KS == 0 && TC_ROWS % d.chunk == 0;
}

bool attend_tc_supported(const xkv_dims &d) {
    return attend_tc_shape_ok(d) && tma_available();
}

int tc_splits(const xkv_dims &d, int n_sel) {
    const int64_t rows = (int64_t)n_sel * d.chunk;
    return (int)((rows + TC_ROWS - 1) / TC_ROWS);
}

cudaError_t launch_attend_tc(const xkv_dims &d, const void *Ak, const void *Av, const void *Bkt,
                             const void *Bvt, const void *q, const int32_t *sel, int n_sel,
                             float *partials, unsigned *status, int *n_split_out,
                             cudaStream_t s) {
    const int64_t d_kv = (int64_t)d.n_kv_heads * d.head_dim;
    CUtensorMap maps[4];
    if (!make_map_bf16_sw128(&maps[0], Ak, (uint64_t)d.batch * d.ctx_len, d.rank_k, 8) ||
        !make_map_bf16_sw128(&maps[1], Av, (uint64_t)d.batch * d.ctx_len, d.rank_v, 8) ||
        !make_map_bf16_sw128(&maps[2], Bkt, (uint64_t)d.batch * d_kv, d.rank_k, TC_HD) ||
        !make_map_bf16_sw128(&maps[3], Bvt, (uint64_t)d.batch * d_kv, d.rank_v, TC_HD))
        return cudaErrorInvalidValue;
    TcParams p;
    p.q = (const __nv_bfloat16 *)q;
    p.sel = sel;
    p.partials = partials;
    p.status = status;
    p.L = d.ctx_len;
    p.n_sel = n_sel;
    p.C = d.chunk;
    p.rk = d.rank_k;
    p.rv = d.rank_v;
    p.Hq = d.n_q_heads;
    p.Hkv = d.n_kv_heads;
    p.B = d.batch;
    const int n_split = tc_splits(d, n_sel);
    p.chunks_per_item = (n_sel + n_split - 1) / n_split;
    p.n_split = (n_sel + p.chunks_per_item - 1) / p.chunks_per_item;
    p.n_items = d.batch * d.n_kv_heads * p.n_split;
    p.qscale = 1.4426950408889634f / sqrtf((float)d.head_dim);
    // XKV_TEST_MMA_SPIN (tests only, read on every call): a shorter poll limit for the MMA
    // issuer's waits on staged data, so a test can make them give up; every other wait,
    // and the drain that follows, keeps its full bound
    p.mma_spin = test_poll_limit("XKV_TEST_MMA_SPIN", SPIN_LIMIT);
    *n_split_out = p.n_split;
    switch (d.n_q_heads / d.n_kv_heads) {
#define XKV_G(GG) \
    case GG: return launch_g<GG>(maps, p, s);
        XKV_G(1) XKV_G(2) XKV_G(3) XKV_G(4) XKV_G(5) XKV_G(6) XKV_G(7) XKV_G(8)
        XKV_G(9) XKV_G(10) XKV_G(11) XKV_G(12) XKV_G(13) XKV_G(14) XKV_G(15) XKV_G(16)
#undef XKV_G
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace xkv
