// Fused landmark scoring + chunk selection (xKV page, section 2.3: rank the chunks by the
// relevance of their landmark key to the current query, max over the GQA group, and keep
// the top-k plus the always-kept sink and recent chunks).
//
// The result is bit for bit the selection that xkv_select_chunks makes from the scores of
// xkv_score_landmarks (canonical fp64 sums of exact products in ascending d, ties to the
// lower chunk index), but the landmarks are scored in fp32 and only the chunks whose order
// the fp32 pass cannot certify are scored again in fp64:
//
//  1. every chunk c gets an fp32 score s~_c (per head an fp32 dot product: fmaf over each
//     lane's columns, then a butterfly sum over the row's lanes; max over the group)
//     with a certified bound |s~_c - s_c| <= E, where s_c is the canonical fp64 score:
//       E = (gamma_hd(2^-24) + gamma_hd(2^-53)) * max|lm| * max_h ||q_h||_1 + hd * 2^-150,
//     gamma_n(u) = n u / (1 - n u) (the classical bound of a dot product of n terms whose
//     every step rounds once, in any order of summation: each term passes through at most
//     n roundings; 2^-150 covers fp32 underflow; the fp64 term covers the rounding of the
//     canonical sum itself), inflated by 1 + 2^-20;
//  2. t = the k-th largest s~ among the candidates.  At least k candidates have s~ >= t,
//     so the k-th largest canonical score s_(k) >= t - E; at most k - 1 have s~ > t, so
//     s_(k) <= t + E.  A candidate with s~ > t + 2E therefore has s > s_(k): it is
//     selected whatever the ties; one with s~ < t - 2E has s < s_(k): it is not;
//  3. the rest (the band) is scored in fp64 exactly as the oracle scores it, and the
//     top (k - #selected) of the band under (score desc, index asc) complete the set.
//
// Work split, two launches chained with programmatic dependent launch:
//  * k_ss_keys streams every unit's landmark rows over the whole GPU.  A row is spread over
//    LPR lanes (16 bytes each: 16 lanes for a bf16 row of 128), so every warp load is
//    whole 128-byte lines, and each lane keeps its columns of the group's queries in
//    registers.  A row's G sums are reduced across its lanes by halving the set of heads
//    at each butterfly step (G - 1 + log2(LPR / G) shuffles instead of G log2 LPR); the
//    lane groups then exchange their heads' sums for the max.  Keys (32-bit, ordered like
//    the fp32 score) go to the workspace with, per CTA, the max |lm| and a non-finite flag.
//  * k_ss_select, one CTA of 512 threads per unit, reads the unit's keys into shared
//    memory and runs steps 2-3: an MSB-first radix descent for t (11, 11, 10 bits; a bin
//    of at most RANK_CAP keys is ranked directly), strided classification into certain /
//    band, the band rescored in fp64 and ranked by counting, the output placed by ballots
//    in ascending chunk order.
// Optionally a per-unit list of reserved chunks (the value-range reservation) joins the
// sink and recent chunks as forced.  Units whose fp32 scores are not all finite or whose
// band is wider than BAND_CAP chunks take the exact path for the whole unit: every chunk is
// scored in fp64 into the workspace and the full radix select runs on those keys.  The
// workspace also records, per unit, the band size (or ~0 for the exact path).
//
// Chosen for B200: 67 MB of landmarks per layer at the bench workload need ~10 us at the
// copy bandwidth, while the fp64 pass spent ~30 us on conversions and fp64 FMAs; fp32
// FMAs and shift-only bf16 widening keep the stream HBM-bound.  A first version kept one
// thread-block cluster per unit (keys gathered in CTA 0 over distributed shared memory);
// its per-thread row reads missed L1 on every 16-byte load and its 256-thread tail left
// most of the GPU idle, 58 us per layer against 44 us for the two-call path.
#include "sm100_util.cuh"
#include "xkv_internal.cuh"

namespace xkv {
namespace {

constexpr int SK_WARPS = 16;                      // key pass: consumer warps
constexpr int SK_THREADS = 32 * (SK_WARPS + 1);   // + one copy-issuing warp
constexpr int SK_STAGE = 32768;                   // bytes of landmark rows per stage
constexpr int SK_STAGES = 6;
constexpr int SK_MAX_CTAS = 1024;                 // key-pass CTAs (one per SM at most)
constexpr uint32_t SK_SPIN = 1u << 24;
constexpr int SL_THREADS = 512;                   // selection pass: one CTA per unit
constexpr int HIST_BINS = 2048;                   // radix digits of 11, 11 and 10 bits
constexpr int RANK_CAP = 32;                      // keys of a bin ranked directly
constexpr int BAND_CAP = 512;                     // band chunks rescored in fp64
constexpr int RES_THREADS = 256;                  // value-range reservation
constexpr uint32_t EXACT_PATH = 0xFFFFFFFFu;
constexpr uint32_t BAD_RESERVED = 0xFFFFFFFEu;   // a reserved list broke its rules

struct SsParams {
    const void *lm;       // [B][Hkv][nC][hd]
    const void *q;        // [B][Hq][hd]
    int32_t *sel;         // [B][Hkv][n_sel]
    uint32_t *band;       // [B][Hkv] band size per unit (EXACT_PATH for the exact path)
    double *scratch;      // [B][Hkv][nC] fp64 scores of units on the exact path
    uint32_t *keys;       // [B][Hkv][nC] fp32 keys
    float *cmx;           // [n_cta] max |lm| per key-pass CTA
    uint32_t *cbad;       // [n_cta] a non-finite fp32 score (or an abandoned wait) in the CTA
    int64_t nC;
    int n_cta;            // key-pass CTAs
    int stage_rows;       // landmark rows per stage
    int sps;              // stages per key-pass CTA (the last CTA may have fewer)
    int64_t n_stages;     // stages over all units' rows
    int64_t rows_total;   // landmark rows of all units
    uint32_t spin;        // poll limit of the key pass's pipeline waits
    int Hq, Hkv, hd;
    int top_k, n_sink, n_recent, n_sel;
    const int32_t *reserved;   // [B][Hkv][n_res] chunks forced in as well, or null
    int n_res;
    double err_rel;       // (gamma_hd(2^-24) + gamma_hd(2^-53)) (1 + 2^-20)
    double err_abs;       // hd 2^-150 (1 + 2^-20)
};

// --------------------------------------------------------------- keys and elements
// 32-bit key that orders like the float (-0 below +0), and its inverse.
__device__ __forceinline__ uint32_t fkey(float f) {
    const uint32_t u = __float_as_uint(f);
    return (u >> 31) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float fkey_inv(uint32_t k) {
    return __uint_as_float((k >> 31) ? (k & 0x7fffffffu) : ~k);
}

template <typename T> struct Vec;
template <> struct Vec<__nv_bfloat16> {
    static constexpr int N = 8;   // elements per 16-byte vector
    static __device__ __forceinline__ float get(const uint4 &w, int k) {
        const int j = k >> 1;   // the 32-bit word holding elements 2j (low) and 2j + 1 (high)
        const uint32_t u = j == 0 ? w.x : j == 1 ? w.y : j == 2 ? w.z : w.w;
        return (k & 1) ? bf16hi(u) : bf16lo(u);
    }
};
template <> struct Vec<float> {
    static constexpr int N = 4;
    static __device__ __forceinline__ float get(const uint4 &w, int k) {
        return __uint_as_float(k == 0 ? w.x : k == 1 ? w.y : k == 2 ? w.z : w.w);
    }
};

// The canonical score of one landmark row: per head the fp64 sum of exact products in
// ascending d, then the max over the group with -0 below +0.  The row is read in batches
// of eight 16-byte loads, all in flight before the arithmetic that consumes them (a row
// rescored by one thread would otherwise wait out a memory latency per 16 bytes).
template <typename T, int G>
__device__ double exact_score(const T *row, const float *qf, int hd) {
    constexpr int EPV = Vec<T>::N;
    constexpr int BATCH = 8;
    double acc[G];
#pragma unroll
    for (int h = 0; h < G; ++h) acc[h] = 0.0;
    const uint4 *v = reinterpret_cast<const uint4 *>(row);
    const int vpr = hd / EPV;
    for (int i0 = 0; i0 < vpr; i0 += BATCH) {
        uint4 w[BATCH];
#pragma unroll
        for (int j = 0; j < BATCH; ++j)
            w[j] = i0 + j < vpr ? __ldg(v + i0 + j) : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
        for (int j = 0; j < BATCH; ++j) {
            if (i0 + j >= vpr) break;
#pragma unroll
            for (int k = 0; k < EPV; ++k) {
                const double x = (double)Vec<T>::get(w[j], k);
                const float *qd = qf + ((i0 + j) * EPV + k) * G;
#pragma unroll
                for (int h = 0; h < G; ++h) acc[h] = fma(x, (double)qd[h], acc[h]);   // exact product
            }
        }
    }
    double best = acc[0];
#pragma unroll
    for (int h = 1; h < G; ++h)
        if (order_key(acc[h]) > order_key(best)) best = acc[h];
    return best;
}

// ------------------------------------------------------------------ block helpers
template <int NT>
struct RadixShared {
    unsigned hist[2][256];
    unsigned warp_tot[NT / 32];
    unsigned total;
    unsigned long long prefix, mask;
    unsigned krem;
    int done;
};

// Exclusive prefix sum over the CTA of one value per thread; *total gets the sum.
template <int NT>
__device__ unsigned block_scan(unsigned v, RadixShared<NT> &rs) {
    constexpr int NW = NT / 32;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    unsigned inc = v;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const unsigned t = __shfl_up_sync(0xffffffffu, inc, off);
        if (lane >= off) inc += t;
    }
    if (lane == 31) rs.warp_tot[warp] = inc;
    __syncthreads();
    if (warp == 0) {
        const unsigned t = lane < NW ? rs.warp_tot[lane] : 0u;
        unsigned ti = t;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const unsigned u = __shfl_up_sync(0xffffffffu, ti, off);
            if (lane >= off) ti += u;
        }
        if (lane < NW) rs.warp_tot[lane] = ti - t;
        if (lane == 31) rs.total = ti;
    }
    __syncthreads();
    const unsigned r = rs.warp_tot[warp] + inc - v;
    __syncthreads();   // warp_tot and total may be reused by the caller after reading total
    return r;
}

// Among the elements i < n with cand(i), take(i) is called for the `need` largest under
// (key(i) descending, i ascending), 1 <= need <= #candidates.  MSB-first radix select on
// 8-bit digits of the 64-bit keys (stopping once a whole bin is needed), then the ties
// of the last bin ranked by index with a prefix count over contiguous runs.
template <int NT, class KeyF, class CandF, class TakeF>
__device__ void radix_select(int n, unsigned need, KeyF key, CandF cand, TakeF take,
                             RadixShared<NT> &rs) {
    if (threadIdx.x == 0) {
        rs.prefix = 0ull;
        rs.mask = 0ull;
        rs.krem = need;
        rs.done = 0;
    }
    for (int i = threadIdx.x; i < 256; i += NT) rs.hist[0][i] = 0u;
    __syncthreads();
    unsigned long long mask = 0ull;
    int buf = 0;
    for (int shift = 56; shift >= 0; shift -= 8, buf ^= 1) {
        const unsigned long long prefix = rs.prefix;
        for (int i = threadIdx.x; i < n; i += NT) {
            if (!cand(i)) continue;
            const unsigned long long k = key(i);
            if ((k & mask) == prefix) atomicAdd(&rs.hist[buf][(unsigned)(k >> shift) & 255u], 1u);
        }
        __syncthreads();
        if (threadIdx.x >= 32) {
            for (int i = threadIdx.x - 32; i < 256; i += NT - 32) rs.hist[buf ^ 1][i] = 0u;
        } else {
            const int lane = threadIdx.x;
            const unsigned want = rs.krem;
            unsigned cnt[8], tot = 0;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                cnt[i] = rs.hist[buf][255 - (lane * 8 + i)];   // lanes walk the digits downwards
                tot += cnt[i];
            }
            unsigned inc = tot;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const unsigned t = __shfl_up_sync(0xffffffffu, inc, off);
                if (lane >= off) inc += t;
            }
            const unsigned exc = inc - tot;
            if (exc < want && want <= inc) {
                unsigned cum = exc;
                for (int i = 0; i < 8; ++i) {
                    if (cum + cnt[i] >= want) {
                        const unsigned long long D = (unsigned long long)(255 - (lane * 8 + i));
                        rs.prefix = prefix | (D << shift);
                        rs.mask = mask | (255ull << shift);
                        rs.krem = want - cum;
                        rs.done = cnt[i] == want - cum;
                        break;
                    }
                    cum += cnt[i];
                }
            }
        }
        mask |= 255ull << shift;
        __syncthreads();
        if (rs.done) break;
    }
    const unsigned long long T = rs.prefix, M = rs.mask;
    const unsigned krem = rs.krem;
    const bool whole = rs.done != 0;
    const int ipt = (n + NT - 1) / NT;
    const int lo = min(n, (int)threadIdx.x * ipt), hi = min(n, lo + ipt);
    unsigned eq_rank = 0;
    if (!whole) {
        unsigned eq = 0;
        for (int i = lo; i < hi; ++i) eq += (cand(i) && (key(i) & M) == T) ? 1u : 0u;
        eq_rank = block_scan(eq, rs);
    }
    for (int i = lo; i < hi; ++i) {
        if (!cand(i)) continue;
        const unsigned long long k = key(i) & M;
        if (k > T || (k == T && (whole || eq_rank++ < krem))) take(i);
    }
    __syncthreads();
}

// ------------------------------------------------------------------ key pass
// Step 1 for every chunk of every unit.  The units' landmark rows are one contiguous array;
// CTA c streams a contiguous run of it (sps stages of SK_STAGE bytes) through a ring of
// SK_STAGES shared-memory stages filled by untiled bulk copies, so each SM keeps up to
// 192 KB in flight with one issuing thread.  The 8 consumer warps split a stage's rows; a
// row is spread over LPR lanes (16 bytes each), so a warp reads RPI = 32 / LPR whole rows
// per conflict-free 16-byte shared load, and each lane keeps its columns of its row's
// queries in registers (reloaded when its row moves to the next unit).  A row's G sums
// are reduced across its lanes by halving the set of heads at each butterfly step; the
// lanes holding other heads then exchange their sums for the max.  Every wait is
// bounded: a CTA that gives up marks itself bad, which sends the units it covers to the
// exact path of the selection pass.
template <int G, int LPR>
struct KeyCfg {
    static constexpr int GP = G <= 1 ? 1 : G <= 2 ? 2 : G <= 4 ? 4 : G <= 8 ? 8 : 16;
    static constexpr int RPI = 32 / LPR;
    static constexpr int NV = GP > LPR ? GP / LPR : 1;        // head sums a lane ends with
};

template <typename T, int G, int LPR>
__global__ void __launch_bounds__(SK_THREADS, 1) k_ss_keys(const SsParams p) {
    using Cfg = KeyCfg<G, LPR>;
    constexpr int EPV = Vec<T>::N, GP = Cfg::GP, RPI = Cfg::RPI, NV = Cfg::NV;
    constexpr int ROW_BYTES = LPR * 16;
    constexpr int SROWS = SK_STAGE / ROW_BYTES;               // rows per stage
    constexpr int WROWS = SROWS / SK_WARPS;                   // rows per warp per stage
    constexpr int LOADS = WROWS / RPI;                        // shared loads per lane per stage
    static_assert(WROWS % RPI == 0, "whole rows per warp load");
    extern __shared__ __align__(128) unsigned char sk_smem[];
    __shared__ uint64_t full[SK_STAGES], empty[SK_STAGES];
    __shared__ float s_mx[SK_WARPS];
    __shared__ int s_bad[SK_WARPS];
    __shared__ int s_abort;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t nC = p.nC;
    const int64_t rows_total = p.rows_total;
    const int64_t st0 = (int64_t)blockIdx.x * p.sps;
    const int n_st = (int)min64((int64_t)p.sps, p.n_stages - st0);
    const unsigned char *lmb = reinterpret_cast<const unsigned char *>(p.lm);
    if (threadIdx.x == 0) {
        for (int s = 0; s < SK_STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], SK_WARPS);
        }
        s_abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();
    grid_dep_wait();    // the landmarks and the query may come from the kernels before
    if (warp == SK_WARPS) {
        // ------------------------------------------------------------ copies
        if (lane == 0) {
            int k = 0;
            for (; k < n_st; ++k) {
                const int slot = k % SK_STAGES, n = k / SK_STAGES;
                if (!mbar_wait_bounded(&empty[slot], (n & 1) ^ 1, &s_abort, p.spin)) {
                    *(volatile int *)&s_abort = 1;
                    break;
                }
                const int64_t r0 = (st0 + k) * SROWS;
                const uint32_t bytes = (uint32_t)(min64((int64_t)SROWS, rows_total - r0) * ROW_BYTES);
                mbar_expect_tx(&full[slot], bytes);
                bulk_load(sk_smem + slot * SK_STAGE, lmb + r0 * ROW_BYTES, bytes, &full[slot]);
            }
            // every copy issued lands before the CTA leaves (its slot's phase completes)
            for (int j = k - SK_STAGES > 0 ? k - SK_STAGES : 0; j < k; ++j)
                for (uint32_t i = 0; i < SK_SPIN; ++i)
                    if (mbar_test(&full[j % SK_STAGES], (uint32_t)(j / SK_STAGES) & 1)) break;
        }
    } else {
        // ------------------------------------------------------------ consumers
        const int piece = lane % LPR, sub = lane / LPR;
        float qr[EPV][G];   // this lane's columns of its row's G queries (exact in fp32)
        int64_t qunit = -1;
        float mx = 0.f;
        bool bad = false;
        auto load_q = [&](int64_t unit) {
            const int b = (int)(unit / p.Hkv), g = (int)(unit % p.Hkv);
            const T *qg = reinterpret_cast<const T *>(p.q) + ((size_t)b * p.Hq + (size_t)g * G) * p.hd;
#pragma unroll
            for (int kk = 0; kk < EPV; ++kk)
#pragma unroll
                for (int h = 0; h < G; ++h)
                    qr[kk][h] = Elem<T>::f32(qg[(size_t)h * p.hd + piece * EPV + kk]);
            qunit = unit;
        };
        // called with a constant per_row_unit: each call site inlines its own copy
        auto rows = [&](const uint4 (&w)[LOADS], int64_t r0, const bool per_row_unit) {
#pragma unroll
            for (int u = 0; u < LOADS; ++u) {
                const int64_t r = r0 + warp * WROWS + u * RPI + sub;   // row of all units
                const bool valid = r < rows_total;
                if (per_row_unit && valid && r / nC != qunit) load_q(r / nC);
                float a[GP];
#pragma unroll
                for (int h = 0; h < GP; ++h) a[h] = 0.f;
#pragma unroll
                for (int kk = 0; kk < EPV; ++kk) {
                    const float x = valid ? Vec<T>::get(w[u], kk) : 0.f;
                    mx = fmaxf(mx, fabsf(x));
#pragma unroll
                    for (int h = 0; h < G; ++h) a[h] = fmaf(x, qr[kk][h], a[h]);
                }
                // sum over the row's LPR lanes; while more than NV heads are held, each
                // step keeps half of them (the upper half on lanes whose bit `o` is set)
                int hb = 0;           // head of a[0]
                int width = GP;
#pragma unroll
                for (int o = LPR / 2; o >= 1; o >>= 1) {
                    if (width > NV) {
                        const int half = width / 2;
                        const bool up = (lane & o) != 0;
#pragma unroll
                        for (int i = 0; i < half; ++i) {
                            const float send = up ? a[i] : a[i + half];
                            const float keep = up ? a[i + half] : a[i];
                            a[i] = keep + __shfl_xor_sync(0xffffffffu, send, o);
                        }
                        if (up) hb += half;
                        width = half;
                    } else {
#pragma unroll
                        for (int i = 0; i < NV; ++i) a[i] += __shfl_xor_sync(0xffffffffu, a[i], o);
                    }
                }
                // the max over the group: the lanes that differ in the halving bits hold
                // the other heads of the row
                float sc = -INFINITY;
                bool fin = true;
#pragma unroll
                for (int i = 0; i < NV; ++i)
                    if (hb + i < G) {
                        sc = fmaxf(sc, a[i]);
                        fin &= fabsf(a[i]) <= 3.402823466e38f;
                    }
                width = GP;
#pragma unroll
                for (int o = LPR / 2; o >= 1; o >>= 1) {
                    if (width > NV) {
                        sc = fmaxf(sc, __shfl_xor_sync(0xffffffffu, sc, o));
                        width /= 2;
                    }
                }
                bad |= valid && !fin;
                if (piece == 0 && valid) p.keys[r] = fkey(sc);
            }
        };
        for (int k = 0; k < n_st; ++k) {
            const int slot = k % SK_STAGES, n = k / SK_STAGES;
            int got = 0;
            if (lane == 0) got = mbar_wait_bounded(&full[slot], n & 1, &s_abort, p.spin) ? 1 : 0;
            if (!__shfl_sync(0xffffffffu, got, 0)) {
                if (lane == 0) *(volatile int *)&s_abort = 1;
                bad = true;
                break;
            }
            const int64_t r0 = (st0 + k) * SROWS;
            const unsigned char *st = sk_smem + slot * SK_STAGE;
            uint4 w[LOADS];
#pragma unroll
            for (int u = 0; u < LOADS; ++u)
                w[u] = *reinterpret_cast<const uint4 *>(
                    st + (warp * WROWS + u * RPI + sub) * ROW_BYTES + piece * 16);
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[slot]);   // this warp's rows are in registers
            // one unit for the whole stage (the common case): its queries once, and rows
            // without a per-row unit test, so the compiler interleaves them freely
            const int64_t u_lo = r0 / nC, u_hi = (min64(r0 + SROWS, rows_total) - 1) / nC;
            if (u_lo == u_hi && u_lo != qunit) load_q(u_lo);
            if (u_lo == u_hi)
                rows(w, r0, false);
            else
                rows(w, r0, true);
        }
#pragma unroll
        for (int off = 16; off; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
        const bool wbad = __any_sync(0xffffffffu, bad);
        if (lane == 0) {
            s_mx[warp] = mx;
            s_bad[warp] = wbad ? 1 : 0;
        }
    }
    // the selection grid may be scheduled only now: its CTAs would otherwise hold SMs
    // that this grid's later CTAs need
    grid_dep_launch();
    __syncthreads();
    if (threadIdx.x == 0) {
        float m = 0.f;
        int bb = *(volatile int *)&s_abort;
#pragma unroll
        for (int i = 0; i < SK_WARPS; ++i) {
            m = fmaxf(m, s_mx[i]);
            bb |= s_bad[i];
        }
        p.cmx[blockIdx.x] = m;
        p.cbad[blockIdx.x] = (uint32_t)bb;
    }
}

// ------------------------------------------------------------------ selection pass
// Warps that rescore the band in parallel: each needs hd x G doubles of products, and the
// products of all of them fit in 64 KB of shared memory.
__host__ __device__ inline int rescore_warps(int hd, int G) {
    const int n = 65536 / (hd * G * 8);
    return n < 1 ? 1 : n > SL_THREADS / 32 ? SL_THREADS / 32 : n;
}
// Shared-memory layout of the selection pass: queries [hd][G] fp32, keys [nC], the radix
// bins [HIST_BINS], two bit sets [nC / 32], then the products (8-byte aligned).
__host__ __device__ inline size_t prod_offset(int hd, int G, int64_t nC) {
    const size_t o = (size_t)4 * hd * G + 4 * (size_t)((nC + 3) & ~3) + 4 * HIST_BINS +
                     8 * (size_t)((nC + 31) / 32);
    return (o + 15) & ~(size_t)15;
}

template <typename T, int G>
__global__ void __launch_bounds__(SL_THREADS) k_ss_select(const SsParams p) {
    constexpr int NW = SL_THREADS / 32;
    extern __shared__ __align__(16) unsigned char ss_smem[];
    const int hd = p.hd;
    const int nC = (int)p.nC;
    float *qf = reinterpret_cast<float *>(ss_smem);                    // [hd][G]
    uint32_t *keys = reinterpret_cast<uint32_t *>(ss_smem + 4 * hd * G);   // [nC] fp32 keys
    uint32_t *r1 = keys + ((nC + 3) & ~3);                                  // [HIST_BINS]
    uint32_t *bits = r1 + HIST_BINS;                                        // [nC / 32]
    uint32_t *rbits = bits + (nC + 31) / 32;                                // [nC / 32]
    double *prod = reinterpret_cast<double *>(ss_smem + prod_offset(hd, G, nC));   // rescoring
    __shared__ RadixShared<SL_THREADS> rs;
    __shared__ int s_exact, s_bad_res;
    __shared__ unsigned s_cnt, s_nin, s_bin, s_above, s_tkey, s_q1, s_umx;
    const int unit = blockIdx.x;
    const int b = unit / p.Hkv, g = unit % p.Hkv;
    const T *lmu = reinterpret_cast<const T *>(p.lm) + (size_t)unit * nC * hd;
    const T *qg = reinterpret_cast<const T *>(p.q) + ((size_t)b * p.Hq + (size_t)g * G) * hd;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int i = threadIdx.x; i < (nC + 31) / 32; i += SL_THREADS) bits[i] = rbits[i] = 0u;
    if (threadIdx.x == 0) {
        s_bad_res = 0;
        s_cnt = 0u;
        s_nin = 0u;
        s_q1 = 0u;
        s_umx = 0u;
        s_exact = 0;
    }
    __syncthreads();    // the flags and bit sets are clear before any thread sets them
    grid_dep_wait();    // keys, the per-CTA flags and the query come from the kernels before
    grid_dep_launch();
    // every global read of the preamble is issued before the one barrier that ends it
    for (int e = threadIdx.x; e < hd * G; e += SL_THREADS) {
        const int h = e / hd, d = e % hd;
        qf[d * G + h] = Elem<T>::f32(qg[(size_t)h * hd + d]);
    }
    {
        // 16-byte copies only when every unit's keys start on a 16-byte boundary
        const uint32_t *src = p.keys + (size_t)unit * nC;
        const int nvec = (nC & 3) == 0 ? nC / 4 : 0;
        for (int i = threadIdx.x; i < nvec; i += SL_THREADS)
            reinterpret_cast<uint4 *>(keys)[i] = reinterpret_cast<const uint4 *>(src)[i];
        for (int i = 4 * nvec + threadIdx.x; i < nC; i += SL_THREADS) keys[i] = src[i];
    }
    {
        // max |lm| and the bad flag over the key-pass CTAs whose rows meet this unit's (a
        // CTA that also covers a neighbour's rows only makes the bound larger)
        const int64_t rpc = (int64_t)p.sps * p.stage_rows;
        const int c0 = (int)((int64_t)unit * nC / rpc);
        const int c1 = (int)(((int64_t)unit * nC + nC - 1) / rpc);
        for (int c = c0 + (int)threadIdx.x; c <= c1; c += SL_THREADS) {
            atomicMax(&s_umx, __float_as_uint(p.cmx[c]));
            if (p.cbad[c]) s_exact = 1;
        }
    }
    if (p.n_res > 0) {
        // the reserved chunks join the forced set: distinct chunks outside sink and recent
        const int32_t *res = p.reserved + (size_t)unit * p.n_res;
        for (int i = threadIdx.x; i < p.n_res; i += SL_THREADS) {
            const int c = res[i];
            bool bad = c < 0 || c >= nC || c < p.n_sink || c >= nC - p.n_recent;
            if (!bad) bad = (atomicOr(&rbits[c >> 5], 1u << (c & 31)) >> (c & 31)) & 1u;
            if (bad) s_bad_res = 1;
        }
    }
    __syncthreads();
    // max_h ||q_h||_1: a warp per head, fp32 partial sums of exact values (rounded up below)
    for (int h = warp; h < G; h += NW) {
        float sum = 0.f;
        for (int d = lane; d < hd; d += 32) sum += fabsf(qf[d * G + h]);
#pragma unroll
        for (int off = 16; off; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
        if (lane == 0) atomicMax(&s_q1, __float_as_uint(sum));
    }
    __syncthreads();
    auto forced = [&](int c) {
        return c < p.n_sink || c >= nC - p.n_recent || ((rbits[c >> 5] >> (c & 31)) & 1u);
    };
    if (s_bad_res) {
        // a reserved list that is not a set of distinct candidates: the unit selects nothing
        for (int i = threadIdx.x; i < p.n_sel; i += SL_THREADS)
            p.sel[(size_t)unit * p.n_sel + i] = -1;
        if (threadIdx.x == 0) p.band[unit] = BAD_RESERVED;
        return;
    }
    const int f_lo = min(p.n_sink, nC), f_hi = max(nC - p.n_recent, 0);
    const int n_forced = f_lo + (nC - f_hi) - max(0, f_lo - f_hi) + p.n_res;
    const int n_cand = nC - n_forced;
    const int k_eff = min(p.top_k, n_cand);
    const bool all_cand = k_eff == n_cand;         // every candidate is taken
    const float umx = __uint_as_float(s_umx);
    unsigned band_size = 0;
    auto set_bit = [&](int c) { atomicOr(&bits[c >> 5], 1u << (c & 31)); };
    if (!s_exact && k_eff > 0 && !all_cand) {
        // the certified error of every fp32 score of the unit; the fp32 sum of hd
        // non-negative terms is within gamma_hd(2^-24) < 2^-14 of its exact value
        const double q1 = (double)__uint_as_float(s_q1) * (1.0 + 0x1p-14);
        const double E = (p.err_rel * (double)umx * q1 * (1.0 + 0x1p-40)) + p.err_abs;
        // (a) t = the k-th largest candidate key: MSB-first radix descent over 11, 11 and
        //     10 bits of the 32-bit keys; once the bin holding t has at most RANK_CAP
        //     keys they are ranked directly
        uint32_t prefix = 0u, mask = 0u;
        unsigned need = (unsigned)k_eff;
        bool ranked = false;
        for (int level = 0; level < 3; ++level) {
            const int shift = level == 0 ? 21 : level == 1 ? 10 : 0;
            const int nbits = level == 2 ? 10 : 11;
            const int nbins = 1 << nbits;
            for (int i = threadIdx.x; i < nbins; i += SL_THREADS) r1[i] = 0u;
            __syncthreads();
            for (int c = threadIdx.x; c < nC; c += SL_THREADS) {
                const uint32_t k = keys[c];
                if (!forced(c) && (k & mask) == prefix)
                    atomicAdd(&r1[(k >> shift) & (uint32_t)(nbins - 1)], 1u);
            }
            __syncthreads();
            const int bpt = nbins / SL_THREADS;             // bins per thread, walked downwards
            const int top = nbins - 1 - (int)threadIdx.x * bpt;
            unsigned cnt = 0;
            for (int i = 0; i < bpt; ++i) cnt += r1[top - i];
            const unsigned above = block_scan(cnt, rs);
            if (above < need && need <= above + cnt) {
                unsigned cum = above;
                for (int i = 0; i < bpt; ++i) {
                    const unsigned ci = r1[top - i];
                    if (cum + ci >= need) {
                        s_bin = (unsigned)(top - i);
                        s_above = cum;
                        s_cnt = ci;
                        break;
                    }
                    cum += ci;
                }
            }
            __syncthreads();
            prefix |= s_bin << shift;
            mask |= (uint32_t)(nbins - 1) << shift;
            need -= s_above;
            if (level < 2 && s_cnt <= (unsigned)RANK_CAP) {
                ranked = true;
                break;
            }
        }
        float t_lo;
        if (!ranked) {
            t_lo = fkey_inv(prefix);            // every key of the last bin equals t
        } else {
            // (b) rank the few keys of the bin: t is the need-th largest of them
            __syncthreads();
            if (threadIdx.x == 0) s_cnt = 0u;
            __syncthreads();
            for (int c = threadIdx.x; c < nC; c += SL_THREADS) {
                const uint32_t k = keys[c];
                if (!forced(c) && (k & mask) == prefix) r1[atomicAdd(&s_cnt, 1u)] = k;
            }
            __syncthreads();
            const unsigned mb = s_cnt;
            for (unsigned i = threadIdx.x; i < mb; i += SL_THREADS) {
                const uint32_t ki = r1[i];
                unsigned gt = 0, ge = 0;
                for (unsigned j = 0; j < mb; ++j) {
                    const uint32_t kj = r1[j];
                    gt += kj > ki;
                    ge += kj >= ki;
                }
                if (gt < need && need <= ge) s_tkey = ki;
            }
            __syncthreads();
            t_lo = fkey_inv(s_tkey);
        }
        const double lo_b = __dsub_rd((double)t_lo, 2.0 * E);
        const double hi_b = __dadd_ru((double)t_lo, 2.0 * E);
        __syncthreads();
        if (threadIdx.x == 0) s_cnt = 0u;
        if (!(fabs(lo_b) <= 1.7e308) || !(fabs(hi_b) <= 1.7e308)) {
            if (threadIdx.x == 0) s_exact = 1;
        }
        __syncthreads();
        if (!s_exact) {
            // (c) certain chunks into the bit set, the band's chunk indices into r1
            uint32_t *bidx = r1;
            unsigned long long *bkey = reinterpret_cast<unsigned long long *>(r1 + BAND_CAP);
            unsigned nin = 0;
            for (int c = threadIdx.x; c < nC; c += SL_THREADS) {
                if (forced(c)) continue;
                const double sc = (double)fkey_inv(keys[c]);
                if (sc > hi_b) {
                    set_bit(c);
                    ++nin;
                } else if (sc >= lo_b) {
                    const unsigned pos = atomicAdd(&s_cnt, 1u);
                    if (pos < (unsigned)BAND_CAP) bidx[pos] = (uint32_t)c;
                }
            }
#pragma unroll
            for (int off = 16; off; off >>= 1) nin += __shfl_xor_sync(0xffffffffu, nin, off);
            if (lane == 0 && nin) atomicAdd(&s_nin, nin);
            __syncthreads();
            const unsigned m = s_cnt, n_in = s_nin;
            const unsigned need2 = (unsigned)k_eff - n_in;
            if (m > (unsigned)BAND_CAP || need2 < 1u || need2 > m) {
                if (threadIdx.x == 0) s_exact = 1;   // (need2 outside [1, m] cannot happen)
            } else {
                // (d) the band in fp64, as the oracle scores it: a warp per band chunk.  Its
                //     lanes form the exact fp64 products of their columns (one load each),
                //     then lane h adds head h's products in ascending d; fma(x, q, acc)
                //     with an exact product x q is the same rounding as acc + (x q).
                constexpr int EPV = Vec<T>::N;
                const int nwr = rescore_warps(hd, G);
                if (warp < nwr) {
                    double *pr = prod + (size_t)warp * hd * G;
                    const int vpr = hd / EPV;
                    for (unsigned i = warp; i < m; i += nwr) {
                        const uint4 *row = reinterpret_cast<const uint4 *>(lmu + (size_t)bidx[i] * hd);
                        if (lane < vpr) {
                            const uint4 wv = __ldg(row + lane);
#pragma unroll
                            for (int k = 0; k < EPV; ++k) {
                                const int dd = lane * EPV + k;
                                const double x = (double)Vec<T>::get(wv, k);
#pragma unroll
                                for (int h = 0; h < G; ++h)
                                    pr[dd * G + h] = x * (double)qf[dd * G + h];   // exact
                            }
                        }
                        __syncwarp();
                        unsigned long long kb = 0ull;
                        if (lane < G) {
                            double acc = 0.0;
                            for (int dd = 0; dd < hd; ++dd) acc = acc + pr[dd * G + lane];
                            kb = order_key(acc);
                        }
#pragma unroll
                        for (int off = 16; off; off >>= 1) {
                            const unsigned long long o = __shfl_xor_sync(0xffffffffu, kb, off);
                            kb = o > kb ? o : kb;
                        }
                        if (lane == 0) bkey[i] = kb;
                        __syncwarp();
                    }
                }
                __syncthreads();
                // (e) the need2 first of the band under (score desc, chunk index asc): a
                //     chunk's rank counts the band chunks that precede it
                for (unsigned i = threadIdx.x; i < m; i += SL_THREADS) {
                    const unsigned long long ki = bkey[i];
                    const uint32_t ci = bidx[i];
                    unsigned rank_i = 0;
                    for (unsigned j = 0; j < m; ++j) {
                        const unsigned long long kj = bkey[j];
                        rank_i += (kj > ki || (kj == ki && bidx[j] < ci)) ? 1u : 0u;
                    }
                    if (rank_i < need2) set_bit((int)ci);
                }
                band_size = m;
            }
            __syncthreads();
        }
    }
    if (s_exact) {
        // ------------------------------------------------------------ exact path
        // every chunk of the unit in fp64 (through the workspace), then the full select
        for (int i = threadIdx.x; i < (nC + 31) / 32; i += SL_THREADS) bits[i] = 0u;
        double *sc = p.scratch + (size_t)unit * nC;
        bool nan_seen = false;
        for (int c = threadIdx.x; c < nC; c += SL_THREADS) {
            const double v = exact_score<T, G>(lmu + (size_t)c * hd, qf, hd);
            sc[c] = v;
            nan_seen |= isnan(v);
        }
        if (__syncthreads_or(nan_seen)) {
            // NaN scores (inputs outside the contract): the unit selects nothing
            for (int i = threadIdx.x; i < p.n_sel; i += SL_THREADS)
                p.sel[(size_t)unit * p.n_sel + i] = -1;
            if (threadIdx.x == 0) p.band[unit] = EXACT_PATH;
            return;
        }
        if (k_eff > 0 && !all_cand)
            radix_select(nC, (unsigned)k_eff, [&](int c) { return order_key(sc[c]); },
                         [&](int c) { return !forced(c); }, [&](int c) { set_bit(c); }, rs);
        band_size = EXACT_PATH;
    }
    // ------------------------------------------------------------ output
    // ascending order: thread t takes chunks [32 t, 32 t + 32) as one word of taken bits
    // (forced, all candidates, or in the bit set), one scan places the words
    __syncthreads();
    {
        const int t = threadIdx.x;
        const int n_words = (nC + 31) / 32;
        uint32_t tw = 0u;
        if (t < n_words) {
            const int c0 = 32 * t;
            auto below = [&](int x) -> uint32_t {   // bits of the chunks c0 + j < x
                const int n = x - c0;
                return n <= 0 ? 0u : n >= 32 ? 0xFFFFFFFFu : ((1u << n) - 1u);
            };
            const uint32_t valid = below(nC);
            const uint32_t sink = below(p.n_sink);
            const uint32_t recent = valid & ~below(nC - p.n_recent);
            tw = (bits[t] | rbits[t] | sink | recent | (all_cand ? 0xFFFFFFFFu : 0u)) & valid;
        }
        unsigned pos = block_scan(__popc(tw), rs);
        int32_t *out = p.sel + (size_t)unit * p.n_sel;
        while (tw) {
            const int j = __ffs(tw) - 1;
            tw &= tw - 1u;
            if (pos < (unsigned)p.n_sel) out[pos] = 32 * t + j;
            ++pos;
        }
    }
    if (threadIdx.x == 0) p.band[unit] = band_size;
}

// The value-range reservation (VASE page, section 2.A, applied to chunks): per (b, g) the
// n_res chunks outside the sink and recent windows with the largest rho, under (rho
// descending, index ascending), written in ascending order.  rho is fp32; its keys are
// those of the value widened to fp64, so the order is exactly the oracle's on the same
// statistics.
__global__ void __launch_bounds__(RES_THREADS) k_reserve(const float *__restrict__ rho,
                                                        int32_t *__restrict__ reserved,
                                                        int nC, int n_res, int n_sink,
                                                        int n_recent) {
    __shared__ RadixShared<RES_THREADS> rs;
    __shared__ uint32_t bits[16384 / 32];
    const int unit = blockIdx.x;
    const float *r = rho + (size_t)unit * nC;
    for (int i = threadIdx.x; i < (nC + 31) / 32; i += RES_THREADS) bits[i] = 0u;
    __syncthreads();
    auto forced = [&](int c) { return c < n_sink || c >= nC - n_recent; };
    radix_select(nC, (unsigned)n_res, [&](int c) { return order_key((double)r[c]); },
                 [&](int c) { return !forced(c); },
                 [&](int c) { atomicOr(&bits[c >> 5], 1u << (c & 31)); }, rs);
    const int ipt = (nC + RES_THREADS - 1) / RES_THREADS;
    const int lo = min(nC, (int)threadIdx.x * ipt), hi = min(nC, lo + ipt);
    unsigned n_local = 0;
    for (int c = lo; c < hi; ++c) n_local += (bits[c >> 5] >> (c & 31)) & 1u;
    unsigned pos = block_scan(n_local, rs);
    int32_t *out = reserved + (size_t)unit * n_res;
    for (int c = lo; c < hi; ++c)
        if ((bits[c >> 5] >> (c & 31)) & 1u) {
            if (pos < (unsigned)n_res) out[pos] = c;
            ++pos;
        }
}

size_t ss_smem_bytes(const xkv_dims &d) {
    const int G = d.n_q_heads / d.n_kv_heads;
    const int64_t nC = d.ctx_len / d.chunk;
    return prod_offset(d.head_dim, G, nC) +
           (size_t)rescore_warps(d.head_dim, G) * d.head_dim * G * 8;
}

double gamma_n(int n, double u) { return n * u / (1.0 - n * u); }

template <typename T, int G, int LPR>
cudaError_t launch_keys(const SsParams &p, cudaStream_t s) {
    auto k = k_ss_keys<T, G, LPR>;
    const size_t smem = (size_t)SK_STAGES * SK_STAGE;
    cudaError_t e = set_smem_limit((const void *)k, smem);
    if (e != cudaSuccess) return e;
    return launch_chained(k, dim3(p.n_cta), dim3(SK_THREADS), smem, s, p);
}

template <typename T, int G>
cudaError_t launch_tg(const xkv_dims &d, const SsParams &p, cudaStream_t s) {
    const int lpr = d.head_dim * (int)sizeof(T) / 16;   // lanes per landmark row
    cudaError_t e = lpr == 8    ? launch_keys<T, G, 8>(p, s)
                    : lpr == 16 ? launch_keys<T, G, 16>(p, s)
                    : lpr == 32 ? launch_keys<T, G, 32>(p, s)
                                : cudaErrorInvalidValue;
    if (e != cudaSuccess) return e;
    auto k = k_ss_select<T, G>;
    const size_t smem = ss_smem_bytes(d);
    if ((e = set_smem_limit((const void *)k, smem)) != cudaSuccess) return e;
    return launch_chained(k, dim3(d.batch * d.n_kv_heads), dim3(SL_THREADS), smem, s, p);
}

template <typename T>
cudaError_t launch_t(const xkv_dims &d, const SsParams &p, cudaStream_t s) {
    switch (d.n_q_heads / d.n_kv_heads) {
        case 1: return launch_tg<T, 1>(d, p, s);
        case 2: return launch_tg<T, 2>(d, p, s);
        case 3: return launch_tg<T, 3>(d, p, s);
        case 4: return launch_tg<T, 4>(d, p, s);
        case 5: return launch_tg<T, 5>(d, p, s);
        case 6: return launch_tg<T, 6>(d, p, s);
        case 7: return launch_tg<T, 7>(d, p, s);
        case 8: return launch_tg<T, 8>(d, p, s);
        case 16: return launch_tg<T, 16>(d, p, s);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace

bool score_select_shape_ok(const xkv_dims &d) {
    const int G = d.n_q_heads / d.n_kv_heads;
    return (G >= 1 && G <= 8) || G == 16;
}

// workspace: band sizes [units] (first 256 bytes-aligned block), fp64 scratch of the exact
// path [units][nC], fp32 keys [units][nC], then per key-pass CTA max |lm| and flag
static size_t al256(size_t n) { return (n + 255) / 256 * 256; }
size_t score_select_ws_bytes(const xkv_dims &d) {
    const size_t units = (size_t)d.batch * d.n_kv_heads;
    const size_t nC = (size_t)(d.ctx_len / d.chunk);
    return al256(units * 4) + al256(units * nC * 8) + al256(units * nC * 4) +
           al256((size_t)SK_MAX_CTAS * 4) + (size_t)SK_MAX_CTAS * 4;
}

size_t score_select_smem_bytes(const xkv_dims &d) { return ss_smem_bytes(d); }

cudaError_t launch_reserve(const xkv_dims &d, const float *rho, int n_res, int n_sink,
                           int n_recent, int32_t *reserved, cudaStream_t s) {
    k_reserve<<<d.batch * d.n_kv_heads, RES_THREADS, 0, s>>>(
        rho, reserved, (int)(d.ctx_len / d.chunk), n_res, n_sink, n_recent);
    return cudaGetLastError();
}

cudaError_t launch_score_select(const xkv_dims &d, const void *lm, const void *q, int top_k,
                                int n_sink, int n_recent, const int32_t *reserved, int n_res,
                                int32_t *sel, int n_sel, void *ws, cudaStream_t s) {
    const size_t units = (size_t)d.batch * d.n_kv_heads;
    const size_t nC = (size_t)(d.ctx_len / d.chunk);
    SsParams p;
    p.lm = lm;
    p.q = q;
    p.sel = sel;
    char *w = (char *)ws;
    p.band = reinterpret_cast<uint32_t *>(w);
    w += al256(units * 4);
    p.scratch = reinterpret_cast<double *>(w);
    w += al256(units * nC * 8);
    p.keys = reinterpret_cast<uint32_t *>(w);
    w += al256(units * nC * 4);
    // key pass: stages of whole landmark rows over all units, about one CTA per SM
    const int esize = d.dtype == XKV_F32 ? 4 : 2;
    p.stage_rows = SK_STAGE / (d.head_dim * esize);
    p.rows_total = (int64_t)(units * nC);
    p.n_stages = (p.rows_total + p.stage_rows - 1) / p.stage_rows;
    int64_t n_cta = sm_count() < SK_MAX_CTAS ? sm_count() : SK_MAX_CTAS;
    if (n_cta > p.n_stages) n_cta = p.n_stages;
    p.sps = (int)((p.n_stages + n_cta - 1) / n_cta);
    p.n_cta = (int)((p.n_stages + p.sps - 1) / p.sps);
    p.cmx = reinterpret_cast<float *>(w);
    w += al256((size_t)SK_MAX_CTAS * 4);
    p.cbad = reinterpret_cast<uint32_t *>(w);
    p.nC = (int64_t)nC;
    p.Hq = d.n_q_heads;
    p.Hkv = d.n_kv_heads;
    p.hd = d.head_dim;
    p.top_k = top_k;
    p.n_sink = n_sink;
    p.n_recent = n_recent;
    p.n_sel = n_sel;
    p.reserved = reserved;
    p.n_res = reserved ? n_res : 0;
    // XKV_TEST_SS_SPIN (tests only, read on every call): a shorter poll limit for the key
    // pass's pipeline waits, so a test can make them give up (the units then take the
    // exact path); the drain of the copies in flight keeps its full bound
    p.spin = test_poll_limit("XKV_TEST_SS_SPIN", SK_SPIN);
    const double slack = 1.0 + 0x1p-20;
    p.err_rel = (gamma_n(d.head_dim, 0x1p-24) + gamma_n(d.head_dim, 0x1p-53)) * slack;
    p.err_abs = d.head_dim * 0x1p-150 * slack;
    return d.dtype == XKV_F32 ? launch_t<float>(d, p, s) : launch_t<__nv_bfloat16>(d, p, s);
}

}  // namespace xkv
