// Fused landmark scoring + chunk selection (xKV page, section 2.3: rank the chunks by the
// relevance of their landmark key to the current query, max over the GQA group, and keep
// the top-k plus the always-kept sink and recent chunks).
//
// The result is bit for bit the selection that xkv_select_chunks makes from the scores of
// xkv_score_landmarks (canonical fp64 sums of exact products in ascending d, ties to the
// lower chunk index), but the landmarks are scored in fp32 and only the chunks whose order
// the fp32 pass cannot certify are scored again in fp64:
//
//  1. every chunk c gets an fp32 score s~_c (fmaf chains, ascending d, max over the group)
//     with a certified bound |s~_c - s_c| <= E, where s_c is the canonical fp64 score:
//       E = (gamma_hd(2^-24) + gamma_hd(2^-53)) * max|lm| * max_h ||q_h||_1 + hd * 2^-150,
//     gamma_n(u) = n u / (1 - n u) (the classical bound of a recursive dot product whose
//     every step rounds once; 2^-150 covers fp32 underflow; the fp64 term covers the
//     rounding of the canonical sum itself), inflated by 1 + 2^-20;
//  2. t = the k-th largest s~ among the candidates.  At least k candidates have s~ >= t,
//     so the k-th largest canonical score s_(k) >= t - E; at most k - 1 have s~ > t, so
//     s_(k) <= t + E.  A candidate with s~ > t + 2E therefore has s > s_(k): it is
//     selected whatever the ties; one with s~ < t - 2E has s < s_(k): it is not;
//  3. the rest (the band) is scored in fp64 exactly as the oracle scores it, and the
//     top (k - #selected) of the band under (score desc, index asc) complete the set.
//
// Work split: one thread-block cluster per (sequence, KV head) unit, a CTA of 256 threads
// per 512 chunks (at most 8, the portable cluster size).  Every CTA of the cluster
// streams its slice of the unit's landmark rows (two rows per thread, 16-byte loads, the
// group's query in shared memory) and sends its fp32 keys to CTA 0's shared memory; CTA 0
// then runs steps 2-3 and writes the selection in ascending chunk order.  The steps of
// CTA 0 are written for latency: strided (bank-conflict-free) passes over the keys, the
// band ranked by counting (no ordering needed), the output placed by ballots.
// Optionally a per-unit list of reserved chunks (the value-range reservation) joins the
// sink and recent chunks as forced.  Units whose fp32 scores are not all finite or whose
// band is wider than BAND_CAP chunks take the exact path for the whole unit: every chunk is
// scored in fp64 into the workspace and the full radix select runs on those keys.  The
// workspace also records, per unit, the band size (or ~0 for the exact path).
//
// Chosen for B200: 67 MB of landmarks per layer at the bench workload need ~10 us at the
// copy bandwidth, while the fp64 pass spent ~30 us on conversions and fp64 FMAs; fp32
// FMAs and shift-only bf16 widening keep the stream HBM-bound.
#include "xkv_internal.cuh"

namespace xkv {
namespace {

constexpr int SS_THREADS = 256;
constexpr int SS_WARPS = SS_THREADS / 32;
constexpr int SS_RPT = 2;                         // rows per thread per pass
constexpr int SS_ROWS = SS_THREADS * SS_RPT;      // rows per CTA pass
constexpr int SS_MAX_CLUSTER = 8;                 // portable cluster size
constexpr int HIST_BINS = 2048;                   // radix digits of 11, 11 and 10 bits
constexpr int RANK_CAP = 32;                      // keys of a bin ranked directly
constexpr int BAND_CAP = 512;                     // band chunks rescored in fp64
constexpr uint32_t EXACT_PATH = 0xFFFFFFFFu;
constexpr uint32_t BAD_RESERVED = 0xFFFFFFFEu;   // a reserved list broke its rules

struct SsParams {
    const void *lm;       // [B][Hkv][nC][hd]
    const void *q;        // [B][Hq][hd]
    int32_t *sel;         // [B][Hkv][n_sel]
    uint32_t *band;       // [B][Hkv] band size per unit (EXACT_PATH for the exact path)
    double *scratch;      // [B][Hkv][nC] fp64 scores of units on the exact path
    int64_t nC;
    int Hq, Hkv, hd;
    int top_k, n_sink, n_recent, n_sel;
    int cpc;              // chunks per CTA (a multiple of 4)
    const int32_t *reserved;   // [B][Hkv][n_res] chunks forced in as well, or null
    int n_res;
    double err_rel;       // (gamma_hd(2^-24) + gamma_hd(2^-53)) (1 + 2^-20)
    double err_abs;       // hd 2^-150 (1 + 2^-20)
};

// --------------------------------------------------------------- cluster primitives
__device__ __forceinline__ uint32_t cta_rank_in_cluster() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
__device__ __forceinline__ uint32_t smem_addr(const void *p) {
    return (uint32_t)__cvta_generic_to_shared(p);
}
// Address of the same shared-memory location in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t map_to_rank(const void *p, uint32_t rank) {
    uint32_t a;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(a) : "r"(smem_addr(p)), "r"(rank));
    return a;
}
__device__ __forceinline__ void st_cluster(uint32_t addr, uint32_t v) {
    asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}
__device__ __forceinline__ void st_cluster(uint32_t addr, uint4 v) {
    asm volatile("st.shared::cluster.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x),
                 "r"(v.y), "r"(v.z), "r"(v.w)
                 : "memory");
}
__device__ __forceinline__ void cluster_arrive_relaxed() {
    asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_arrive_release() {
    asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait() {
    asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

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
// ascending d, then the max over the group with -0 below +0.
template <typename T, int G>
__device__ double exact_score(const T *row, const float *qf, int hd) {
    constexpr int EPV = Vec<T>::N;
    double acc[G];
#pragma unroll
    for (int h = 0; h < G; ++h) acc[h] = 0.0;
    const uint4 *v = reinterpret_cast<const uint4 *>(row);
    for (int i = 0; i < hd / EPV; ++i) {
        const uint4 w = __ldg(v + i);
#pragma unroll
        for (int k = 0; k < EPV; ++k) {
            const double x = (double)Vec<T>::get(w, k);
            const float *qd = qf + (i * EPV + k) * G;
#pragma unroll
            for (int h = 0; h < G; ++h) acc[h] = fma(x, (double)qd[h], acc[h]);   // exact product
        }
    }
    double best = acc[0];
#pragma unroll
    for (int h = 1; h < G; ++h)
        if (order_key(acc[h]) > order_key(best)) best = acc[h];
    return best;
}

// ------------------------------------------------------------------ block helpers
struct RadixShared {
    unsigned hist[2][256];
    unsigned warp_tot[SS_WARPS];
    unsigned total;
    unsigned long long prefix, mask;
    unsigned krem;
    int done;
};

// Exclusive prefix sum over the CTA of one value per thread; *total gets the sum.
__device__ unsigned block_scan(unsigned v, RadixShared &rs) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    unsigned inc = v;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const unsigned t = __shfl_up_sync(0xffffffffu, inc, off);
        if (lane >= off) inc += t;
    }
    if (lane == 31) rs.warp_tot[warp] = inc;
    __syncthreads();
    if (threadIdx.x == 0) {
        unsigned run = 0;
        for (int w = 0; w < SS_WARPS; ++w) {
            const unsigned t = rs.warp_tot[w];
            rs.warp_tot[w] = run;
            run += t;
        }
        rs.total = run;
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
template <class KeyF, class CandF, class TakeF>
__device__ void radix_select(int n, unsigned need, KeyF key, CandF cand, TakeF take,
                             RadixShared &rs) {
    if (threadIdx.x == 0) {
        rs.prefix = 0ull;
        rs.mask = 0ull;
        rs.krem = need;
        rs.done = 0;
    }
    for (int i = threadIdx.x; i < 256; i += SS_THREADS) rs.hist[0][i] = 0u;
    __syncthreads();
    unsigned long long mask = 0ull;
    int buf = 0;
    for (int shift = 56; shift >= 0; shift -= 8, buf ^= 1) {
        const unsigned long long prefix = rs.prefix;
        for (int i = threadIdx.x; i < n; i += SS_THREADS) {
            if (!cand(i)) continue;
            const unsigned long long k = key(i);
            if ((k & mask) == prefix) atomicAdd(&rs.hist[buf][(unsigned)(k >> shift) & 255u], 1u);
        }
        __syncthreads();
        if (threadIdx.x >= 32) {
            for (int i = threadIdx.x - 32; i < 256; i += SS_THREADS - 32) rs.hist[buf ^ 1][i] = 0u;
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
    const int ipt = (n + SS_THREADS - 1) / SS_THREADS;
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

template <typename T, int G>
__global__ void __launch_bounds__(SS_THREADS) k_score_select(const SsParams p) {
    extern __shared__ __align__(16) unsigned char ss_smem[];
    const int hd = p.hd;
    const int nC = (int)p.nC;
    float *qf = reinterpret_cast<float *>(ss_smem);                    // [hd][G]
    uint32_t *keys = reinterpret_cast<uint32_t *>(ss_smem + 4 * hd * G);   // [nC] fp32 keys
    uint32_t *r1 = keys + ((nC + 3) & ~3);                                  // [HIST_BINS]
    uint32_t *bits = r1 + HIST_BINS;                                        // [nC / 32]
    uint32_t *rbits = bits + (nC + 31) / 32;                                // [nC / 32]
    __shared__ float s_mx[SS_MAX_CLUSTER];
    __shared__ int s_bad[SS_MAX_CLUSTER];
    __shared__ RadixShared rs;
    __shared__ int s_bad_cta, s_exact, s_bad_res;
    __shared__ unsigned s_cnt, s_nin, s_bin, s_above, s_tkey, s_q1;
    __shared__ float s_mx_cta;

    // announce this CTA; the matching wait comes before the first remote store
    cluster_arrive_relaxed();
    const uint32_t rank = cta_rank_in_cluster();
    const int g = blockIdx.y, b = blockIdx.z;
    const int unit = b * p.Hkv + g;
    const T *lmu = reinterpret_cast<const T *>(p.lm) + (size_t)unit * nC * hd;
    const T *qg = reinterpret_cast<const T *>(p.q) + ((size_t)b * p.Hq + (size_t)g * G) * hd;
    grid_dep_wait();    // the landmarks and the query may come from the kernels before
    grid_dep_launch();
    for (int e = threadIdx.x; e < hd * G; e += SS_THREADS) {
        const int h = e / hd, d = e % hd;
        qf[d * G + h] = Elem<T>::f32(qg[(size_t)h * hd + d]);
    }
    if (rank == 0) {
        for (int i = threadIdx.x; i < HIST_BINS; i += SS_THREADS) r1[i] = 0u;
        for (int i = threadIdx.x; i < (nC + 31) / 32; i += SS_THREADS) bits[i] = rbits[i] = 0u;
    }
    if (threadIdx.x == 0) {
        s_bad_cta = 0;
        s_mx_cta = 0.f;
        s_bad_res = 0;
    }
    __syncthreads();
    if (rank == 0 && p.n_res > 0) {
        // the reserved chunks join the forced set: distinct chunks outside sink and recent
        const int32_t *res = p.reserved + (size_t)unit * p.n_res;
        for (int i = threadIdx.x; i < p.n_res; i += SS_THREADS) {
            const int c = res[i];
            bool bad = c < 0 || c >= nC || c < p.n_sink || c >= nC - p.n_recent;
            if (!bad) bad = (atomicOr(&rbits[c >> 5], 1u << (c & 31)) >> (c & 31)) & 1u;
            if (bad) s_bad_res = 1;
        }
    }

    // ---------------------------------------------------------------- fp32 pass
    constexpr int EPV = Vec<T>::N;
    const int vpr = hd / EPV;
    const int c_begin = min(nC, (int)rank * p.cpc), c_end = min(nC, c_begin + p.cpc);
    float mx = 0.f;
    bool bad = false;
    for (int base = c_begin; base < c_end; base += SS_ROWS) {
        int cr[SS_RPT];
        const uint4 *rp[SS_RPT];
#pragma unroll
        for (int i = 0; i < SS_RPT; ++i) {
            cr[i] = base + (int)threadIdx.x + i * SS_THREADS;
            rp[i] = reinterpret_cast<const uint4 *>(lmu + (size_t)(cr[i] < c_end ? cr[i] : c_begin) * hd);
        }
        float acc[SS_RPT][G];
#pragma unroll
        for (int i = 0; i < SS_RPT; ++i)
#pragma unroll
            for (int h = 0; h < G; ++h) acc[i][h] = 0.f;
        // a row is read a 128-byte line at a time: the eight 16-byte loads of a line go
        // out back to back and merge in flight (shared memory leaves L1 too small to keep
        // a line between loads spread over the arithmetic)
        for (int v0 = 0; v0 < vpr; v0 += 8) {
            uint4 w[SS_RPT][8];
#pragma unroll
            for (int i = 0; i < SS_RPT; ++i)
#pragma unroll
                for (int v = 0; v < 8; ++v) w[i][v] = __ldg(rp[i] + v0 + v);
#pragma unroll
            for (int v = 0; v < 8; ++v)
#pragma unroll
                for (int k = 0; k < EPV; ++k) {
                    float x[SS_RPT];
#pragma unroll
                    for (int i = 0; i < SS_RPT; ++i) {
                        x[i] = Vec<T>::get(w[i][v], k);
                        mx = fmaxf(mx, fabsf(x[i]));
                    }
                    const float *qd = qf + ((v0 + v) * EPV + k) * G;
#pragma unroll
                    for (int h = 0; h < G; ++h) {
                        const float qv = qd[h];
#pragma unroll
                        for (int i = 0; i < SS_RPT; ++i) acc[i][h] = fmaf(x[i], qv, acc[i][h]);
                    }
                }
        }
#pragma unroll
        for (int i = 0; i < SS_RPT; ++i) {
            if (cr[i] >= c_end) continue;
            float s = acc[i][0];
            bool fin = fabsf(acc[i][0]) <= 3.402823466e38f;
#pragma unroll
            for (int h = 1; h < G; ++h) {
                s = fmaxf(s, acc[i][h]);
                fin &= fabsf(acc[i][h]) <= 3.402823466e38f;
            }
            bad |= !fin;
            keys[cr[i]] = fkey(s);
        }
    }
    // the CTA's max |lm| and non-finite flag, sent to CTA 0 with its keys
#pragma unroll
    for (int off = 16; off; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
    if ((threadIdx.x & 31) == 0) atomicMax(reinterpret_cast<int *>(&s_mx_cta), __float_as_int(mx));
    if (__syncthreads_or(bad) && threadIdx.x == 0) s_bad_cta = 1;
    __syncthreads();
    cluster_wait();                 // every CTA of the cluster is running
    if (rank != 0) {
        const int n = c_end - c_begin;
        if (n > 0) {
            const uint32_t dst = map_to_rank(keys + c_begin, 0);
            const uint4 *src = reinterpret_cast<const uint4 *>(keys + c_begin);
            for (int i = threadIdx.x; i < n / 4; i += SS_THREADS) st_cluster(dst + 16u * i, src[i]);
            for (int i = (n & ~3) + threadIdx.x; i < n; i += SS_THREADS)
                st_cluster(dst + 4u * i, keys[c_begin + i]);
        }
    }
    if (threadIdx.x == 0) {
        st_cluster(map_to_rank(&s_mx[rank], 0), __float_as_uint(s_mx_cta));
        st_cluster(map_to_rank(&s_bad[rank], 0), (uint32_t)s_bad_cta);
    }
    cluster_arrive_release();
    cluster_wait();                 // CTA 0 now holds every key of the unit
    if (rank != 0) return;

    // ---------------------------------------------------------------- CTA 0: selection
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int ncl = (int)((nC + p.cpc - 1) / p.cpc);
    const int f_lo = min(p.n_sink, nC), f_hi = max(nC - p.n_recent, 0);
    auto forced = [&](int c) {
        return c < p.n_sink || c >= nC - p.n_recent || ((rbits[c >> 5] >> (c & 31)) & 1u);
    };
    if (s_bad_res) {
        // a reserved list that is not a set of distinct candidates: the unit selects nothing
        for (int i = threadIdx.x; i < p.n_sel; i += SS_THREADS)
            p.sel[(size_t)unit * p.n_sel + i] = -1;
        if (threadIdx.x == 0) p.band[unit] = BAD_RESERVED;
        return;
    }
    const int n_forced = f_lo + (nC - f_hi) - max(0, f_lo - f_hi) + p.n_res;
    const int n_cand = nC - n_forced;
    const int k_eff = min(p.top_k, n_cand);
    const bool all_cand = k_eff == n_cand;         // every candidate is taken
    float umx = 0.f;
    int ubad = 0;
    for (int r = 0; r < ncl; ++r) {
        umx = fmaxf(umx, s_mx[r]);
        ubad |= s_bad[r];
    }
    if (threadIdx.x == 0) {
        s_exact = ubad;
        s_cnt = 0u;
        s_nin = 0u;
        s_q1 = 0u;
    }
    __syncthreads();
    // max_h ||q_h||_1: a warp per head, fp32 partial sums of exact values (rounded up below)
    for (int h = warp; h < G; h += SS_WARPS) {
        float sum = 0.f;
        for (int d = lane; d < hd; d += 32) sum += fabsf(qf[d * G + h]);
#pragma unroll
        for (int off = 16; off; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
        if (lane == 0) atomicMax(&s_q1, __float_as_uint(sum));
    }
    __syncthreads();
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
            for (int i = threadIdx.x; i < nbins; i += SS_THREADS) r1[i] = 0u;
            __syncthreads();
            for (int c = threadIdx.x; c < nC; c += SS_THREADS) {
                const uint32_t k = keys[c];
                if (!forced(c) && (k & mask) == prefix)
                    atomicAdd(&r1[(k >> shift) & (uint32_t)(nbins - 1)], 1u);
            }
            __syncthreads();
            const int bpt = nbins / SS_THREADS;             // bins per thread, walked downwards
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
            if (threadIdx.x == 0) s_cnt = 0u;
            __syncthreads();
            for (int c = threadIdx.x; c < nC; c += SS_THREADS) {
                const uint32_t k = keys[c];
                if (!forced(c) && (k & mask) == prefix) r1[atomicAdd(&s_cnt, 1u)] = k;
            }
            __syncthreads();
            const unsigned mb = s_cnt;
            for (unsigned i = threadIdx.x; i < mb; i += SS_THREADS) {
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
            for (int c = threadIdx.x; c < nC; c += SS_THREADS) {
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
                // (d) the band in fp64, as the oracle scores it
                for (unsigned i = threadIdx.x; i < m; i += SS_THREADS)
                    bkey[i] = order_key(exact_score<T, G>(lmu + (size_t)bidx[i] * hd, qf, hd));
                __syncthreads();
                // (e) the need2 first of the band under (score desc, chunk index asc): a
                //     chunk's rank counts the band chunks that precede it
                for (unsigned i = threadIdx.x; i < m; i += SS_THREADS) {
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
        for (int i = threadIdx.x; i < (nC + 31) / 32; i += SS_THREADS) bits[i] = 0u;
        double *sc = p.scratch + (size_t)unit * nC;
        bool nan_seen = false;
        for (int c = threadIdx.x; c < nC; c += SS_THREADS) {
            const double v = exact_score<T, G>(lmu + (size_t)c * hd, qf, hd);
            sc[c] = v;
            nan_seen |= isnan(v);
        }
        if (__syncthreads_or(nan_seen)) {
            // NaN scores (inputs outside the contract): the unit selects nothing
            for (int i = threadIdx.x; i < p.n_sel; i += SS_THREADS)
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
    // ascending order: 32-chunk groups, a ballot per group, a scan over the group counts
    const int n_groups = (nC + 31) / 32;
    uint32_t *gcount = r1, *gbase = r1 + HIST_BINS / 2;
    auto taken = [&](int c) {
        return c < nC && (forced(c) || all_cand || ((bits[c >> 5] >> (c & 31)) & 1u));
    };
    __syncthreads();
    for (int gi = warp; gi < n_groups; gi += SS_WARPS) {
        const unsigned bal = __ballot_sync(0xffffffffu, taken(gi * 32 + lane));
        if (lane == 0) gcount[gi] = __popc(bal);
    }
    __syncthreads();
    {
        const int gpt = (n_groups + SS_THREADS - 1) / SS_THREADS;   // groups per thread
        const int g0 = min(n_groups, (int)threadIdx.x * gpt), g1 = min(n_groups, g0 + gpt);
        unsigned cnt = 0;
        for (int gi = g0; gi < g1; ++gi) cnt += gcount[gi];
        unsigned run = block_scan(cnt, rs);
        for (int gi = g0; gi < g1; ++gi) {
            gbase[gi] = run;
            run += gcount[gi];
        }
    }
    __syncthreads();
    int32_t *out = p.sel + (size_t)unit * p.n_sel;
    for (int gi = warp; gi < n_groups; gi += SS_WARPS) {
        const int c = gi * 32 + lane;
        const bool tk = taken(c);
        const unsigned bal = __ballot_sync(0xffffffffu, tk);
        const unsigned pos = gbase[gi] + __popc(bal & ((1u << lane) - 1u));
        if (tk && pos < (unsigned)p.n_sel) out[pos] = c;
    }
    if (threadIdx.x == 0) p.band[unit] = band_size;
}

// The value-range reservation (VASE page, section 2.A, applied to chunks): per (b, g) the
// n_res chunks outside the sink and recent windows with the largest rho, under (rho
// descending, index ascending), written in ascending order.  rho is fp32; its keys are
// those of the value widened to fp64, so the order is exactly the oracle's on the same
// statistics.
__global__ void __launch_bounds__(SS_THREADS) k_reserve(const float *__restrict__ rho,
                                                        int32_t *__restrict__ reserved,
                                                        int nC, int n_res, int n_sink,
                                                        int n_recent) {
    __shared__ RadixShared rs;
    __shared__ uint32_t bits[16384 / 32];
    const int unit = blockIdx.x;
    const float *r = rho + (size_t)unit * nC;
    for (int i = threadIdx.x; i < (nC + 31) / 32; i += SS_THREADS) bits[i] = 0u;
    __syncthreads();
    auto forced = [&](int c) { return c < n_sink || c >= nC - n_recent; };
    radix_select(nC, (unsigned)n_res, [&](int c) { return order_key((double)r[c]); },
                 [&](int c) { return !forced(c); },
                 [&](int c) { atomicOr(&bits[c >> 5], 1u << (c & 31)); }, rs);
    const int ipt = (nC + SS_THREADS - 1) / SS_THREADS;
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
    return (size_t)4 * d.head_dim * G + 4 * (size_t)((nC + 3) & ~3) + 4 * HIST_BINS +
           8 * (size_t)((nC + 31) / 32);
}

double gamma_n(int n, double u) { return n * u / (1.0 - n * u); }

template <typename T, int G>
cudaError_t launch_tg(const xkv_dims &d, const SsParams &p0, cudaStream_t s) {
    auto k = k_score_select<T, G>;
    const size_t smem = ss_smem_bytes(d);
    cudaError_t e = set_smem_limit((const void *)k, smem);
    if (e != cudaSuccess) return e;
    const int64_t nC = d.ctx_len / d.chunk;
    int cs = (int)((nC + SS_ROWS - 1) / SS_ROWS);
    cs = cs < 1 ? 1 : cs > SS_MAX_CLUSTER ? SS_MAX_CLUSTER : cs;
    cudaLaunchConfig_t cfg = {};
    cfg.blockDim = dim3(SS_THREADS);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    SsParams p = p0;
    p.cpc = (int)(((nC + cs - 1) / cs + 3) & ~3);
    cudaLaunchAttribute at[2];
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = cs;
    at[0].val.clusterDim.y = 1;
    at[0].val.clusterDim.z = 1;
    at[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.gridDim = dim3(cs, d.n_kv_heads, d.batch);
    cfg.attrs = at;
    cfg.numAttrs = chain_enabled() ? 2 : 1;
    return cudaLaunchKernelEx(&cfg, k, p);
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

size_t score_select_ws_bytes(const xkv_dims &d) {
    const size_t units = (size_t)d.batch * d.n_kv_heads;
    return (units * 4 + 255) / 256 * 256 + units * (size_t)(d.ctx_len / d.chunk) * 8;
}

size_t score_select_smem_bytes(const xkv_dims &d) { return ss_smem_bytes(d); }

cudaError_t launch_reserve(const xkv_dims &d, const float *rho, int n_res, int n_sink,
                           int n_recent, int32_t *reserved, cudaStream_t s) {
    k_reserve<<<d.batch * d.n_kv_heads, SS_THREADS, 0, s>>>(
        rho, reserved, (int)(d.ctx_len / d.chunk), n_res, n_sink, n_recent);
    return cudaGetLastError();
}

cudaError_t launch_score_select(const xkv_dims &d, const void *lm, const void *q, int top_k,
                                int n_sink, int n_recent, const int32_t *reserved, int n_res,
                                int32_t *sel, int n_sel, void *ws, cudaStream_t s) {
    const size_t units = (size_t)d.batch * d.n_kv_heads;
    SsParams p;
    p.lm = lm;
    p.q = q;
    p.sel = sel;
    p.band = reinterpret_cast<uint32_t *>(ws);
    p.scratch = reinterpret_cast<double *>((char *)ws + (units * 4 + 255) / 256 * 256);
    p.nC = d.ctx_len / d.chunk;
    p.Hq = d.n_q_heads;
    p.Hkv = d.n_kv_heads;
    p.hd = d.head_dim;
    p.top_k = top_k;
    p.n_sink = n_sink;
    p.n_recent = n_recent;
    p.n_sel = n_sel;
    p.cpc = 0;
    p.reserved = reserved;
    p.n_res = reserved ? n_res : 0;
    const double slack = 1.0 + 0x1p-20;
    p.err_rel = (gamma_n(d.head_dim, 0x1p-24) + gamma_n(d.head_dim, 0x1p-53)) * slack;
    p.err_abs = d.head_dim * 0x1p-150 * slack;
    return d.dtype == XKV_F32 ? launch_t<float>(d, p, s) : launch_t<__nv_bfloat16>(d, p, s);
}

}  // namespace xkv
