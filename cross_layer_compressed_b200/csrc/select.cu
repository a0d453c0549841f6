// Chunk selection (xKV page, section 2.3: keep the chunks most relevant to the query,
// plus the always-kept sink and recent chunks).
//
// One CTA per (sequence, KV head).  Scores become 64-bit keys that order like the
// doubles (-0 below +0); an MSB-first radix select over 8-bit digits narrows a key prefix
// T (under a mask M) holding the k-th best candidate and counts how many candidates with
// that prefix are still needed.  It stops early once every candidate with the prefix is
// needed; otherwise after 8 passes T is the k-th key itself and the remaining ties are
// taken in ascending index (the tie-break), found with a block-wide prefix count.  A second
// prefix count writes the selected chunks in ascending order.  No floating-point
// arithmetic is involved, so the result is exactly the oracle's.
#include "xkv_internal.cuh"

namespace xkv {
namespace {

constexpr int SEL_THREADS = 1024;
constexpr int SEL_WARPS = SEL_THREADS / 32;

// Exclusive prefix sum of one value per thread over the CTA; also returns the total.
__device__ __forceinline__ unsigned block_exclusive_scan(unsigned v, unsigned *warp_tot,
                                                         unsigned *total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    unsigned inc = v;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        unsigned t = __shfl_up_sync(0xffffffffu, inc, off);
        if (lane >= off) inc += t;
    }
    if (lane == 31) warp_tot[warp] = inc;
    __syncthreads();
    if (warp == 0) {
        unsigned w = lane < SEL_WARPS ? warp_tot[lane] : 0u;
        unsigned winc = w;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            unsigned t = __shfl_up_sync(0xffffffffu, winc, off);
            if (lane >= off) winc += t;
        }
        if (lane < SEL_WARPS) warp_tot[lane] = winc - w;  // exclusive warp offsets
        if (lane == 31) *total = winc;
    }
    __syncthreads();
    const unsigned r = warp_tot[warp] + inc - v;
    __syncthreads();  // warp_tot may be reused by the caller
    return r;
}

__global__ void __launch_bounds__(SEL_THREADS) k_select(const double *__restrict__ scores,
                                                        int32_t *__restrict__ sel, int64_t nC_,
                                                        int top_k, int n_sink, int n_recent,
                                                        int n_sel) {
    extern __shared__ unsigned long long keys[];  // [nC]
    __shared__ unsigned hist[2][256];             // passes alternate: one is zeroed while
                                                  // the other is scanned
    __shared__ unsigned warp_tot[SEL_WARPS];
    __shared__ unsigned s_total;
    __shared__ unsigned long long s_prefix, s_mask;
    __shared__ unsigned s_krem;
    __shared__ int s_done;

    grid_dep_wait();    // the scores come from the kernel before
    grid_dep_launch();
    const int nC = (int)nC_;
    const int unit = blockIdx.x;
    const double *s = scores + (size_t)unit * nC;
    auto forced = [&](int c) { return c < n_sink || c >= nC - n_recent; };

    // forced chunks: [0, n_sink) and [nC - n_recent, nC), which may overlap
    const int f_lo = min(n_sink, nC), f_hi = max(nC - n_recent, 0);
    const int n_forced = f_lo + (nC - f_hi) - max(0, f_lo - f_hi);
    const int n_cand = nC - n_forced;
    const int k_eff = min(top_k, n_cand);
    // 0: take no candidate, 1: take every candidate, 2: threshold select with ties ranked
    // by index, 3: threshold select whose whole last bin is taken
    int mode = k_eff == 0 ? 0 : (k_eff == n_cand ? 1 : 2);
    if (mode == 2) {
        if (threadIdx.x == 0) {
            s_prefix = 0ull;
            s_mask = 0ull;
            s_krem = (unsigned)k_eff;
            s_done = 0;
        }
        for (int i = threadIdx.x; i < 256; i += SEL_THREADS) hist[0][i] = 0u;
    }
    bool nan_seen = false;
    for (int c = threadIdx.x; c < nC; c += SEL_THREADS) {
        const double v = s[c];
        nan_seen |= isnan(v);
        keys[c] = order_key(v);
    }
    // a NaN score marks a failed scoring launch: the unit selects nothing (-1 entries),
    // which makes the attention call that consumes it fail with NaN outputs.  The same
    // barrier publishes the keys and the first pass's state.
    if (__syncthreads_or(nan_seen)) {
        for (int i = threadIdx.x; i < n_sel; i += SEL_THREADS)
            sel[(size_t)unit * n_sel + i] = -1;
        return;
    }
    unsigned long long T = 0, M = 0;
    unsigned krem = 0;
    if (mode == 2) {
        unsigned long long mask = 0ull;
        int buf = 0;
        for (int shift = 56; shift >= 0; shift -= 8, buf ^= 1) {
            const unsigned long long prefix = s_prefix;
            for (int c = threadIdx.x; c < nC; c += SEL_THREADS) {
                const unsigned long long k = keys[c];
                if (!forced(c) && (k & mask) == prefix)
                    atomicAdd(&hist[buf][(unsigned)(k >> shift) & 255u], 1u);
            }
            __syncthreads();
            if (threadIdx.x >= 32) {                   // the next pass's histogram
                for (int i = threadIdx.x - 32; i < 256; i += SEL_THREADS - 32) hist[buf ^ 1][i] = 0u;
            } else {
                const int lane = threadIdx.x;
                const unsigned need = s_krem;
                unsigned cnt[8], tot = 0;
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    cnt[i] = hist[buf][255 - (lane * 8 + i)];  // lanes walk the digits downwards
                    tot += cnt[i];
                }
                unsigned inc = tot;
#pragma unroll
                for (int off = 1; off < 32; off <<= 1) {
                    unsigned t = __shfl_up_sync(0xffffffffu, inc, off);
                    if (lane >= off) inc += t;
                }
                const unsigned exc = inc - tot;
                if (exc < need && need <= inc) {
                    unsigned cum = exc;
                    for (int i = 0; i < 8; ++i) {
                        if (cum + cnt[i] >= need) {
                            const unsigned long long D = (unsigned long long)(255 - (lane * 8 + i));
                            s_prefix = prefix | (D << shift);
                            s_mask = mask | (255ull << shift);
                            s_krem = need - cum;
                            s_done = cnt[i] == need - cum;  // the whole bin is needed
                            break;
                        }
                        cum += cnt[i];
                    }
                }
            }
            mask |= 255ull << shift;
            __syncthreads();
            if (s_done) break;                          // uniform: read after the barrier
        }
        T = s_prefix;
        M = s_mask;
        krem = s_krem;
        if (s_done) mode = 3;   // every candidate with the prefix is taken: no tie ranks
    }

    // Each thread owns a contiguous run of chunks so prefix counts follow chunk order.
    const int ipt = (nC + SEL_THREADS - 1) / SEL_THREADS;
    const int lo = min(nC, (int)threadIdx.x * ipt), hi = min(nC, lo + ipt);
    unsigned eq_rank = 0;
    if (mode == 2) {                            // uniform: only when ties must be ranked
        unsigned eq_local = 0;
        for (int c = lo; c < hi; ++c) eq_local += (!forced(c) && (keys[c] & M) == T) ? 1u : 0u;
        eq_rank = block_exclusive_scan(eq_local, warp_tot, &s_total);
    }

    // selection flags for the thread's run, as a bit mask (ipt <= 16)
    unsigned flags = 0, n_local = 0;
    for (int c = lo; c < hi; ++c) {
        bool take;
        if (forced(c)) {
            take = true;
        } else if (mode == 0) {
            take = false;
        } else if (mode == 1) {
            take = true;
        } else if (mode == 3) {
            take = (keys[c] & M) >= T;
        } else {
            const unsigned long long k = keys[c] & M;
            if (k > T) {
                take = true;
            } else if (k == T) {
                take = eq_rank < krem;
                ++eq_rank;
            } else {
                take = false;
            }
        }
        if (take) {
            flags |= 1u << (c - lo);
            ++n_local;
        }
    }
    unsigned pos = block_exclusive_scan(n_local, warp_tot, &s_total);
    int32_t *out = sel + (size_t)unit * n_sel;
    for (int c = lo; c < hi; ++c)
        if ((flags >> (c - lo)) & 1u) {
            if (pos < (unsigned)n_sel) out[pos] = c;
            ++pos;
        }
}

}  // namespace

cudaError_t launch_select(const xkv_dims &d, const double *scores, int top_k, int n_sink,
                          int n_recent, int32_t *sel, int n_sel, cudaStream_t s) {
    const int64_t nC = d.ctx_len / d.chunk;
    const size_t smem = (size_t)nC * sizeof(unsigned long long);
    set_smem_limit((const void *)k_select, smem);
    return launch_chained(k_select, dim3(d.batch * d.n_kv_heads), dim3(SEL_THREADS), smem, s,
                          scores, sel, nC, top_k, n_sink, n_recent, n_sel);
}

}  // namespace xkv
