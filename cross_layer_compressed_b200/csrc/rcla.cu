// R-CLA decode attention over a leader's KV cache (Stochastic KV Routing page: at
// inference a fixed set S of layers stores KV; a layer outside S reads the nearest
// previous leader's cache and skips its own K/V load and update, the page's
// Algorithm 2).  HBM-bound stream of K and V; CUDA cores.
//
// Grid (split, KV head, sequence), flash-decoding style: a CTA owns a contiguous range
// of rows.  Phase 1 stages K tiles of 128 rows in shared memory (coalesced 16-byte
// loads, XOR-swizzled 16-byte columns) and one thread per row forms the G logits.
// The range's max and sum are then exact.  Phase 2 stages V tiles the same way and
// thread j accumulates column j of the G outputs.  Partials (m, l, acc) per range go
// to the workspace; a combine kernel merges them.
//
// The leader's update: when `update_row` >= 0, the CTAs of split 0 copy k_new / v_new
// into that row of the cache, and every CTA reads that row from k_new / v_new (never
// from the cache), so no CTA depends on another's write.
#include "sm100_util.cuh"

namespace xkv {
namespace {

constexpr int RC_THREADS = 128;
constexpr int RC_TILE = 128;

template <typename T, int G>
__global__ void __launch_bounds__(RC_THREADS) k_rcla(
    T *__restrict__ K, T *__restrict__ V, const T *__restrict__ k_new,
    const T *__restrict__ v_new, const T *__restrict__ q, int slot, int Hq, int Hkv, int hd,
    int64_t L_max, int64_t n_rows, int64_t update_row, int64_t rows_per_split,
    float *__restrict__ partials) {
    constexpr int EPV = 16 / sizeof(T);
    extern __shared__ __align__(16) unsigned char smem[];
    const int split = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
    const int B = gridDim.z;
    const int vpr = hd / EPV;
    uint4 *tile = reinterpret_cast<uint4 *>(smem);                         // [RC_TILE][vpr]
    float *qs = reinterpret_cast<float *>(smem + (size_t)RC_TILE * hd * sizeof(T));  // [hd][G]
    float *stat = qs + hd * G;                                              // [2][G]
    float *z = stat + 2 * G;                                                // [rows][G]

    const size_t cache_off = (((size_t)slot * B + b) * Hkv + g) * (size_t)L_max * hd;
    const size_t new_off = ((size_t)b * Hkv + g) * hd;
    if (update_row >= 0 && split == 0) {
        for (int e = threadIdx.x; e < hd; e += RC_THREADS) {
            K[cache_off + (size_t)update_row * hd + e] = k_new[new_off + e];
            V[cache_off + (size_t)update_row * hd + e] = v_new[new_off + e];
        }
    }
    for (int e = threadIdx.x; e < G * hd; e += RC_THREADS) {
        const int h = e / hd, dd = e % hd;
        qs[dd * G + h] = Elem<T>::f32(q[((size_t)b * Hq + (size_t)g * G + h) * hd + dd]);
    }
    const int64_t r0 = (int64_t)split * rows_per_split;
    const int nr = (int)min64(rows_per_split, n_rows - r0);
    const float scale = 1.0f / sqrtf((float)hd);

    auto stage = [&](const T *cache, const T *newrow, int t0, int nt) {
        const uint4 *src = reinterpret_cast<const uint4 *>(cache + cache_off + (size_t)(r0 + t0) * hd);
        const uint4 *nsrc = reinterpret_cast<const uint4 *>(newrow + new_off);
        for (int e = threadIdx.x; e < nt * vpr; e += RC_THREADS) {
            const int r = e / vpr, v = e % vpr;
            const bool is_new = (r0 + t0 + r) == update_row;
            tile[r * vpr + (v ^ (r & 7))] = is_new ? nsrc[v] : src[e];  // plain loads: this kernel writes the cache
        }
    };

    // ---------------- phase 1: logits
    for (int t0 = 0; t0 < nr; t0 += RC_TILE) {
        const int nt = min(RC_TILE, nr - t0);
        __syncthreads();
        stage(K, k_new, t0, nt);
        __syncthreads();
        const int r = threadIdx.x;
        if (r < nt) {
            float acc[G];
#pragma unroll
            for (int h = 0; h < G; ++h) acc[h] = 0.f;
            for (int v = 0; v < vpr; ++v) {
                const uint4 w = tile[r * vpr + (v ^ (r & 7))];
                const T *e = reinterpret_cast<const T *>(&w);
#pragma unroll
                for (int k = 0; k < EPV; ++k) {
                    const float x = Elem<T>::f32(e[k]);
                    const float *qd = qs + (v * EPV + k) * G;
#pragma unroll
                    for (int h = 0; h < G; ++h) acc[h] = fmaf(x, qd[h], acc[h]);
                }
            }
#pragma unroll
            for (int h = 0; h < G; ++h) z[(t0 + r) * G + h] = acc[h] * scale;
        }
    }
    __syncthreads();

    // ---------------- softmax statistics of the range
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int h = warp; h < G; h += RC_THREADS / 32) {
        float m = -INFINITY;
        for (int r = lane; r < nr; r += 32) m = fmaxf(m, z[r * G + h]);
#pragma unroll
        for (int off = 16; off; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
        float l = 0.f;
        for (int r = lane; r < nr; r += 32) {
            const float p = expf(z[r * G + h] - m);
            z[r * G + h] = p;
            l += p;
        }
#pragma unroll
        for (int off = 16; off; off >>= 1) l += __shfl_xor_sync(0xffffffffu, l, off);
        if (lane == 0) {
            stat[h] = m;
            stat[G + h] = l;
        }
    }

    // ---------------- phase 2: p . V
    float o[G];
#pragma unroll
    for (int h = 0; h < G; ++h) o[h] = 0.f;
    const int j = threadIdx.x;
    const int jv = j / EPV, jk = j % EPV;
    for (int t0 = 0; t0 < nr; t0 += RC_TILE) {
        const int nt = min(RC_TILE, nr - t0);
        __syncthreads();
        stage(V, v_new, t0, nt);
        __syncthreads();
        if (j < hd) {
            for (int r = 0; r < nt; ++r) {
                const T *row = reinterpret_cast<const T *>(tile + r * vpr + (jv ^ (r & 7)));
                const float x = Elem<T>::f32(row[jk]);
#pragma unroll
                for (int h = 0; h < G; ++h) o[h] = fmaf(z[(t0 + r) * G + h], x, o[h]);
            }
        }
    }
    if (j < hd) {
        for (int h = 0; h < G; ++h) {
            float *dst = partials + (((size_t)split * B + b) * Hq + (size_t)g * G + h) * (hd + 2);
            dst[2 + j] = o[h];
            if (j == 0) {
                dst[0] = stat[h];
                dst[1] = stat[G + h];
            }
        }
    }
}

template <typename T, int G>
cudaError_t launch_g(const xkv_dims &d, int slot, int64_t L_max, int64_t n_rows,
                     int64_t update_row, void *K, void *V, const void *k_new,
                     const void *v_new, const void *q, const SplitPlan &plan, float *partials,
                     cudaStream_t s) {
    const size_t smem = (size_t)RC_TILE * d.head_dim * sizeof(T) +
                        sizeof(float) * ((size_t)d.head_dim * G + 2 * G +
                                         (size_t)plan.rows_per_split * G);
    auto k = k_rcla<T, G>;
    set_smem_limit((const void *)k, smem);
    dim3 grid(plan.n_split, d.n_kv_heads, d.batch);
    k<<<grid, RC_THREADS, smem, s>>>((T *)K, (T *)V, (const T *)k_new, (const T *)v_new,
                                     (const T *)q, slot, d.n_q_heads, d.n_kv_heads, d.head_dim,
                                     L_max, n_rows, update_row, plan.rows_per_split, partials);
    return cudaGetLastError();
}

template <typename T>
cudaError_t launch_t(const xkv_dims &d, int slot, int64_t L_max, int64_t n_rows,
                     int64_t update_row, void *K, void *V, const void *k_new,
                     const void *v_new, const void *q, const SplitPlan &plan, float *partials,
                     cudaStream_t s) {
    switch (d.n_q_heads / d.n_kv_heads) {
#define XKV_G(GG)                                                                            \
    case GG:                                                                                 \
        return launch_g<T, GG>(d, slot, L_max, n_rows, update_row, K, V, k_new, v_new, q,    \
                               plan, partials, s);
        XKV_G(1) XKV_G(2) XKV_G(3) XKV_G(4) XKV_G(5) XKV_G(6) XKV_G(7) XKV_G(8)
        XKV_G(9) XKV_G(10) XKV_G(11) XKV_G(12) XKV_G(13) XKV_G(14) XKV_G(15) XKV_G(16)
#undef XKV_G
        default: return cudaErrorInvalidValue;
    }
}

// ---------------------------------------------------------------- TMA-pipelined path
// bf16 caches, head_dim 128.  Persistent CTAs walk (unit, split) items; every item streams
// its key tiles, then its value tiles (256 rows x 256 B = two 128-byte-swizzled boxes)
// through three shared-memory stages.  Key phase: thread = row, G fp32 logits per row.
// Then the exact max / sum of the item's rows.  Value phase: four row streams of 64
// threads, each thread two columns, summed across streams at the end of the item.
constexpr int R3_ROWS = 256;
constexpr int R3_THREADS = 256;
constexpr int R3_STAGES = 3;
constexpr int R3_HALF = R3_ROWS * 128;
constexpr int R3_TILE = 2 * R3_HALF;             // 64 KB
constexpr uint32_t R3_SPIN = 1u << 24;

struct RclaParams {
    __nv_bfloat16 *K, *V;                        // caches (the update row is written here)
    const __nv_bfloat16 *k_new, *v_new, *q;
    float *partials;
    int slot, B, Hq, Hkv;
    int64_t L_max, n_rows, update_row;
    int rows_per_split, n_split, n_items;
    float qscale;                                // log2(e) / sqrt(hd)
    uint32_t stage_spin;                         // poll limit of the waits for staged data
};

template <int G>
__global__ void __launch_bounds__(R3_THREADS, 1)
    k_rcla_tma(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
               const RclaParams p) {
    extern __shared__ unsigned char smem_raw[];
    unsigned char *smem = (unsigned char *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    float *qs = reinterpret_cast<float *>(smem + R3_STAGES * R3_TILE);   // [128][G]
    float *z = qs + 128 * G;                                             // [rows_per_split][G]
    float *ob = z + (size_t)p.rows_per_split * G;                        // [4][G][128]
    uint64_t *full = reinterpret_cast<uint64_t *>(ob + 4 * G * 128);
    __shared__ float red[8][16];
    __shared__ int s_abort;
    const int t = threadIdx.x, warp = t >> 5, lane = t & 31;

    // load cursor (thread 0): loads are issued in consumption order, R3_STAGES ahead
    int l_item = blockIdx.x, l_phase = 0, l_tile = 0, n_loaded = 0;
    auto tiles_of = [&](int item) {
        const int split = item % p.n_split;
        const int64_t r0 = (int64_t)split * p.rows_per_split;
        const int64_t nr = min64(p.rows_per_split, p.n_rows - r0);
        return (int)((nr + R3_ROWS - 1) / R3_ROWS);
    };
    auto issue_next = [&]() {                    // thread 0 only
        if (l_item >= p.n_items) return;
        const int st = n_loaded % R3_STAGES;
        const int u = l_item / p.n_split, split = l_item % p.n_split;
        const int b = u / p.Hkv, g = u % p.Hkv;
        const int64_t row = (((int64_t)p.slot * p.B + b) * p.Hkv + g) * p.L_max +
                            (int64_t)split * p.rows_per_split + (int64_t)l_tile * R3_ROWS;
        const CUtensorMap *m = l_phase == 0 ? &tmK : &tmV;
        mbar_expect_tx(&full[st], (uint32_t)R3_TILE);
        tma_load_2d(m, &full[st], smem + st * R3_TILE, 0, (int)row);
        tma_load_2d(m, &full[st], smem + st * R3_TILE + R3_HALF, 64, (int)row);
        ++n_loaded;
        if (++l_tile == tiles_of(l_item)) {
            l_tile = 0;
            if (++l_phase == 2) {
                l_phase = 0;
                l_item += gridDim.x;
            }
        }
    };
    if (t == 0) {
        for (int st = 0; st < R3_STAGES; ++st) mbar_init(&full[st], 1);
        s_abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        prefetch_tmap(&tmK);
        prefetch_tmap(&tmV);
        for (int k = 0; k < R3_STAGES; ++k) issue_next();
    }
    __syncthreads();

    int n_used = 0;                                 // loads consumed so far
    auto wait_stage = [&](int &st) -> bool {   // CTA-uniform outcome
        st = n_used % R3_STAGES;
        const bool got = mbar_wait_bounded(&full[st], (uint32_t)((n_used / R3_STAGES) & 1),
                                           &s_abort, p.stage_spin);
        if (!got) s_abort = 1;
        return !__syncthreads_or(!got);
    };
    auto release_stage = [&]() {                    // every thread done with the stage
        ++n_used;
        __syncthreads();
        if (t == 0) issue_next();
    };

    bool ok = true;
    int item = blockIdx.x;
    for (; item < p.n_items && ok; item += gridDim.x) {
        const int u = item / p.n_split, split = item % p.n_split;
        const int b = u / p.Hkv, g = u % p.Hkv;
        const int64_t r0 = (int64_t)split * p.rows_per_split;
        const int nr = (int)min64(p.rows_per_split, p.n_rows - r0);
        const int tiles = (nr + R3_ROWS - 1) / R3_ROWS;
        const size_t new_off = ((size_t)b * p.Hkv + g) * 128;
        if (p.update_row >= 0 && split == 0 && t < 128) {   // the leader's update
            const size_t row = ((((size_t)p.slot * p.B + b) * p.Hkv + g) * p.L_max +
                                (size_t)p.update_row) * 128;
            p.K[row + t] = p.k_new[new_off + t];
            p.V[row + t] = p.v_new[new_off + t];
        }
        const __nv_bfloat16 *qg = p.q + ((size_t)b * p.Hq + (size_t)g * G) * 128;
        for (int e = t; e < G * 128; e += R3_THREADS)
            qs[(e % 128) * G + e / 128] = __bfloat162float(qg[e]) * p.qscale;
        __syncthreads();
        // ---------------- key phase: logits
        for (int tt = 0; tt < tiles && ok; ++tt) {
            int st;
            if (!wait_stage(st)) { ok = false; break; }
            const int r = tt * R3_ROWS + t;
            if (r < nr) {
                float acc[G];
#pragma unroll
                for (int h = 0; h < G; ++h) acc[h] = 0.f;
                const bool is_new = r0 + r == p.update_row;
                const unsigned char *base = smem + st * R3_TILE;
#pragma unroll 4
                for (int v = 0; v < 16; ++v) {
                    uint4 w4;
                    if (is_new)
                        w4 = reinterpret_cast<const uint4 *>(p.k_new + new_off)[v];
                    else
                        w4 = *reinterpret_cast<const uint4 *>(
                            base + (v >> 3) * R3_HALF + t * 128 + (((v & 7) ^ (t & 7)) << 4));
                    const uint32_t wv[4] = {w4.x, w4.y, w4.z, w4.w};
#pragma unroll
                    for (int k2 = 0; k2 < 4; ++k2) {
                        const float x0 = bf16lo(wv[k2]), x1 = bf16hi(wv[k2]);
                        const float *q0 = qs + (v * 8 + 2 * k2) * G;
#pragma unroll
                        for (int h = 0; h < G; ++h) {
                            acc[h] = fmaf(x0, q0[h], acc[h]);
                            acc[h] = fmaf(x1, q0[G + h], acc[h]);
                        }
                    }
                }
#pragma unroll
                for (int h = 0; h < G; ++h) z[(size_t)r * G + h] = acc[h];
            }
            release_stage();
        }
        if (!ok) break;
        // ---------------- exact max / sum of the item's rows (log2 domain)
        float m[G], l[G];
#pragma unroll
        for (int h = 0; h < G; ++h) m[h] = -INFINITY;
        for (int r = t; r < nr; r += R3_THREADS)
#pragma unroll
            for (int h = 0; h < G; ++h) m[h] = fmaxf(m[h], z[(size_t)r * G + h]);
#pragma unroll
        for (int h = 0; h < G; ++h) {
#pragma unroll
            for (int off = 16; off; off >>= 1)
                m[h] = fmaxf(m[h], __shfl_xor_sync(0xffffffffu, m[h], off));
            if (lane == 0) red[warp][h] = m[h];
        }
        __syncthreads();
#pragma unroll
        for (int h = 0; h < G; ++h) {
            float mm = red[0][h];
            for (int k2 = 1; k2 < 8; ++k2) mm = fmaxf(mm, red[k2][h]);
            m[h] = mm;
        }
        __syncthreads();
#pragma unroll
        for (int h = 0; h < G; ++h) l[h] = 0.f;
        for (int r = t; r < nr; r += R3_THREADS)
#pragma unroll
            for (int h = 0; h < G; ++h) {
                const float pv = exp2f(z[(size_t)r * G + h] - m[h]);
                z[(size_t)r * G + h] = pv;
                l[h] += pv;
            }
#pragma unroll
        for (int h = 0; h < G; ++h) {
#pragma unroll
            for (int off = 16; off; off >>= 1) l[h] += __shfl_xor_sync(0xffffffffu, l[h], off);
            if (lane == 0) red[warp][h] = l[h];
        }
        __syncthreads();
#pragma unroll
        for (int h = 0; h < G; ++h) {
            float ll = 0.f;
            for (int k2 = 0; k2 < 8; ++k2) ll += red[k2][h];
            l[h] = ll;
        }
        // ---------------- value phase: stream s = t / 64 takes rows s, s+4, ...; columns
        // 2c, 2c+1 with c = t % 64
        const int sidx = t >> 6, c = t & 63;
        float o0[G], o1[G];
#pragma unroll
        for (int h = 0; h < G; ++h) o0[h] = o1[h] = 0.f;
        const uint32_t new_pair =
            p.update_row >= 0 ? reinterpret_cast<const uint32_t *>(p.v_new + new_off)[c] : 0u;
        for (int tt = 0; tt < tiles && ok; ++tt) {
            int st;
            if (!wait_stage(st)) { ok = false; break; }
            const unsigned char *base = smem + st * R3_TILE;
            const int rmax = min(R3_ROWS, nr - tt * R3_ROWS);
            // column pair c lives in box c / 32, 16-byte column (c % 32) / 4, word c % 4
            const int box = c >> 5, col16 = (c & 31) >> 2, word = c & 3;
            for (int rr = sidx; rr < rmax; rr += 4) {
                const int r = tt * R3_ROWS + rr;
                uint32_t pair;
                if (r0 + r == p.update_row)
                    pair = new_pair;
                else
                    pair = *reinterpret_cast<const uint32_t *>(
                        base + box * R3_HALF + rr * 128 + ((col16 ^ (rr & 7)) << 4) + word * 4);
                const float v0 = bf16lo(pair), v1 = bf16hi(pair);
                const float *pz = z + (size_t)r * G;
#pragma unroll
                for (int h = 0; h < G; ++h) {
                    o0[h] = fmaf(pz[h], v0, o0[h]);
                    o1[h] = fmaf(pz[h], v1, o1[h]);
                }
            }
            release_stage();
        }
        if (!ok) break;
#pragma unroll
        for (int h = 0; h < G; ++h) {
            ob[(sidx * G + h) * 128 + 2 * c] = o0[h];
            ob[(sidx * G + h) * 128 + 2 * c + 1] = o1[h];
        }
        __syncthreads();
        if (t < 128) {
            float *dst = p.partials + (((size_t)split * p.B + b) * p.Hq + (size_t)g * G) * 130;
#pragma unroll
            for (int h = 0; h < G; ++h) {
                const float sum = (ob[(0 * G + h) * 128 + t] + ob[(1 * G + h) * 128 + t]) +
                                  (ob[(2 * G + h) * 128 + t] + ob[(3 * G + h) * 128 + t]);
                dst[h * 130 + 2 + t] = sum;
                if (t == 0) {
                    dst[h * 130] = m[h] * 0.6931471805599453f;   // natural log
                    dst[h * 130 + 1] = l[h];
                }
            }
        }
        __syncthreads();                          // ob, z and qs are reused by the next item
    }
    if (!ok) {
        // A bounded wait gave up.  Poison the partials of every item this CTA still owed
        // (NaN running max, so the combine writes NaN outputs), then let this CTA's own
        // copies land (bounded) before it exits.
        for (int it2 = item; it2 < p.n_items; it2 += gridDim.x) {
            const int u = it2 / p.n_split, split = it2 % p.n_split;
            const int b = u / p.Hkv, g = u % p.Hkv;
            if (t < G)
                p.partials[(((size_t)split * p.B + b) * p.Hq + (size_t)g * G + t) * 130] =
                    __int_as_float(0x7fc00000);
        }
        if (t == 0) {   // the last R3_STAGES loads issued complete their phase
            for (int j = n_loaded - R3_STAGES > 0 ? n_loaded - R3_STAGES : 0; j < n_loaded; ++j)
                for (uint32_t k = 0; k < R3_SPIN; ++k)
                    if (mbar_test(&full[j % R3_STAGES], (uint32_t)(j / R3_STAGES) & 1)) break;
        }
    }
}

template <int G>
cudaError_t launch_rcla_tma_g(const xkv_dims &d, int slot, int64_t L_max, int64_t n_rows,
                              int64_t update_row, void *K, void *V, const void *k_new,
                              const void *v_new, const void *q, const SplitPlan &plan,
                              float *partials, cudaStream_t s) {
    const uint64_t rows = (uint64_t)(slot + 1) * d.batch * d.n_kv_heads * (uint64_t)L_max;
    CUtensorMap tm[2];
    if (!make_map_bf16_sw128(&tm[0], K, rows, 128, R3_ROWS) ||
        !make_map_bf16_sw128(&tm[1], V, rows, 128, R3_ROWS))
        return cudaErrorInvalidValue;
    RclaParams p;
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
    p.qscale = 1.4426950408889634f / sqrtf(128.f);
    // XKV_TEST_MMA_SPIN (tests only, read on every call): a shorter poll limit for the
    // waits on staged data, so a test can make them give up; the drain keeps its bound
    p.stage_spin = test_poll_limit("XKV_TEST_MMA_SPIN", R3_SPIN);
    const size_t smem = 1024 + (size_t)R3_STAGES * R3_TILE +
                        sizeof(float) * (128 * G + (size_t)plan.rows_per_split * G + 4 * G * 128) +
                        R3_STAGES * sizeof(uint64_t);
    auto k = k_rcla_tma<G>;
    cudaError_t e = set_smem_limit((const void *)k, smem);
    if (e != cudaSuccess) return e;
    const int grid = p.n_items < sm_count() ? p.n_items : sm_count();
    k<<<grid, R3_THREADS, smem, s>>>(tm[0], tm[1], p);
    return cudaGetLastError();
}

}  // namespace

bool rcla_tma_ok(const xkv_dims &d, int slot, int64_t L_max, const SplitPlan &plan) {
    const int G = d.n_q_heads / d.n_kv_heads;
    const int64_t rows = (int64_t)(slot + 1) * d.batch * d.n_kv_heads * L_max;
    return d.dtype == XKV_BF16 && d.head_dim == 128 && (G == 1 || G == 2 || G == 4 ||
           G == 5 || G == 8) && (int64_t)plan.rows_per_split * G <= 4096 &&
           rows + R3_ROWS < ((int64_t)1 << 31) &&
           tma_available() && !env_flag(ENV_FORCE_SIMT);
}

cudaError_t launch_rcla(const xkv_dims &d, int slot, int64_t L_max, int64_t n_rows,
                        int64_t update_row, void *K, void *V, const void *k_new,
                        const void *v_new, const void *q, const SplitPlan &plan,
                        float *partials, cudaStream_t s) {
    if (rcla_tc_ok(d, slot, L_max, plan))
        return launch_rcla_tc(d, slot, L_max, n_rows, update_row, K, V, k_new, v_new, q, plan,
                              partials, s);
    if (rcla_tma_ok(d, slot, L_max, plan)) {
        switch (d.n_q_heads / d.n_kv_heads) {
#define XKV_R(GG)                                                                             \
    case GG:                                                                                  \
        return launch_rcla_tma_g<GG>(d, slot, L_max, n_rows, update_row, K, V, k_new, v_new, \
                                     q, plan, partials, s);
            XKV_R(1) XKV_R(2) XKV_R(4) XKV_R(5) XKV_R(8)
#undef XKV_R
        }
    }
    return d.dtype == XKV_F32
               ? launch_t<float>(d, slot, L_max, n_rows, update_row, K, V, k_new, v_new, q,
                                 plan, partials, s)
               : launch_t<__nv_bfloat16>(d, slot, L_max, n_rows, update_row, K, V, k_new,
                                         v_new, q, plan, partials, s);
}

}  // namespace xkv
