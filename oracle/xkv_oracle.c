/*
 * CPU oracle for decode attention over a cross-layer-compressed KV cache.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the plain, slow, scalar fp64 statement of
 * what the library computes.  Only the tests, the smoke check and the CPU-baseline
 * leg of the benchmark load it.  It shares no code, header, table or helper with the
 * CUDA library, and the library never calls it.
 *
 * Sources (cited by page title and section):
 *  [xKV]   "xKV: Cross-Layer KV-Cache Compression via Aligned Singular Vector
 *          Extraction" (technical summary page).  Section 2.2, cross-layer
 *          factorization: a window's caches concatenated, truncated SVD, a shared token
 *          basis A and per-layer reconstruction matrices B_l, storage
 *          O(L*r + W*r*d).  Section 2.3, selective reconstruction: landmark-based
 *          chunk selection, then only the selected rows are rebuilt from A and B_l.
 *          Section 4: dense reconstruction mode.
 *  [VASE]  "Value-Aware Stochastic KV cache Eviction" technical summary page.  Section
 *          2.A: the N_v tokens whose value vector has the largest range max(v) - min(v)
 *          are always kept.
 *  [R-CLA] "Stochastic KV Routing: adaptive depth-wise cache sharing" page.  Inference
 *          uses a fixed sharing set S; a layer outside S reuses the nearest previous
 *          cached layer's KV and skips its own K/V load and update (its Algorithm 2).
 *
 * Readings where the pages are silent (each is listed in the design notes):
 *  - two bases per window, A^K (L x r_K) and A^V (L x r_V); factors per sequence;
 *  - B_l is stored column-major (element (i, j) of the r x d_kv matrix at j*r + i);
 *  - query head h belongs to KV group g = h / G, G = Hq / Hkv;
 *  - landmark of chunk c = mean of the chunk's C reconstructed key rows, rounded
 *    to nearest-even into the storage type;
 *  - landmark score = unscaled dot product lm . q_h summed in fp64 in order
 *    d = 0 .. hd-1 (every product is exact in fp64), max over the group's heads
 *    under the total order in which -0 < +0;
 *  - selection: forced = sink chunks {0..n_sink-1} and recent chunks
 *    {nC-n_recent..nC-1}; the top-k of the remaining chunks by (score descending,
 *    index ascending); the union sorted ascending;
 *  - attention: z = (q . K_hat) / sqrt(hd), softmax over the selected rows,
 *    o = sum p * V_hat; no mask, no positional rotation (the factors represent the
 *    keys as attended);
 *  - value-range reservation (after the VASE page, section 2.A, applied to chunks): a
 *    chunk's statistic is the largest max(v) - min(v) over the reconstructed value rows
 *    of its tokens (one KV head's slice); the n_value largest chunks outside the sink
 *    and recent windows are kept whatever the scores, in addition to the top-k;
 *  - R-CLA: lead(l) = max{s in S : s <= l}; the cache slot of a leader is its rank
 *    in S; a leader call with a new row writes it at row len and attends len+1 rows;
 *    any other call attends the len rows present.
 *
 * Storage types: 0 = fp32, 1 = bf16 (bit pattern = high 16 bits of an fp32).
 * Every function returns 0 on success and a negative value on a rejected argument.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORA_F32 0
#define ORA_BF16 1

/* ---------------------------------------------------------------- scalar helpers */

static double ora_load(const void *base, int dtype, int64_t i)
{
    if (dtype == ORA_F32)
        return (double)((const float *)base)[i];
    uint32_t bits = (uint32_t)((const uint16_t *)base)[i] << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return (double)f; /* exact: bf16 -> fp32 -> fp64 widen without rounding */
}

/* Round an fp64 value to nearest-even bf16 in one step (no intermediate fp32). */
static uint16_t ora_round_bf16(double x)
{
    if (x == 0.0 || isnan(x) || isinf(x)) {
        float f = (float)x;
        uint32_t b;
        memcpy(&b, &f, sizeof b);
        return (uint16_t)(b >> 16);
    }
    int e;
    (void)frexp(x, &e);              /* x = m * 2^e, 0.5 <= |m| < 1 */
    int quantum = e - 8;             /* bf16 keeps 8 significant bits */
    if (quantum < -133)              /* below the normal range: fixed subnormal quantum */
        quantum = -133;
    double k = nearbyint(ldexp(x, -quantum)); /* default rounding: nearest-even */
    double r = ldexp(k, quantum);
    float f = (float)r;              /* exact: r has at most 8 significant bits */
    if (fabs(r) > 3.3895313892515355e38)
        f = (float)(x > 0 ? INFINITY : -INFINITY);
    uint32_t b;
    memcpy(&b, &f, sizeof b);
    return (uint16_t)(b >> 16);
}

static void ora_store(void *base, int dtype, int64_t i, double x)
{
    if (dtype == ORA_F32)
        ((float *)base)[i] = (float)x; /* C's double -> float conversion: nearest-even */
    else
        ((uint16_t *)base)[i] = ora_round_bf16(x);
}

uint16_t oracle_round_bf16(double x) { return ora_round_bf16(x); }

/* Key under which a larger score compares larger, with -0 below +0. */
static uint64_t ora_order_key(double s)
{
    uint64_t u;
    memcpy(&u, &s, sizeof u);
    return (u >> 63) ? ~u : (u | 0x8000000000000000ull);
}

/* ------------------------------------------------------ [xKV] 2.2 reconstruction */

/*
 * One reconstructed row, restricted to KV head g:
 *   out[j] = sum_{i < r} A[t][i] * B[i][g*hd + j],   j < hd,
 * with A one sequence's basis (L x r, row-major) and B stored column-major
 * (Bt[(g*hd + j) * r + i]).  fp64, i ascending.
 */
static void ora_recon_row(const void *A, const void *Bt, int dtype, int64_t t, int r,
                          int g, int hd, double *out)
{
    for (int j = 0; j < hd; ++j) {
        double acc = 0.0;
        int64_t col = (int64_t)(g * hd + j) * r;
        for (int i = 0; i < r; ++i)
            acc += ora_load(A, dtype, t * r + i) * ora_load(Bt, dtype, col + i);
        out[j] = acc;
    }
}

/* Rows [t0, t0+n) of A * B_l over all d_kv columns, for tests of the factorization. */
int oracle_reconstruct_rows(int d_kv, int r, int dtype, const void *A, const void *Bt,
                            int64_t t0, int64_t n, double *out /* [n][d_kv] */)
{
    if (!A || !Bt || !out || d_kv <= 0 || r <= 0 || n < 0)
        return -1;
    for (int64_t t = 0; t < n; ++t)
        ora_recon_row(A, Bt, dtype, t0 + t, r, 0, d_kv, out + t * d_kv);
    return 0;
}

/* ------------------------------------------------- landmarks (built once per cache) */

/*
 * lm[b][g][c][j] = round( (1/C) * sum_{t in chunk c} K_hat[t][g*hd + j] )
 * One sequence's basis is Ak + b*L*rk, its matrix Bkt + b*d_kv*rk.
 */
int oracle_build_landmarks(int B, int Hkv, int hd, int64_t L, int C, int rk, int dtype,
                           const void *Ak, const void *Bkt, void *lm)
{
    if (!Ak || !Bkt || !lm || B <= 0 || Hkv <= 0 || hd <= 0 || C <= 0 || rk <= 0 || L % C)
        return -1;
    int64_t nC = L / C, d_kv = (int64_t)Hkv * hd;
    double *row = malloc(sizeof(double) * hd), *mean = malloc(sizeof(double) * hd);
    if (!row || !mean) {
        free(row);
        free(mean);
        return -2;
    }
    size_t esz = dtype == ORA_F32 ? 4 : 2;
    for (int b = 0; b < B; ++b) {
        const char *A = (const char *)Ak + (size_t)b * L * rk * esz;
        const char *Bt = (const char *)Bkt + (size_t)b * d_kv * rk * esz;
        for (int g = 0; g < Hkv; ++g)
            for (int64_t c = 0; c < nC; ++c) {
                for (int j = 0; j < hd; ++j)
                    mean[j] = 0.0;
                for (int u = 0; u < C; ++u) {
                    ora_recon_row(A, Bt, dtype, c * C + u, rk, g, hd, row);
                    for (int j = 0; j < hd; ++j)
                        mean[j] += row[j];
                }
                int64_t o = (((int64_t)b * Hkv + g) * nC + c) * hd;
                for (int j = 0; j < hd; ++j)
                    ora_store(lm, dtype, o + j, mean[j] / C);
            }
    }
    free(row);
    free(mean);
    return 0;
}

/* ------------------------------------------------------ [xKV] 2.3 landmark scoring */

/*
 * scores[b][g][c] = max_{h in group g} sum_{d < hd} lm[b][g][c][d] * q[b][h][d]
 * The sum runs in fp64 in order d = 0..hd-1; each product is exact in fp64.
 */
int oracle_score_landmarks(int B, int Hq, int Hkv, int hd, int64_t nC, int dtype,
                           const void *lm, const void *q, double *scores)
{
    if (!lm || !q || !scores || B <= 0 || Hkv <= 0 || Hq % Hkv || hd <= 0 || nC < 0)
        return -1;
    int G = Hq / Hkv;
    for (int b = 0; b < B; ++b)
        for (int g = 0; g < Hkv; ++g)
            for (int64_t c = 0; c < nC; ++c) {
                int64_t lo = (((int64_t)b * Hkv + g) * nC + c) * hd;
                double best = 0.0;
                for (int hh = 0; hh < G; ++hh) {
                    int64_t qo = ((int64_t)b * Hq + g * G + hh) * hd;
                    double acc = 0.0;
                    for (int d = 0; d < hd; ++d)
                        acc = acc + ora_load(lm, dtype, lo + d) * ora_load(q, dtype, qo + d);
                    if (hh == 0 || ora_order_key(acc) > ora_order_key(best))
                        best = acc;
                }
                scores[((int64_t)b * Hkv + g) * nC + c] = best;
            }
    return 0;
}

/* ------------------------------------------------------ [xKV] 2.3 chunk selection */

typedef struct {
    uint64_t key;
    int32_t idx;
} ora_cand;

static int ora_cmp_rank(const void *pa, const void *pb)
{
    const ora_cand *a = pa, *b = pb;
    if (a->key != b->key)
        return a->key > b->key ? -1 : 1; /* score descending */
    return a->idx < b->idx ? -1 : (a->idx > b->idx); /* then index ascending */
}

static int ora_cmp_int(const void *pa, const void *pb)
{
    int32_t a = *(const int32_t *)pa, b = *(const int32_t *)pb;
    return a < b ? -1 : (a > b);
}

/* Number of chunks selected per (sequence, KV head). */
int64_t oracle_n_selected(int64_t nC, int top_k, int n_sink, int n_recent)
{
    if (nC < 0 || top_k < 0 || n_sink < 0 || n_recent < 0)
        return -1;
    int64_t forced = 0;
    for (int64_t c = 0; c < nC; ++c)
        forced += (c < n_sink) || (c >= nC - n_recent);
    int64_t cand = nC - forced;
    return (top_k < cand ? top_k : cand) + forced;
}

/*
 * sel[b][g][0..n_sel) = ascending union of the forced chunks and the top_k remaining
 * chunks under (score descending, index ascending).
 */
int oracle_select_chunks(int B, int Hkv, int64_t nC, const double *scores, int top_k,
                         int n_sink, int n_recent, int32_t *sel, int64_t *n_sel_out)
{
    int64_t n_sel = oracle_n_selected(nC, top_k, n_sink, n_recent);
    if (!scores || !sel || B <= 0 || Hkv <= 0 || n_sel < 0)
        return -1;
    ora_cand *cand = malloc(sizeof(ora_cand) * (nC ? nC : 1));
    int32_t *pick = malloc(sizeof(int32_t) * (nC ? nC : 1));
    if (!cand || !pick) {
        free(cand);
        free(pick);
        return -2;
    }
    for (int b = 0; b < B; ++b)
        for (int g = 0; g < Hkv; ++g) {
            const double *s = scores + ((int64_t)b * Hkv + g) * nC;
            int64_t nc = 0, np = 0;
            for (int64_t c = 0; c < nC; ++c) {
                int forced = (c < n_sink) || (c >= nC - n_recent);
                if (forced) {
                    pick[np++] = (int32_t)c;
                } else {
                    cand[nc].key = ora_order_key(s[c]);
                    cand[nc].idx = (int32_t)c;
                    ++nc;
                }
            }
            qsort(cand, nc, sizeof(ora_cand), ora_cmp_rank);
            for (int64_t i = 0; i < nc && i < top_k; ++i)
                pick[np++] = cand[i].idx;
            qsort(pick, np, sizeof(int32_t), ora_cmp_int);
            memcpy(sel + ((int64_t)b * Hkv + g) * n_sel, pick, sizeof(int32_t) * np);
        }
    free(cand);
    free(pick);
    if (n_sel_out)
        *n_sel_out = n_sel;
    return 0;
}

/* ------------------------- [VASE] 2.A value-range reservation, applied to the chunks */

/*
 * The VASE page keeps, whatever the scores, the N_v tokens whose value vector has the
 * largest range Range(v) = max(v) - min(v).  Applied to this path's chunk selection:
 *   rho[b][g][c] = max over the C rows t of chunk c of Range(V_hat[t][g*hd .. g*hd+hd-1]),
 * V_hat = A^V B^V_l reconstructed exactly in fp64 (one KV head's slice of each row).
 */
int oracle_value_ranges(int B, int Hkv, int hd, int64_t L, int C, int rv, int dtype,
                        const void *Av, const void *Bvt, double *rho)
{
    if (B <= 0 || Hkv <= 0 || hd <= 0 || L <= 0 || C <= 0 || L % C || rv <= 0 || !Av ||
        !Bvt || !rho)
        return -1;
    const int64_t nC = L / C, d_kv = (int64_t)Hkv * hd, es = dtype == 1 ? 2 : 4;
    double *v = malloc(sizeof(double) * hd);
    if (!v)
        return -2;
    for (int b = 0; b < B; ++b) {
        const char *A = (const char *)Av + (size_t)b * L * rv * es;
        const char *Bt = (const char *)Bvt + (size_t)b * d_kv * rv * es;
        for (int g = 0; g < Hkv; ++g)
            for (int64_t c = 0; c < nC; ++c) {
                double best = 0.0;
                for (int64_t t = c * C; t < (c + 1) * C; ++t) {
                    ora_recon_row(A, Bt, dtype, t, rv, g, hd, v);
                    double lo = v[0], hi = v[0];
                    for (int j = 1; j < hd; ++j) {
                        if (v[j] < lo) lo = v[j];
                        if (v[j] > hi) hi = v[j];
                    }
                    if (hi - lo > best)
                        best = hi - lo;
                }
                rho[((int64_t)b * Hkv + g) * nC + c] = best;
            }
    }
    free(v);
    return 0;
}

/* Chunks reserved per (sequence, KV head): min(n_value, chunks outside sink and recent). */
int64_t oracle_n_reserved(int64_t nC, int n_value, int n_sink, int n_recent)
{
    int64_t base = oracle_n_selected(nC, 0, n_sink, n_recent);
    if (base < 0 || n_value < 0)
        return -1;
    int64_t cand = nC - base;
    return n_value < cand ? n_value : cand;
}

/*
 * reserved[b][g][0..n_res) = the n_res chunks outside the sink and recent windows with
 * the largest rho under (rho descending, index ascending), written in ascending order.
 */
int oracle_reserve_value_chunks(int B, int Hkv, int64_t nC, const double *rho, int n_value,
                                int n_sink, int n_recent, int32_t *reserved,
                                int64_t *n_res_out)
{
    int64_t n_res = oracle_n_reserved(nC, n_value, n_sink, n_recent);
    if (!rho || B <= 0 || Hkv <= 0 || n_res < 0 || (n_res > 0 && !reserved))
        return -1;
    ora_cand *cand = malloc(sizeof(ora_cand) * (nC ? nC : 1));
    int32_t *pick = malloc(sizeof(int32_t) * (nC ? nC : 1));
    if (!cand || !pick) {
        free(cand);
        free(pick);
        return -2;
    }
    for (int b = 0; b < B; ++b)
        for (int g = 0; g < Hkv; ++g) {
            const double *r = rho + ((int64_t)b * Hkv + g) * nC;
            int64_t nc = 0;
            for (int64_t c = 0; c < nC; ++c) {
                if ((c < n_sink) || (c >= nC - n_recent))
                    continue;
                cand[nc].key = ora_order_key(r[c]);
                cand[nc].idx = (int32_t)c;
                ++nc;
            }
            qsort(cand, nc, sizeof(ora_cand), ora_cmp_rank);
            for (int64_t i = 0; i < n_res; ++i)
                pick[i] = cand[i].idx;
            qsort(pick, n_res, sizeof(int32_t), ora_cmp_int);
            if (n_res)
                memcpy(reserved + ((int64_t)b * Hkv + g) * n_res, pick, sizeof(int32_t) * n_res);
        }
    free(cand);
    free(pick);
    if (n_res_out)
        *n_res_out = n_res;
    return 0;
}

/*
 * Selection with value-reserved chunks: the forced chunks are the sink and recent
 * windows plus reserved[b][g][0..n_res) (chunks outside those windows, no repeats);
 * then the top_k of the other chunks under (score descending, index ascending); the
 * union sorted ascending.  n_sel = |sink U recent| + n_res + min(top_k, rest).
 */
int oracle_select_chunks_reserved(int B, int Hkv, int64_t nC, const double *scores,
                                  const int32_t *reserved, int n_res, int top_k, int n_sink,
                                  int n_recent, int32_t *sel, int64_t *n_sel_out)
{
    int64_t base = oracle_n_selected(nC, 0, n_sink, n_recent);
    if (!scores || !sel || B <= 0 || Hkv <= 0 || base < 0 || n_res < 0 || top_k < 0 ||
        (n_res > 0 && !reserved) || n_res > nC - base)
        return -1;
    const int64_t rest = nC - base - n_res;
    const int64_t n_sel = base + n_res + (top_k < rest ? top_k : rest);
    ora_cand *cand = malloc(sizeof(ora_cand) * (nC ? nC : 1));
    int32_t *pick = malloc(sizeof(int32_t) * (nC ? nC : 1));
    unsigned char *held = calloc(nC ? nC : 1, 1);
    if (!cand || !pick || !held) {
        free(cand);
        free(pick);
        free(held);
        return -2;
    }
    for (int b = 0; b < B; ++b)
        for (int g = 0; g < Hkv; ++g) {
            const double *s = scores + ((int64_t)b * Hkv + g) * nC;
            const int32_t *res = reserved ? reserved + ((int64_t)b * Hkv + g) * n_res : NULL;
            memset(held, 0, nC);
            for (int i = 0; i < n_res; ++i) {
                int32_t c = res[i];
                if (c < 0 || c >= nC || held[c] || c < n_sink || c >= nC - n_recent) {
                    free(cand);
                    free(pick);
                    free(held);
                    return -3;       /* a reserved chunk must be a distinct candidate */
                }
                held[c] = 1;
            }
            int64_t nc = 0, np = 0;
            for (int64_t c = 0; c < nC; ++c) {
                if ((c < n_sink) || (c >= nC - n_recent) || held[c]) {
                    pick[np++] = (int32_t)c;
                } else {
                    cand[nc].key = ora_order_key(s[c]);
                    cand[nc].idx = (int32_t)c;
                    ++nc;
                }
            }
            qsort(cand, nc, sizeof(ora_cand), ora_cmp_rank);
            for (int64_t i = 0; i < nc && i < top_k; ++i)
                pick[np++] = cand[i].idx;
            qsort(pick, np, sizeof(int32_t), ora_cmp_int);
            memcpy(sel + ((int64_t)b * Hkv + g) * n_sel, pick, sizeof(int32_t) * np);
        }
    free(cand);
    free(pick);
    free(held);
    if (n_sel_out)
        *n_sel_out = n_sel;
    return 0;
}

/* --------------------------------- [xKV] 2.3 + section 4: reconstruct, then attend */

/*
 * One (sequence b, KV head g) unit.  Rows T = the C rows of each chunk in sel_bg
 * (ascending), or all L rows when sel_bg is NULL (dense reconstruction).
 * For each head h of the group: z_t = (q_h . K_hat[t]) / sqrt(hd);
 * p_t = exp(z_t - max z) / sum; out_h = sum_t p_t * V_hat[t].
 */
int oracle_attend_unit(int b, int g, int B, int Hq, int Hkv, int hd, int64_t L, int C,
                       int rk, int rv, int dtype, const void *Ak, const void *Av,
                       const void *Bkt, const void *Bvt, const void *q,
                       const int32_t *sel_bg, int64_t n_sel, float *out)
{
    if (!Ak || !Av || !Bkt || !Bvt || !q || !out || B <= 0 || Hkv <= 0 || Hq % Hkv ||
        C <= 0 || L % C || b < 0 || b >= B || g < 0 || g >= Hkv)
        return -1;
    int G = Hq / Hkv;
    int64_t nC = L / C, d_kv = (int64_t)Hkv * hd;
    int64_t nT = sel_bg ? n_sel * C : L;
    if (nT <= 0)
        return -1;
    size_t esz = dtype == ORA_F32 ? 4 : 2;
    const char *ak = (const char *)Ak + (size_t)b * L * rk * esz;
    const char *av = (const char *)Av + (size_t)b * L * rv * esz;
    const char *bk = (const char *)Bkt + (size_t)b * d_kv * rk * esz;
    const char *bv = (const char *)Bvt + (size_t)b * d_kv * rv * esz;
    double *z = malloc(sizeof(double) * nT * G);
    double *row = malloc(sizeof(double) * hd);
    double *acc = calloc((size_t)G * hd, sizeof(double));
    double *qd = malloc(sizeof(double) * G * hd);
    if (!z || !row || !acc || !qd) {
        free(z); free(row); free(acc); free(qd);
        return -2;
    }
    for (int hh = 0; hh < G; ++hh)
        for (int d = 0; d < hd; ++d)
            qd[hh * hd + d] = ora_load(q, dtype, ((int64_t)b * Hq + g * G + hh) * hd + d);
    double scale = 1.0 / sqrt((double)hd);
    int rc = 0;
    /* pass 1: logits over the reconstructed keys */
    for (int64_t i = 0; i < nT; ++i) {
        int64_t t;
        if (sel_bg) {
            int64_t c = sel_bg[i / C];
            if (c < 0 || c >= nC) {
                rc = -1;
                goto done;
            }
            t = c * C + i % C;
        } else {
            t = i;
        }
        ora_recon_row(ak, bk, dtype, t, rk, g, hd, row);
        for (int hh = 0; hh < G; ++hh) {
            double s = 0.0;
            for (int d = 0; d < hd; ++d)
                s += qd[hh * hd + d] * row[d];
            z[i * G + hh] = s * scale;
        }
    }
    /* softmax weights, then pass 2: weighted sum of the reconstructed values */
    for (int hh = 0; hh < G; ++hh) {
        double m = -INFINITY, l = 0.0;
        for (int64_t i = 0; i < nT; ++i)
            if (z[i * G + hh] > m)
                m = z[i * G + hh];
        for (int64_t i = 0; i < nT; ++i) {
            z[i * G + hh] = exp(z[i * G + hh] - m);
            l += z[i * G + hh];
        }
        for (int64_t i = 0; i < nT; ++i)
            z[i * G + hh] /= l;
    }
    for (int64_t i = 0; i < nT; ++i) {
        int64_t t = sel_bg ? (int64_t)sel_bg[i / C] * C + i % C : i;
        ora_recon_row(av, bv, dtype, t, rv, g, hd, row);
        for (int hh = 0; hh < G; ++hh)
            for (int d = 0; d < hd; ++d)
                acc[hh * hd + d] += z[i * G + hh] * row[d];
    }
    for (int hh = 0; hh < G; ++hh)
        for (int d = 0; d < hd; ++d)
            out[((int64_t)b * Hq + g * G + hh) * hd + d] = (float)acc[hh * hd + d];
done:
    free(z); free(row); free(acc); free(qd);
    return rc;
}

/* All units; sel is [B][Hkv][n_sel] or NULL for dense reconstruction. */
int oracle_reconstruct_attend(int B, int Hq, int Hkv, int hd, int64_t L, int C, int rk,
                              int rv, int dtype, const void *Ak, const void *Av,
                              const void *Bkt, const void *Bvt, const void *q,
                              const int32_t *sel, int64_t n_sel, float *out)
{
    if (B <= 0 || Hkv <= 0)
        return -1;
    for (int b = 0; b < B; ++b)
        for (int g = 0; g < Hkv; ++g) {
            const int32_t *s = sel ? sel + ((int64_t)b * Hkv + g) * n_sel : NULL;
            int rc = oracle_attend_unit(b, g, B, Hq, Hkv, hd, L, C, rk, rv, dtype, Ak, Av,
                                        Bkt, Bvt, q, s, n_sel, out);
            if (rc)
                return rc;
        }
    return 0;
}

/*
 * One (sequence b, KV head g) unit attending the reconstructed rows T (as in
 * oracle_attend_unit) followed by n_tail uncompressed rows of a tail buffer (tokens
 * generated after the cache was compressed), Kt/Vt [B][Hkv][T_max][hd] in the storage
 * type.  The pages are silent on generated tokens; the reading taken: they are kept
 * as they are and always attended, in one softmax with the selected rows.
 */
int oracle_attend_unit_tail(int b, int g, int B, int Hq, int Hkv, int hd, int64_t L, int C,
                            int rk, int rv, int dtype, const void *Ak, const void *Av,
                            const void *Bkt, const void *Bvt, const void *q,
                            const int32_t *sel_bg, int64_t n_sel, const void *Kt,
                            const void *Vt, int64_t T_max, int64_t n_tail, float *out)
{
    if (!Ak || !Av || !Bkt || !Bvt || !q || !out || B <= 0 || Hkv <= 0 || Hq % Hkv ||
        C <= 0 || L % C || b < 0 || b >= B || g < 0 || g >= Hkv || n_tail < 0 ||
        n_tail > T_max || (n_tail > 0 && (!Kt || !Vt)))
        return -1;
    int G = Hq / Hkv;
    int64_t nC = L / C, d_kv = (int64_t)Hkv * hd;
    int64_t nT = sel_bg ? n_sel * C : L;
    if (nT <= 0)
        return -1;
    int64_t nR = nT + n_tail;
    size_t esz = dtype == ORA_F32 ? 4 : 2;
    const char *ak = (const char *)Ak + (size_t)b * L * rk * esz;
    const char *av = (const char *)Av + (size_t)b * L * rv * esz;
    const char *bk = (const char *)Bkt + (size_t)b * d_kv * rk * esz;
    const char *bv = (const char *)Bvt + (size_t)b * d_kv * rv * esz;
    int64_t tail0 = ((int64_t)b * Hkv + g) * T_max * hd;   /* element offset of row 0 */
    double *z = malloc(sizeof(double) * nR * G);
    double *row = malloc(sizeof(double) * hd);
    double *acc = calloc((size_t)G * hd, sizeof(double));
    double *qd = malloc(sizeof(double) * G * hd);
    if (!z || !row || !acc || !qd) {
        free(z); free(row); free(acc); free(qd);
        return -2;
    }
    for (int hh = 0; hh < G; ++hh)
        for (int d = 0; d < hd; ++d)
            qd[hh * hd + d] = ora_load(q, dtype, ((int64_t)b * Hq + g * G + hh) * hd + d);
    double scale = 1.0 / sqrt((double)hd);
    int rc = 0;
    /* logits: the reconstructed keys of the selected rows, then the tail's keys */
    for (int64_t i = 0; i < nR; ++i) {
        if (i < nT) {
            int64_t t = i;
            if (sel_bg) {
                int64_t c = sel_bg[i / C];
                if (c < 0 || c >= nC) {
                    rc = -1;
                    goto done;
                }
                t = c * C + i % C;
            }
            ora_recon_row(ak, bk, dtype, t, rk, g, hd, row);
        } else {
            for (int d = 0; d < hd; ++d)
                row[d] = ora_load(Kt, dtype, tail0 + (i - nT) * hd + d);
        }
        for (int hh = 0; hh < G; ++hh) {
            double s = 0.0;
            for (int d = 0; d < hd; ++d)
                s += qd[hh * hd + d] * row[d];
            z[i * G + hh] = s * scale;
        }
    }
    for (int hh = 0; hh < G; ++hh) {
        double m = -INFINITY, l = 0.0;
        for (int64_t i = 0; i < nR; ++i)
            if (z[i * G + hh] > m)
                m = z[i * G + hh];
        for (int64_t i = 0; i < nR; ++i) {
            z[i * G + hh] = exp(z[i * G + hh] - m);
            l += z[i * G + hh];
        }
        for (int64_t i = 0; i < nR; ++i)
            z[i * G + hh] /= l;
    }
    /* values: the reconstructed rows, then the tail's rows */
    for (int64_t i = 0; i < nR; ++i) {
        if (i < nT) {
            int64_t t = sel_bg ? (int64_t)sel_bg[i / C] * C + i % C : i;
            ora_recon_row(av, bv, dtype, t, rv, g, hd, row);
        } else {
            for (int d = 0; d < hd; ++d)
                row[d] = ora_load(Vt, dtype, tail0 + (i - nT) * hd + d);
        }
        for (int hh = 0; hh < G; ++hh)
            for (int d = 0; d < hd; ++d)
                acc[hh * hd + d] += z[i * G + hh] * row[d];
    }
    for (int hh = 0; hh < G; ++hh)
        for (int d = 0; d < hd; ++d)
            out[((int64_t)b * Hq + g * G + hh) * hd + d] = (float)acc[hh * hd + d];
done:
    free(z); free(row); free(acc); free(qd);
    return rc;
}

/* ------------------------------------------------------------ [R-CLA] sharing set */

/* leader_of[l] = max{s in S : s <= l}; S must contain layer 0. */
int oracle_leader_map(const int32_t *S, int nS, int n_layers, int32_t *leader_of)
{
    if (!S || !leader_of || nS <= 0 || n_layers <= 0)
        return -1;
    for (int l = 0; l < n_layers; ++l) {
        int32_t best = -1;
        for (int i = 0; i < nS; ++i)
            if (S[i] <= l && S[i] > best)
                best = S[i];
        if (best < 0)
            return -1;
        leader_of[l] = best;
    }
    return 0;
}

/*
 * Decode attention of layer `layer` under R-CLA sharing.  K_lead, V_lead are
 * [n_lead][B][Hkv][L_max][hd]; the slot of leader s is |{s' in S : s' < s}| where
 * S = {l : leader_of[l] == l}.  If `layer` is a leader and k_new/v_new are given,
 * row `len` of its cache receives them first and len+1 rows are attended; otherwise
 * `len` rows are attended.  q and out are [B][Hq][hd].
 */
int oracle_rcla_decode_attend(int B, int Hq, int Hkv, int hd, int dtype, int layer,
                              const int32_t *leader_of, int n_layers, void *K_lead,
                              void *V_lead, int64_t L_max, int64_t len, const void *k_new,
                              const void *v_new, const void *q, float *out)
{
    if (!leader_of || !K_lead || !V_lead || !q || !out || B <= 0 || Hkv <= 0 ||
        Hq % Hkv || layer < 0 || layer >= n_layers || len < 0)
        return -1;
    int32_t lead = leader_of[layer];
    if (lead < 0 || lead > layer || leader_of[lead] != lead)
        return -1;
    int is_leader = lead == layer;
    if (!is_leader && (k_new || v_new))
        return -1; /* a non-leader owns no cache and skips the update */
    if ((k_new == NULL) != (v_new == NULL))
        return -1;
    int update = is_leader && k_new;
    int64_t n_rows = len + (update ? 1 : 0);
    if (n_rows > L_max || n_rows <= 0)
        return -1;
    int slot = 0;
    for (int l = 0; l < lead; ++l)
        slot += leader_of[l] == l;
    int G = Hq / Hkv;
    size_t esz = dtype == ORA_F32 ? 4 : 2;
    double scale = 1.0 / sqrt((double)hd);
    double *z = malloc(sizeof(double) * n_rows);
    double *acc = malloc(sizeof(double) * hd);
    if (!z || !acc) {
        free(z);
        free(acc);
        return -2;
    }
    for (int b = 0; b < B; ++b)
        for (int g = 0; g < Hkv; ++g) {
            int64_t base = (((int64_t)slot * B + b) * Hkv + g) * L_max * hd;
            if (update) { /* the leader's update: copy the new row into its cache */
                int64_t src = ((int64_t)b * Hkv + g) * hd;
                memcpy((char *)K_lead + (base + len * hd) * esz,
                       (const char *)k_new + src * esz, hd * esz);
                memcpy((char *)V_lead + (base + len * hd) * esz,
                       (const char *)v_new + src * esz, hd * esz);
            }
            for (int hh = 0; hh < G; ++hh) {
                int64_t qo = ((int64_t)b * Hq + g * G + hh) * hd;
                double m = -INFINITY, l = 0.0;
                for (int64_t t = 0; t < n_rows; ++t) {
                    double s = 0.0;
                    for (int d = 0; d < hd; ++d)
                        s += ora_load(q, dtype, qo + d) * ora_load(K_lead, dtype, base + t * hd + d);
                    z[t] = s * scale;
                    if (z[t] > m)
                        m = z[t];
                }
                for (int64_t t = 0; t < n_rows; ++t) {
                    z[t] = exp(z[t] - m);
                    l += z[t];
                }
                for (int d = 0; d < hd; ++d)
                    acc[d] = 0.0;
                for (int64_t t = 0; t < n_rows; ++t)
                    for (int d = 0; d < hd; ++d)
                        acc[d] += (z[t] / l) * ora_load(V_lead, dtype, base + t * hd + d);
                for (int d = 0; d < hd; ++d)
                    out[qo + d] = (float)acc[d];
            }
        }
    free(z);
    free(acc);
    return 0;
}

/* ------------------------------------------------------ [xKV] 2.2 storage, [R-CLA] */

/*
 * Bytes held by the compressed cache of B sequences and n_layers layers in windows of
 * W: per window one basis pair (L x (r_K + r_V)) and per layer one matrix pair
 * ((r_K + r_V) x d_kv), i.e. O(L*r + W*r*d) per window; plus the landmark keys
 * (n_layers * nC * d_kv per sequence) when with_landmarks is set.
 */
int64_t oracle_footprint_bytes(int B, int Hkv, int hd, int64_t L, int C, int rk, int rv,
                               int dtype, int n_layers, int W, int with_landmarks)
{
    if (B <= 0 || Hkv <= 0 || hd <= 0 || L <= 0 || W <= 0 || n_layers <= 0 || C <= 0)
        return -1;
    int64_t e = dtype == ORA_F32 ? 4 : 2;
    int64_t n_win = (n_layers + W - 1) / W;
    int64_t d_kv = (int64_t)Hkv * hd;
    int64_t per_seq = n_win * L * (rk + rv) * e + (int64_t)n_layers * (rk + rv) * d_kv * e;
    if (with_landmarks)
        per_seq += (int64_t)n_layers * (L / C) * d_kv * e;
    return B * per_seq;
}

/* Bytes of the leader-only K and V caches under R-CLA sharing with n_leaders leaders. */
int64_t oracle_rcla_cache_bytes(int B, int Hkv, int hd, int64_t L, int dtype, int n_leaders)
{
    if (B <= 0 || Hkv <= 0 || hd <= 0 || L <= 0 || n_leaders <= 0)
        return -1;
    int64_t e = dtype == ORA_F32 ? 4 : 2;
    return (int64_t)n_leaders * B * Hkv * L * hd * 2 * e;
}
