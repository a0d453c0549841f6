/*
 * xkv.h -- C ABI of the B200 (sm_100a) decode-attention library for a
 * cross-layer-compressed KV cache.
 *
 * The operations follow two pages:
 *  [xKV]   "xKV: Cross-Layer KV-Cache Compression via Aligned Singular Vector
 *          Extraction" (technical summary).  Section 2.2, cross-layer factorization
 *          (CLF): each window of W layers keeps one shared token basis A (L x r) and
 *          one small reconstruction matrix B_l (r x d_kv) per layer.  Section 2.3,
 *          selective reconstruction (SR): landmark-based chunk selection, then only
 *          the selected rows of K = A B_l (and V) are rebuilt.  Section 4, dense
 *          reconstruction (all rows).  The prefill side of section 2.2 -- the
 *          concatenation, the rank-r factorization, A and the B_l -- is here too
 *          (xkv_factorize_window), and so is folding generated rows back into the
 *          factors (xkv_refold_window).
 *  [R-CLA] "Stochastic KV Routing: adaptive depth-wise cache sharing".  Inference
 *          with a fixed sharing set S: a layer outside S reuses the KV cache of the
 *          nearest previous layer in S and skips its own K/V load and update
 *          (the page's Algorithm 2).
 *
 * Conventions for every call
 *  - All tensor arguments are DEVICE pointers to dense row-major arrays (last index
 *    fastest) in the layouts stated below, unless marked "host".  The caller owns
 *    every buffer; the library never allocates, frees or keeps a pointer after the
 *    call returns.
 *  - Storage type (dims->dtype): XKV_F32 or XKV_BF16, shared by the factors,
 *    landmarks, queries and caches of a call.  Outputs are fp32; scores are fp64.
 *  - Every pointer the kernels read or write must be 16-byte aligned.
 *  - Calls are asynchronous on `stream` (a cudaStream_t; NULL = the legacy default
 *    stream) and return after the launches are queued.
 *  - Every call returns an xkv_status; no C++ exception crosses the ABI.  On a
 *    non-OK status nothing was launched (argument errors) or a launch failed
 *    (XKV_ERR_CUDA); xkv_last_error() gives a message for the calling thread.
 *  - Query head h belongs to KV group g = h / G, G = n_q_heads / n_kv_heads.
 *  - Inputs holding NaN or Inf are outside the contract.
 *  - The library runs on compute capability 10.0 devices only (XKV_ERR_UNSUPPORTED
 *    otherwise).
 *  - Environment switches, read on every call:
 *      XKV_FORCE_SIMT  take the CUDA-core kernels for both attention paths instead of
 *                      the tensor-core ones (same results within the output tolerance)
 *      XKV_NO_TC       take the TMA + CUDA-core R-CLA kernel instead of the tensor-core one
 *      XKV_NO_PDL      launch every kernel in plain stream order (no programmatic
 *                      dependent launch between the kernels of a call)
 *      XKV_FAULT       "<entry point>:<status>": that entry point returns the status after
 *                      its argument checks, launching nothing (fault injection for tests;
 *                      read on every call)
 */
#ifndef XKV_H
#define XKV_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    XKV_OK = 0,
    XKV_ERR_INVALID_ARG = 1, /* a pointer, size, alignment or layout rule is broken */
    XKV_ERR_UNSUPPORTED = 2, /* valid, but outside what the kernels handle */
    XKV_ERR_CUDA = 3,        /* a CUDA runtime call or a launch failed */
    XKV_ERR_TIMEOUT = 4,     /* a bounded device-side wait gave up */
    XKV_ERR_INTERNAL = 5     /* a device-side consistency check failed */
} xkv_status;

typedef enum { XKV_F32 = 0, XKV_BF16 = 1 } xkv_dtype;

typedef enum {
    XKV_MODE_SELECTIVE = 0,
    XKV_MODE_DENSE = 1,
    XKV_MODE_RCLA = 2,
    XKV_MODE_REASSOC = 3  /* xkv_reassociated_attend; n_sel = 0 for every row (dense) */
} xkv_mode;

/*
 * Shapes of one decode call.
 *   batch       B  sequences
 *   n_q_heads   Hq query heads; n_kv_heads Hkv KV heads (Hq % Hkv == 0, G = Hq/Hkv <= 16)
 *   head_dim    hd in {64, 128}
 *   ctx_len     L  tokens in the compressed cache (xKV) or rows of cache capacity
 *                  L_max (R-CLA workspace sizing only)
 *   chunk       C  tokens per landmark chunk (xKV; L % C == 0; C % 8 == 0)
 *   rank_k/v    r_K, r_V ranks of the key / value bases (multiples of 16, <= 1024)
 *   dtype       xkv_dtype
 * d_kv = Hkv * hd, nC = L / C.
 */
typedef struct {
    int32_t batch;
    int32_t n_q_heads;
    int32_t n_kv_heads;
    int32_t head_dim;
    int64_t ctx_len;
    int32_t chunk;
    int32_t rank_k;
    int32_t rank_v;
    int32_t dtype;
} xkv_dims;

/*
 * Landmark keys of one layer [xKV 2.3, "landmark-based chunk selection"], built once
 * per cache (not part of a decode step).  The landmark of chunk c of KV head g is the
 * mean of the chunk's reconstructed key rows:
 *   lm[b][g][c][j] = round( (1/C) * sum_{t = cC}^{cC+C-1} (A^K[b][t] . B^K_l[:, g*hd + j]) )
 * accumulated in fp64 and rounded to nearest-even into the storage type.
 *   Ak_win    [B][L][r_K]      the layer's window basis A^K
 *   Bkt_layer [B][d_kv][r_K]   B^K_l stored column-major (element (i, j) at j*r_K + i)
 *   lm_layer  [B][Hkv][nC][hd] output
 */
xkv_status xkv_build_landmarks(const xkv_dims *dims, const void *Ak_win, const void *Bkt_layer,
                               void *lm_layer, void *stream);

/*
 * Landmark scores of one layer [xKV 2.3; the query-relevance step of SR]:
 *   scores[b][g][c] = max_{h in group g} sum_{d=0}^{hd-1} lm[b][g][c][d] * q[b][h][d]
 * Each product is formed exactly in fp64 and the sum runs in fp64 in ascending d,
 * so the value is reproducible bit for bit; the max orders -0 below +0.  Unscaled
 * (a positive scale does not change the ranking).
 *   lm_layer [B][Hkv][nC][hd], q [B][Hq][hd], scores [B][Hkv][nC] fp64 (output)
 * A score of NaN marks a failed launch (a bounded device-side wait gave up); scores
 * are never NaN otherwise.
 */
xkv_status xkv_score_landmarks(const xkv_dims *dims, const void *lm_layer, const void *q,
                               double *scores, void *stream);

/*
 * Chunk selection [xKV 2.3: "the sparse subset most relevant to the current query"]:
 * per (b, g), the forced chunks F = {0..n_sink-1} U {nC-n_recent..nC-1} plus the
 * top_k of the remaining chunks under (score descending, chunk index ascending),
 * written in ascending chunk order.  n_sel = min(top_k, nC - |F|) + |F| chunks per
 * unit; *n_sel_out (host pointer, may be NULL) receives it, computed on the host.
 *   scores [B][Hkv][nC] fp64, sel [B][Hkv][n_sel] int32 (output)
 * nC <= 16384.  A unit whose scores hold a NaN (a failed scoring launch) gets every
 * entry -1.
 */
xkv_status xkv_select_chunks(const xkv_dims *dims, const double *scores, int32_t top_k,
                             int32_t n_sink, int32_t n_recent, int32_t *sel,
                             int32_t *n_sel_out, void *stream);

/*
 * Scoring and selection in one call [xKV 2.3]: with no reserved chunks, sel is bit for
 * bit what xkv_select_chunks(xkv_score_landmarks(lm_layer, q), top_k, n_sink, n_recent)
 * gives --
 * the canonical fp64 scores, the forced chunks, the top_k by (score descending, chunk
 * index ascending), ascending order -- without writing the scores.  The landmarks are
 * scored in fp32 with a certified error bound; only the chunks whose membership that
 * bound leaves open (the band around the k-th score) are scored again in fp64, exactly as
 * xkv_score_landmarks scores them.  Arguments as for those two calls, plus
 *   ws, ws_bytes: scratch of at least xkv_score_select_workspace_bytes(dims) bytes.  On
 *       return (in stream order) its first B * Hkv 32-bit words hold, per (b, g), the
 *       number of chunks rescored in fp64, or 0xFFFFFFFF when the unit was scored wholly
 *       in fp64 (a band wider than 512 chunks, e.g. many equal scores, or fp32 scores out
 *       of range); the rest holds the fp64 scores of such units, the fp32 keys of every
 *       chunk and the per-CTA flags of the scoring pass.
 * G = n_q_heads / n_kv_heads in 1..8 or 16; nC <= 16384.  A unit whose fp64 scores hold a
 * NaN (inputs outside the contract) gets every entry -1.  reserved [B][Hkv][n_reserved]
 * (or NULL with n_reserved = 0): chunks forced in as well, see the value-range-aware
 * selection below.
 */
xkv_status xkv_score_select(const xkv_dims *dims, const void *lm_layer, const void *q,
                            int32_t top_k, int32_t n_sink, int32_t n_recent,
                            const int32_t *reserved, int32_t n_reserved, int32_t *sel,
                            int32_t *n_sel_out, void *ws, size_t ws_bytes, void *stream);
/* Scratch bytes of xkv_score_select (0 on bad dims). */
size_t xkv_score_select_workspace_bytes(const xkv_dims *dims);

/*
 * Value-range-aware selection [VASE, "Value-Aware Stochastic KV cache Eviction" page,
 * section 2.A: the tokens whose value vector has the largest range max(v) - min(v) are
 * always kept], applied to this path's chunks.  Setup, once per cache and layer:
 *
 * xkv_build_value_ranges: rho[b][g][c] = the largest max_j V_hat[t][g*hd + j] -
 *   min_j V_hat[t][g*hd + j] over the rows t of chunk c, V_hat = A^V B^V_l (the
 *   reconstructed values, never written to memory; bf16 caches on the tensor cores with
 *   fp32 accumulation, fp32 caches on the CUDA cores).
 *   Av_win [B][L][r_V], Bvt_layer [B][d_kv][r_V], rho_layer [B][Hkv][nC] fp32 (output).
 *   status: optional device word (4-byte aligned, may be NULL) that receives 0 or the OR
 *   of (1 << xkv_status) over device-side failures (a bounded wait that gave up).
 *
 * xkv_reserve_value_chunks: reserved[b][g][0..n_res) = the n_res chunks outside the sink
 *   and recent windows with the largest rho under (rho descending, chunk index
 *   ascending), in ascending order; n_res = xkv_n_reserved(nC, n_value, n_sink,
 *   n_recent) = min(n_value, nC - |sink U recent|), also written to *n_res_out (host,
 *   may be NULL).  nC <= 16384.
 *
 * Each decode step then passes reserved / n_res to xkv_score_select: the reserved chunks
 * join the forced ones and top_k more are chosen by score among the rest, so
 *   n_sel = |sink U recent| + n_res + min(top_k, nC - |sink U recent| - n_res).
 * A reserved list that is not a set of distinct chunks outside the sink and recent
 * windows makes its unit's entries -1 (and its band word 0xFFFFFFFE).  reserved = NULL
 * with n_reserved = 0 is the plain selection.
 */
xkv_status xkv_build_value_ranges(const xkv_dims *dims, const void *Av_win,
                                  const void *Bvt_layer, float *rho_layer, unsigned *status,
                                  void *stream);
xkv_status xkv_reserve_value_chunks(const xkv_dims *dims, const float *rho_layer,
                                    int32_t n_value, int32_t n_sink, int32_t n_recent,
                                    int32_t *reserved, int32_t *n_res_out, void *stream);
/* min(n_value, n_chunks - |sink U recent|); -1 on bad arguments. */
int64_t xkv_n_reserved(int64_t n_chunks, int32_t n_value, int32_t n_sink, int32_t n_recent);

/*
 * Selective (or dense) reconstruction followed by GQA attention
 * [xKV 2.3 "only the rows of the selected tokens are reconstructed from the shared
 * basis and the per-layer matrices"; xKV 4, dense reconstruction].
 * For each (b, g) let T = the C rows of every chunk in sel[b][g] (sel != NULL), or
 * all L rows (sel == NULL, dense).  With K_hat[t] = A^K[b][t] B^K_l[:, g-slice] and
 * V_hat[t] = A^V[b][t] B^V_l[:, g-slice] (never written to memory):
 *   z[h][t] = q[b][h] . K_hat[t] / sqrt(hd),  p = softmax_t(z),
 *   out[b][h] = sum_t p[h][t] V_hat[t]                       for every h in group g.
 *   Ak_win [B][L][r_K], Av_win [B][L][r_V]          the layer's window bases
 *   Bkt_layer [B][d_kv][r_K], Bvt_layer [B][d_kv][r_V] (column-major B_l)
 *   q [B][Hq][hd]; sel [B][Hkv][n_sel] int32 ascending chunk indices, or NULL
 *   out [B][Hq][hd] fp32 (output)
 *   ws, ws_bytes: scratch of at least xkv_workspace_bytes(dims, n_sel, mode) bytes
 *   (mode = XKV_MODE_SELECTIVE, or XKV_MODE_DENSE when sel == NULL).
 * Device-side failures of the call (an entry of sel outside [0, nC), a bounded wait
 * that gave up) make every output of the call NaN; the first 4 bytes of ws then hold
 * the OR of (1 << xkv_status) over the failures seen, until the next call.
 */
xkv_status xkv_reconstruct_attend(const xkv_dims *dims, const void *Ak_win, const void *Av_win,
                                  const void *Bkt_layer, const void *Bvt_layer, const void *q,
                                  const int32_t *sel, int32_t n_sel, float *out, void *ws,
                                  size_t ws_bytes, void *stream);

/*
 * Decode attention of layer `layer` under R-CLA sharing [R-CLA, inference strategy S
 * and Algorithm 2].  leader_of (HOST, [n_layers]) maps each layer to the layer whose
 * cache it reads: leader_of[0] == 0, leader_of[l] <= l, leader_of[leader_of[l]] ==
 * leader_of[l]; the leaders are S = {l : leader_of[l] == l}, and the cache slot of
 * leader s is |{s' in S : s' < s}|.
 *   K_lead, V_lead [n_lead][B][Hkv][L_max][hd] leader-only caches
 *   len    rows valid in the leader's cache when the call starts
 *   k_new, v_new [B][Hkv][hd]: only for a leader layer (both or neither).  When given,
 *          the call first writes them at row `len` of the layer's own cache (the
 *          update) and attends len+1 rows; otherwise it attends `len` rows.  A
 *          non-leader owns no cache and gets XKV_ERR_INVALID_ARG if given a row.
 *   q [B][Hq][hd], out [B][Hq][hd] fp32 (output)
 *   ws, ws_bytes: scratch of at least xkv_workspace_bytes(dims with ctx_len = L_max,
 *          0, XKV_MODE_RCLA) bytes.
 * dims->chunk, rank_k and rank_v are ignored.  A bounded device-side wait that gives up
 * makes the outputs of the (b, g) units whose rows it had not finished NaN (there is no
 * status word on this path).
 */
xkv_status rcla_decode_attend(const xkv_dims *dims, int32_t layer, const int32_t *leader_of,
                              int32_t n_layers, void *K_lead, void *V_lead, int64_t L_max,
                              int64_t len, const void *k_new, const void *v_new, const void *q,
                              float *out, void *ws, size_t ws_bytes, void *stream);

/*
 * xkv_reconstruct_attend without a workspace, for callers that cannot allocate device
 * memory (engine plugin hooks handed no workspace, processes whose HBM is reserved by a
 * serving engine's KV pool, paths where an allocation's device synchronisation is not
 * allowed).  No counterpart on the pages: this is a library convenience.
 *   Same arguments, layouts and results as xkv_reconstruct_attend, minus ws / ws_bytes.
 *   Scratch: a fixed 16 MiB array of device memory inside the library, held by every
 *   GPU that loads the library until the process exits.  A call whose scratch need
 *   (xkv_workspace_bytes) exceeds 16 MiB returns XKV_ERR_UNSUPPORTED.
 *   The first call on a device (with that device current) looks up the array's device
 *   address once and keeps it; make that first call before any stream capture, and do
 *   not use this entry point after cudaDeviceReset (the kept address would be stale).
 *   Argument errors are reported as by xkv_reconstruct_attend, before any CUDA call;
 *   XKV_FAULT injection uses this entry point's own name.
 *   Every call on a device shares the one array: calls whose kernels overlap on the GPU
 *   (different streams, or graphs replayed concurrently) race and give wrong results.
 *   Calls queued on one stream are safe.  The function calls no allocator.
 */
xkv_status xkv_reconstruct_attend_noalloc(const xkv_dims *dims, const void *Ak_win,
                                          const void *Av_win, const void *Bkt_layer,
                                          const void *Bvt_layer, const void *q,
                                          const int32_t *sel, int32_t n_sel, float *out,
                                          void *stream);

/*
 * xkv_reconstruct_attend plus a tail of tokens generated after the cache was compressed,
 * kept uncompressed and always attended: for each (b, g) the softmax runs over the rows T
 * of xkv_reconstruct_attend followed by rows [0, n_tail) of the tail.  The pages are
 * silent on generated tokens; this is the reading taken (they are not refolded into
 * the basis here).
 *   K_tail, V_tail [B][Hkv][T_max][hd] in the storage type; 0 <= n_tail <= T_max,
 *   T_max > 0; NULL tails are allowed when n_tail == 0.
 *   ws, ws_bytes: at least xkv_tail_workspace_bytes(dims, sel ? n_sel : 0, T_max).
 * Other arguments, layouts and failure signalling as for xkv_reconstruct_attend.
 */
xkv_status xkv_reconstruct_attend_tail(const xkv_dims *dims, const void *Ak_win,
                                       const void *Av_win, const void *Bkt_layer,
                                       const void *Bvt_layer, const void *q,
                                       const int32_t *sel, int32_t n_sel, const void *K_tail,
                                       const void *V_tail, int64_t T_max, int64_t n_tail,
                                       float *out, void *ws, size_t ws_bytes, void *stream);
/* Workspace bytes for xkv_reconstruct_attend_tail (0 on invalid arguments). */
size_t xkv_tail_workspace_bytes(const xkv_dims *dims, int32_t n_sel, int64_t T_max);

/*
 * The same decode attention as xkv_reconstruct_attend, computed by associativity in the
 * rank space of the window's basis [xKV 2.2: K_hat = A^K B^K_l, V_hat = A^V B^V_l]:
 *   q~_h = B^K_g q_h,   z_h[t] = A^K[b][t] . q~_h / sqrt(hd),   p_h = softmax_t(z_h),
 *   u_h = sum_t p_h[t] A^V[b][t],   out[b][h] = u_h B^V_g
 * The pages describe the explicit form; this reassociation is exact in real arithmetic
 * and is not printed there.  It reads the same rows of A once and does r-deep dot
 * products instead of r x hd GEMMs, so dense reconstruction becomes bound by HBM rather
 * than by the tensor cores.  Arguments, layouts and failure signalling as for
 * xkv_reconstruct_attend; ws holds at least
 * xkv_workspace_bytes(dims, sel ? n_sel : 0, XKV_MODE_REASSOC) bytes.  Runs for bf16,
 * head_dim 128, G in {1, 2, 4, 5, 8}, ranks multiples of 128 up to 1024 (r_K up to 512
 * when G > 4) and chunks dividing 256; other shapes return XKV_ERR_UNSUPPORTED.  Dense
 * calls (sel == NULL) with 8, 16, 24 or 32 query heads read the window once for all heads
 * of a sequence (per-sequence spans of 128-token tiles); the workspace then also holds
 * an fp32 logit scratch of B * Hq * L floats (rounded up to whole tiles).
 */
xkv_status xkv_reassociated_attend(const xkv_dims *dims, const void *Ak_win, const void *Av_win,
                                   const void *Bkt_layer, const void *Bvt_layer, const void *q,
                                   const int32_t *sel, int32_t n_sel, float *out, void *ws,
                                   size_t ws_bytes, void *stream);

/* Scratch bytes the attention calls need (the split-K partial results). 0 on bad dims. */
size_t xkv_workspace_bytes(const xkv_dims *dims, int32_t n_sel, int32_t mode);

/*
 * Cross-layer factorization of one window [xKV 2.2, steps 1-3: concatenate the W
 * layers' caches side by side, rank-r SVD, one shared token basis A and one
 * reconstruction matrix B_l per layer].  Per sequence b, with
 * X_b = [X_0,b | ... | X_{W-1},b] (L x W*d_kv), it returns A_b (L x r, orthonormal
 * columns spanning the dominant rank-r left singular subspace of X_b) and
 * B_l,b = A_b^T X_l,b, so that A_b B_l,b is the rank-r truncated SVD of X_b restricted
 * to layer l's columns once the iteration has converged.  Computed by randomized
 * subspace iteration (Halko, Martinsson and Tropp 2011, Algorithm 4.4) with n_iter
 * power passes and CholeskyQR2 orthonormalisation; the error against the exact
 * truncated SVD shrinks like (s_{r+1} / s_r)^(2 n_iter + 1).  If rank(X_b) < r the
 * surplus columns of A_b (and rows of B_l,b) are zero.
 *
 *   dims        batch, n_kv_heads, head_dim, ctx_len (= L) and dtype are used; the
 *               query-head, chunk and rank fields are ignored
 *   window      W >= 1 layers in the window
 *   rank        r: a multiple of 16, 16 <= r <= min(1024, L, W*d_kv)
 *   X           [W][B][L][d_kv] in dtype: layer l's cache, token-major, the KV heads of
 *               a token side by side (d_kv = n_kv_heads * head_dim)
 *   omega       [W*d_kv][r] fp32, device: the Gaussian test matrix (the caller draws it)
 *   n_iter      power passes, 0..16
 *   A_out       [B][L][r] in dtype (the window basis the decode calls take as Ak_win /
 *               Av_win)
 *   Bt_out      [W][B][d_kv][r] in dtype: B_l stored column-major per layer (what the
 *               decode calls take as Bkt_layer / Bvt_layer)
 *   ws          device scratch of xkv_factorize_workspace_bytes bytes.  Its first 4 bytes
 *               hold, after the call (in stream order), the OR of (1 << xkv_status) over
 *               device-side failures (a bounded wait that gave up); A_out and Bt_out are
 *               then NaN.
 * All device pointers 16-byte aligned.  The products run on the library's own kernels:
 * bf16 caches on the tensor cores (the fp32 bases split into bf16 hi + lo parts, the
 * products with R^-1 in TF32), fp32 caches in plain fp32 on the CUDA cores; fp64 Gram
 * matrices and Cholesky factors.  Asynchronous on `stream`; INVALID_ARG / UNSUPPORTED
 * before any launch.
 */
xkv_status xkv_factorize_window(const xkv_dims *dims, int32_t window, int32_t rank,
                                const void *X, const float *omega, int32_t n_iter,
                                void *A_out, void *Bt_out, void *ws, size_t ws_bytes,
                                void *stream);

/* Scratch bytes of xkv_factorize_window for these dims, window and rank (0 on bad
 * arguments). */
size_t xkv_factorize_workspace_bytes(const xkv_dims *dims, int32_t window, int32_t rank);

/*
 * Refold the tail of generated rows into a window's factors [xKV 2.2 applied again at
 * decode time; the pages give no schedule]: per layer the cache the decode calls see,
 * X'_l = [A·B_l ; tail_l] ((L + T) x d_kv, the reconstructed part rounded to dtype),
 * is factored at rank r exactly as xkv_factorize_window does, so the next decode steps
 * read L + T compressed rows and an empty tail.
 *
 *   dims        as for xkv_factorize_window; ctx_len = L, the rows already compressed
 *   A_win       [B][L][r], Bt_win [W][B][d_kv][r]: the current factors (dtype)
 *   tail        [W][B][T][d_kv] (dtype): the generated rows of each layer; may be NULL
 *               when n_tail = T = 0
 *   omega, n_iter, Bt_out   as for xkv_factorize_window
 *   A_out       [B][L + T][r]
 *   ws          device scratch of xkv_refold_workspace_bytes bytes (the factorization's
 *               scratch, then the extended caches); status word as for
 *               xkv_factorize_window
 * Bt_out may be Bt_win (it is read before it is written, in stream order).  Asynchronous;
 * INVALID_ARG / UNSUPPORTED before any launch.
 */
xkv_status xkv_refold_window(const xkv_dims *dims, int32_t window, int32_t rank,
                             const void *A_win, const void *Bt_win, const void *tail,
                             int64_t n_tail, const float *omega, int32_t n_iter, void *A_out,
                             void *Bt_out, void *ws, size_t ws_bytes, void *stream);

/* Scratch bytes of xkv_refold_window (0 on bad arguments). */
size_t xkv_refold_workspace_bytes(const xkv_dims *dims, int32_t window, int32_t rank,
                                  int64_t n_tail);

/* Chunks selected per (b, g): min(top_k, nC - |F|) + |F|; -1 on bad arguments. */
int64_t xkv_n_selected(int64_t n_chunks, int32_t top_k, int32_t n_sink, int32_t n_recent);

/*
 * Bytes of the compressed cache [xKV 2.2 storage, O(L*r + W*r*d) per window]: for
 * each sequence, ceil(n_layers / W) bases (L x (r_K + r_V)) and n_layers matrix pairs
 * ((r_K + r_V) x d_kv), plus the landmark keys (n_layers x nC x d_kv) when
 * with_landmarks != 0.  -1 on bad arguments.
 */
int64_t xkv_footprint_bytes(const xkv_dims *dims, int32_t n_layers, int32_t window,
                            int32_t with_landmarks);

/* Bytes of the leader-only K and V caches [R-CLA]: n_leaders x B x Hkv x L_max x hd x 2. */
int64_t rcla_cache_bytes(const xkv_dims *dims, int32_t n_leaders, int64_t L_max);

/* Message for the calling thread's last non-OK status ("" if none). */
const char *xkv_last_error(void);

#ifdef __cplusplus
}
#endif

#endif /* XKV_H */
