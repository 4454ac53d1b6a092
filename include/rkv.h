/*
 * rkv.h -- C ABI of librkv: one decode step of retention-scored, globally
 * budgeted KV-cache eviction with grouped-query decode attention over the
 * surviving ragged paged cache, on NVIDIA B200 (sm_100a).
 *
 * The operations follow three web summaries of papers:
 *   [DBTrimKV]  "Make Each Token Count: Towards Improving Long-Context
 *               Performance with KV Cache Eviction"
 *   [TRIM-KV]   "Cache What Lasts: Token Retention for Memory-Bounded KV
 *               Cache in LLMs"
 *   [ContourKV] "Trust the Mass: Forced Weights in KV-Cache Eviction"
 *   [IndexMem]  "IndexMem: learned KV eviction with latent memory" (only
 *               its latent memory for evicted tokens)
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * - Every call returns an int status: RKV_OK (0) or a negative RKV_ERR_*.
 *   Host-side argument errors are reported synchronously and nothing is
 *   enqueued.  rkv_last_error() returns a per-thread message for the last
 *   failure on the calling thread.
 * - Work is enqueued asynchronously on the caller's CUDA stream (`stream`
 *   is a cudaStream_t passed as void*; NULL = legacy default stream).  No
 *   call synchronises the device, and no call allocates or frees device
 *   memory: the caller owns every buffer, including the workspace.
 * - All pointers in rkv_cache_t / rkv_select_t and all array arguments are
 *   DEVICE pointers unless a comment says "host".
 * - Data-dependent failures found on the device (bad input values, pool
 *   exhaustion, a timed-out grid barrier) do not abort: the kernel records
 *   RKV_DEV_* bits in a status word inside the workspace and skips the
 *   offending work.  rkv_device_status() returns the device address of that
 *   word; after a nonzero status the cache contents are unspecified.
 * - Several calls of one step share a workspace; calls on one workspace must
 *   be ordered (same stream, or otherwise serialised).
 *
 * Cache layout (this library's own specification of the paged, per-head
 * variable-length layout of [DBTrimKV] Methodology 4 and the physically
 * enforced ragged storage of [ContourKV] Methodology 2)
 * ---------------------------------------------------------------------
 * C = B*L*H heads; head c = (b*L + l)*H + h.  Query head hq = h*G + g
 * (G = Hq/H) of layer l reads KV head h.  Page size P = 16.
 * Logical slot k (0 <= k < len[c]) of head c lives in page
 * block_table[c*max_pages + k/16] at offset k%16; rows of a page are
 * contiguous: k_pool + (page*16 + k%16)*D elements.  Slot order within a
 * head is not position order.  free_stack[0 .. *free_top) holds the free
 * pages; the top is free_stack[*free_top - 1].
 */
#ifndef RKV_H_
#define RKV_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define RKV_API __attribute__((visibility("default")))
#else
#define RKV_API
#endif

/* ---- status codes (host) ---- */
#define RKV_OK 0
#define RKV_ERR_INVALID_ARG (-1)         /* null pointer, bad size, bad shape */
#define RKV_ERR_UNSUPPORTED (-2)         /* valid but not built: (dtype, D, G), P != 16 */
#define RKV_ERR_WORKSPACE_TOO_SMALL (-3) /* ws_bytes < rkv_workspace_size() */
#define RKV_ERR_CUDA (-4)                /* a CUDA runtime call failed; see rkv_last_error() */
#define RKV_ERR_NOT_IMPLEMENTED (-5)

/* ---- device status bits (in the workspace status word) ---- */
#define RKV_DEV_BAD_INPUT 1      /* NaN log-retention, age t-i outside [1, 2^24), position too wide */
#define RKV_DEV_POOL_EXHAUSTED 2 /* append found the free-page stack empty */
#define RKV_DEV_TABLE_OVERFLOW 4 /* append past max_pages of a head */
#define RKV_DEV_TIMEOUT 8        /* a bounded wait gave up (2 s, or the workspace's wait limit) */

/* ---- element types of the K/V pools ---- */
#define RKV_BF16 0
#define RKV_F32 1

/* The paged cache.  Every pointer is a device pointer owned by the caller.
 *   k_pool, v_pool  [n_pages][16][D] of dtype (RKV_BF16 or RKV_F32)
 *   pos_pool        [n_pages][16] int32, token position i of each row
 *   lb_pool         [n_pages][16] float, log-retention log(beta_i) of each row
 *                   (the retention gate output, [TRIM-KV] core mechanism 1)
 *   block_table     [C][max_pages] int32, page id or -1
 *   len             [C] int32, entries per head
 *   free_stack      [n_pages] int32, free_top [1] int32
 * Positions within one head must be distinct.  Pools must be 16-byte
 * aligned (row bytes D*elt are a multiple of 16).  A len outside
 * [0, max_pages*16] is read as the nearest bound and recorded as
 * RKV_DEV_BAD_INPUT. */
typedef struct rkv_cache {
    void *k_pool;
    void *v_pool;
    int32_t *pos_pool;
    float *lb_pool;
    int32_t *block_table;
    int32_t *len;
    int32_t *free_stack;
    int32_t *free_top;
    int32_t B, L, H, Hq, D, P;
    int32_t n_pages, max_pages;
    int32_t dtype;
} rkv_cache_t;

/* Result of one selection, consumed by attention, dropped mass and
 * compaction of the same step.  Device buffers owned by the caller:
 *   kappa      [B] uint64   entry e of sequence b is kept iff key(e) < kappa[b];
 *                           kappa = (largest kept key) + 1, or 0 when nothing
 *                           and ~0 when everything is kept
 *                           (key defined at rkv_score_select)
 *   kept       [C] int32    entries of head c that are kept
 *   n_pre      [C] int32    len[c] when the selection ran
 *   keep_mask  [C][max_pages] uint16, bit r of word (c, p) set iff slot
 *                           16p + r of head c is kept
 *   plan       [C + 2] int32: plan[c] = pages freed by compaction in heads
 *                           < c (exclusive prefix), plan[C] = total freed,
 *                           plan[C+1] = *free_top when the selection ran */
typedef struct rkv_select {
    uint64_t *kappa;
    int32_t *kept;
    int32_t *n_pre;
    uint16_t *keep_mask;
    int32_t *plan;
} rkv_select_t;

/* Library version string (host, static). */
RKV_API const char *rkv_version(void);

/* Message of the last failed call on this thread (host, thread-local). */
RKV_API const char *rkv_last_error(void);

/* Bytes of workspace the calls below need for this cache shape (host only,
 * no CUDA call).  Returns 0 if the shape is invalid. */
RKV_API size_t rkv_workspace_size(const rkv_cache_t *cache);

/* Zero the workspace (async memset on `stream`).  Call once after
 * allocating it, and again after a nonzero device status. */
RKV_API int rkv_workspace_init(void *ws, size_t ws_bytes, void *stream);

/* Device address of the status block inside the workspace: int32[5] =
 *   [0] RKV_DEV_* bits (sticky until rkv_workspace_init)
 *   [1] site of the first bounded wait that gave up (0: none), for reports
 *   [2] rkv_decode_step calls whose selection was resolved in the threshold
 *       window, [3] those that ran the exact selection (cumulative counters)
 *   [4] the wait limit set by rkv_workspace_set_wait_limit (0: default).
 * Pure pointer arithmetic. */
RKV_API int32_t *rkv_device_status(void *ws);

/* Limit, in microseconds, of the kernels' waits on other CTAs of the same
 * launch (grid-wide barriers, the fused step's wait for the compactions
 * before a pop) for calls on this workspace; 0 restores the default of 2 s.
 * A wait that runs out records RKV_DEV_TIMEOUT and its site, and the CTA
 * leaves the kernel; the workspace must then be re-initialised and the
 * cache contents are unspecified.  Waits of a CTA on its own asynchronous
 * copies keep the 2 s guard.  A tiny limit makes the timeout path run on
 * purpose, without any hang.  Enqueued on `stream` (one small launch). */
RKV_API int rkv_workspace_set_wait_limit(void *ws, size_t ws_bytes, uint32_t microseconds, void *stream);

/* ---------------------------------------------------------------------------
 * rkv_score_select -- score every cached entry and find the global top-M.
 *
 * [DBTrimKV] Methodology 2 / [TRIM-KV] core mechanism 2: the retention
 * weight of token i at step t is beta_i^(t-i); its logarithm is taken as one
 * IEEE binary32 multiply s = fl32(float(t - i) * lb_i) (round to nearest
 * even; -0 counts as +0).  [DBTrimKV] Methodology 3: all entries of all
 * layers and heads of a sequence are ranked together and the top M_global
 * are kept ([TRIM-KV] core mechanism 4: the lowest are evicted).  Order:
 * higher s first; equal s by ascending (l, h, i).  The 64-bit key is
 * (order-preserving map of s) << 32 | ((l*H + h) << ib | i), ib = 32 -
 * ceil(log2(L*H)); positions must be < 2^ib.
 *
 *   t         [B] int32   decode step of each sequence; entries present are
 *                         those with position < t (age t-i in [1, 2^24))
 *   m_global  [B] int64   budget per sequence (negative = 0)
 *   sel       outputs (rkv_select_t), all written
 * Errors: RKV_ERR_INVALID_ARG (shape), RKV_ERR_WORKSPACE_TOO_SMALL,
 * RKV_ERR_UNSUPPORTED (L*H > 2^24), RKV_ERR_CUDA (launch).  Device:
 * RKV_DEV_BAD_INPUT (entry ignored), RKV_DEV_TIMEOUT.
 * One cooperative persistent launch (grid-wide barriers with a bounded wait).
 */
RKV_API int rkv_score_select(const rkv_cache_t *cache, const int32_t *t, const int64_t *m_global,
                             const rkv_select_t *sel, void *ws, size_t ws_bytes, void *stream);

/* ---------------------------------------------------------------------------
 * rkv_score_select_budget -- the selection under another budget allocation,
 * with the same outputs as rkv_score_select (so attention, dropped mass,
 * compaction and append follow unchanged).
 *
 * RKV_BUDGET_PER_HEAD ([TRIM-KV] core mechanism 4 with a budget for each
 * head; [DBTrimKV] Methodology 3 names this fixed per-head allocation as
 * what its global budget replaces): head c keeps its top m_head[c] entries
 * by score (negative = 0), equal scores by ascending position.  kappa = 0
 * (there is no sequence-wide threshold).
 *
 * RKV_BUDGET_CONTOUR ([ContourKV] Methodology 3: the dropped-mass statistic
 * marks "flat" cells, which get a fixed budget; every cell keeps a recency
 * floor; the scores are reused with this allocation).  This library's
 * reading, per sequence:
 *   - a cell is a KV head c; it is flat iff the binary32 mean of its query
 *     heads' dropped mass at the previous evicting step, dm_prev[c][0..G-1]
 *     summed in ascending order and divided by G, exceeds flat_threshold;
 *   - every head keeps its min(recency_floor, len) most recent entries
 *     (largest positions);
 *   - a flat head also keeps the top flat_budget of its other entries by
 *     score (equal scores by ascending position);
 *   - the rest of the budget, max(0, m_global[b] - entries kept so far), goes
 *     to the global order of rkv_score_select over the other entries of the
 *     non-flat heads; kappa[b] is that part's threshold.
 *   Floors and flat budgets are kept even when they exceed m_global.
 *
 *   budget    host pointer to the parameters below (device arrays inside)
 * Errors: RKV_ERR_INVALID_ARG (unknown mode, missing array, NaN threshold),
 * RKV_ERR_WORKSPACE_TOO_SMALL, RKV_ERR_UNSUPPORTED, RKV_ERR_CUDA.  Device:
 * RKV_DEV_BAD_INPUT (entry ignored), RKV_DEV_TIMEOUT.  One launch per head
 * plus a plan launch (per head) or the global selection (ContourKV); the
 * threshold window of the decode step is not used or changed.
 */
#define RKV_BUDGET_PER_HEAD 0
#define RKV_BUDGET_CONTOUR 1
typedef struct rkv_budget {
    int32_t mode;            /* RKV_BUDGET_PER_HEAD or RKV_BUDGET_CONTOUR */
    const int32_t *m_head;   /* [C] per-head budgets (PER_HEAD) */
    const int64_t *m_global; /* [B] budget per sequence (CONTOUR) */
    const float *dm_prev;    /* [C][G] dropped mass of the previous evicting step (CONTOUR) */
    float flat_threshold;    /* a head is flat iff its mean dropped mass > this (CONTOUR) */
    int32_t flat_budget;     /* entries a flat head keeps beyond its floor (CONTOUR) */
    int32_t recency_floor;   /* most recent entries every head keeps (CONTOUR) */
} rkv_budget_t;

RKV_API int rkv_score_select_budget(const rkv_cache_t *cache, const int32_t *t, const rkv_budget_t *budget,
                                    const rkv_select_t *sel, void *ws, size_t ws_bytes, void *stream);

/* ---------------------------------------------------------------------------
 * rkv_score_select_noalloc -- rkv_score_select without a workspace argument,
 * for callers that cannot allocate device memory themselves (for example
 * code running where cudaMalloc is not permitted, such as inside a host
 * callback or under an allocator they do not control).  It has no
 * counterpart in the papers: it is a deployment convenience.  Same inputs,
 * outputs and results as rkv_score_select, and the same host-side errors;
 * device-side RKV_DEV_* errors and timeouts are not reported (the status
 * word lives in the private scratch).  Its scratch (status word, barrier
 * counters, radix histograms, window candidates) is a fixed __device__ array
 * of about 0.9 MiB inside the library, which every GPU that loads the
 * library holds until the process exits.  Limits: at most 16 sequences
 * (B <= 16), else RKV_ERR_UNSUPPORTED.  The first call on a device looks up
 * that array's device address (cudaGetSymbolAddress), so make the first
 * call on each device before any stream capture.  Each call clears the
 * scratch it uses (an async memset on `stream`), threshold window included:
 * no window is carried between calls, so every call runs the exact radix
 * passes (its cost is that of a first call of rkv_score_select).  It
 * allocates nothing.  All calls share the one array: calls that overlap on
 * the GPU (different streams, or other threads) race and must be serialised
 * by the caller.
 */
RKV_API int rkv_score_select_noalloc(const rkv_cache_t *cache, const int32_t *t, const int64_t *m_global,
                                     const rkv_select_t *sel, void *stream);

/* ---------------------------------------------------------------------------
 * rkv_paged_decode_attn -- grouped-query decode attention over the kept
 * entries, read from the pre-compaction pages.
 *
 * [ContourKV] Problem definition: after selection the softmax is
 * renormalised over the kept set (forced weights):
 *   o[c,g] = sum_{j kept} exp(z_j) v_j / sum_{j kept} exp(z_j),
 *   z_j = scale * <q[c,g], k_j>   (fp32 accumulation of bf16/f32 data).
 * With `dropped` non-NULL the same pass also returns [ContourKV]
 * Methodology 3's dropped mass (see rkv_dropped_mass).
 *
 *   q         [C][G][D] float (== [B][L][Hq][D])
 *   scale     logit scale (1/sqrt(D) for standard attention)
 *   sel       selection of this step, or NULL: every entry is kept
 *   out       [C][G][D] float   written (0 where nothing is kept)
 *   lse_kept  [C][G] float or NULL: natural-log sum of exp(z) over kept
 *             entries (-inf where nothing is kept)
 *   dropped   [C][G] float or NULL
 * Errors: RKV_ERR_INVALID_ARG, RKV_ERR_UNSUPPORTED ((dtype, D, G) not
 * instantiated), RKV_ERR_WORKSPACE_TOO_SMALL, RKV_ERR_CUDA.
 */
RKV_API int rkv_paged_decode_attn(const rkv_cache_t *cache, const float *q, float scale,
                                  const rkv_select_t *sel, float *out, float *lse_kept,
                                  float *dropped, void *ws, size_t ws_bytes, void *stream);

/* ---------------------------------------------------------------------------
 * rkv_dropped_mass -- per query head, the dense softmax weight held by the
 * evicted entries ([ContourKV] Methodology 3 and main contributions):
 *   dm[c,g] = sum_{j evicted} exp(z_j) / sum_{j present} exp(z_j)
 * over every entry present before this step's eviction (K only; V is not
 * read).  0 for a head with no entries; 1 if all of its entries are
 * evicted.  sel must be non-NULL.
 *   dropped   [C][G] float   written
 * Errors as rkv_paged_decode_attn.
 */
RKV_API int rkv_dropped_mass(const rkv_cache_t *cache, const float *q, float scale,
                             const rkv_select_t *sel, float *dropped, void *ws, size_t ws_bytes,
                             void *stream);

/* ---------------------------------------------------------------------------
 * rkv_eviction_error -- per query head, the distance between the dense
 * attention output mu (softmax over every entry present before this step's
 * eviction) and the forced-weight output m_A over the kept set:
 *   err[c,g] = || mu - m_A ||   (Euclidean norm over the head dimension)
 * ([ContourKV] Methodology 1, theoretical analysis: the eviction error of a
 * kept subset A).  Computed as dm * || m_ev - m_A ||, with m_ev the
 * forced-weight output over the evicted entries (mu is the dm-weighted mix
 * of m_ev and m_A): only the evicted rows' K and V and the keep words are
 * read.  Call it after rkv_paged_decode_attn of the same step (whose out
 * and dropped it takes) and before rkv_compact_pages.
 *   q, scale    as rkv_paged_decode_attn
 *   sel         the step's selection (keep masks), non-NULL
 *   out_kept    [C][G][D] float: m_A, rkv_paged_decode_attn's out
 *   dropped     [C][G] float: that call's dropped mass
 *   err         [C][G] float   written (0 where nothing is evicted; ||mu||
 *               where nothing is kept)
 * ws, ws_bytes are checked like the other calls' but not written.
 * Errors: RKV_ERR_INVALID_ARG, RKV_ERR_UNSUPPORTED ((D, G) not built: D 64 or
 * 128 with G in {1, 2, 4, 7, 8}), RKV_ERR_WORKSPACE_TOO_SMALL, RKV_ERR_CUDA.
 */
RKV_API int rkv_eviction_error(const rkv_cache_t *cache, const float *q, float scale,
                               const rkv_select_t *sel, const float *out_kept, const float *dropped,
                               float *err, void *ws, size_t ws_bytes, void *stream);

/* ---------------------------------------------------------------------------
 * Latent memory for evicted tokens ([IndexMem] "learned KV eviction with
 * latent memory", Methodology B: evicted tokens update a fixed-size state M
 * and a stabilising vector b online by outer-product accumulation with
 * decay; a learned projection and a gate g(q) read it; the output is
 * o = o_attn + g(q) * m(q)).  The page gives no formulas; this library's
 * form, per KV head c of layer l:
 *   phi(x) = elu(P_l x) + 1   (elu(y) = y for y > 0, exp(y) - 1 else)
 *   update:  M_c = decay * M_c + sum_{j evicted} phi(k_j) v_j^T
 *            b_c = decay * b_c + sum_{j evicted} phi(k_j)
 *   read:    m = phi(q)^T M_c / (phi(q)^T b_c)   (0 when that is 0)
 *            g = sigmoid(gate_w[l][hq] . q + gate_b[l][hq]);  out += g * m
 * The slow weights are the caller's (random ones in this repository's
 * benchmark); the state is the caller's, zero at the start of a sequence. */
typedef struct rkv_memory {
    const float *proj;    /* [L][D][D] projection P_l, row i gives feature i */
    const float *gate_w;  /* [L][Hq][D] gate weights (read only) */
    const float *gate_b;  /* [L][Hq] gate biases (read only) */
    float decay;          /* in [0, 1], applied once per update call */
    float *M;             /* [C][D][D] state, fp32, 16-byte aligned */
    float *b;             /* [C][D] normaliser */
} rkv_memory_t;

/* rkv_memory_update -- fold this step's evicted entries (keep-mask bit clear
 * among the first n_pre[c] slots) into the state.  Call it after the
 * selection and before rkv_compact_pages (the rows are read in place).
 *   sel   the step's selection (keep_mask, n_pre)
 *   mem   host pointer; proj, decay, M, b used
 * Errors: RKV_ERR_INVALID_ARG (NULL, decay outside [0, 1]), RKV_ERR_UNSUPPORTED
 * (D not 64/128 or G > 8), RKV_ERR_CUDA.  One launch, one CTA per head. */
RKV_API int rkv_memory_update(const rkv_cache_t *cache, const rkv_select_t *sel, const rkv_memory_t *mem,
                              void *stream);

/* rkv_memory_read -- add the gated memory read to the attention output:
 * out[c][g][:] += g(q) * m(q) for every query row.
 *   q     [C][G][D] float, the step's queries
 *   out   [C][G][D] float, rkv_paged_decode_attn's output, updated in place
 * Errors as rkv_memory_update.  One launch, one CTA per head. */
RKV_API int rkv_memory_read(const rkv_cache_t *cache, const float *q, const rkv_memory_t *mem, float *out,
                            void *stream);

/* ---------------------------------------------------------------------------
 * rkv_compact_pages -- physically remove the evicted entries
 * ([ContourKV] Methodology 2: ragged storage, not a mask; [DBTrimKV]
 * Methodology 4: variable length per head).  Per head c with n = n_pre[c]
 * and n_new = kept[c]: the j-th kept slot at or above n_new (ascending)
 * fills the j-th non-kept slot below n_new (ascending), moving its K, V,
 * position and log-retention; pages at table indices [ceil(n_new/16),
 * ceil(n/16)) are pushed onto the free stack (heads in ascending c, pages in
 * ascending table index), their table entries set to -1; len[c] = n_new;
 * *free_top grows by the pages pushed.  Must follow rkv_score_select of the
 * same step with no append in between.
 * Errors: RKV_ERR_INVALID_ARG, RKV_ERR_WORKSPACE_TOO_SMALL, RKV_ERR_CUDA.
 */
RKV_API int rkv_compact_pages(const rkv_cache_t *cache, const rkv_select_t *sel, void *ws,
                              size_t ws_bytes, void *stream);

/* ---------------------------------------------------------------------------
 * rkv_append -- write the decoded token of every sequence into every head:
 * slot len[c] receives k_new[c], v_new[c], position t[b] and lb_new[c];
 * when len[c] % 16 == 0 the head first pops a page from the top of the free
 * stack (heads in ascending c); len[c] += 1.
 *   t         [B] int32
 *   k_new, v_new [C][D] of the pool dtype
 *   lb_new    [C] float
 * Errors: RKV_ERR_INVALID_ARG, RKV_ERR_WORKSPACE_TOO_SMALL, RKV_ERR_CUDA.
 * Device: RKV_DEV_POOL_EXHAUSTED, RKV_DEV_TABLE_OVERFLOW, RKV_DEV_BAD_INPUT
 * (negative len): the head is skipped and keeps its length; a head whose
 * table is full takes no page, so later heads still pop in order.
 */
RKV_API int rkv_append(const rkv_cache_t *cache, const int32_t *t, const void *k_new,
                       const void *v_new, const float *lb_new, void *ws, size_t ws_bytes,
                       void *stream);

/* ---------------------------------------------------------------------------
 * rkv_decode_step -- one whole decode step in one launch, with the results
 * of the separate calls
 *     m_global != NULL:  rkv_score_select -> rkv_paged_decode_attn (with
 *                        the selection, dropped mass included) ->
 *                        rkv_compact_pages -> rkv_append
 *     m_global == NULL:  rkv_paged_decode_attn (every entry kept) ->
 *                        rkv_append  (a step that evicts nothing)
 * Selection outputs, keep masks, block tables, lengths, pools and the free
 * stack are identical to those calls; out / lse_kept / dropped agree with
 * them within floating-point rounding (the sums are grouped differently).
 *
 * Steady decoding keeps each sequence's threshold in a window inside the
 * workspace (shared with rkv_score_select): entries whose keys fall outside
 * the previous call's window are classified while their K/V stream through
 * the attention, the few inside it are ranked after one grid barrier.  When
 * the window cannot decide (first call on a workspace, a prefill-sized
 * eviction, a sharp change of scores) the exact radix selection runs inside
 * the same launch before the attention, so the result never depends on the
 * window -- only the time does.
 *
 *   t, q, scale, out, lse_kept, dropped   as rkv_paged_decode_attn
 *   m_global  [B] int64 or NULL   budgets, as rkv_score_select
 *   k_new, v_new, lb_new          as rkv_append
 *   sel       selection outputs (required when m_global != NULL; kappa,
 *             kept, n_pre, keep_mask and plan are written)
 * Limits: B <= 64; B*L*H <= 384 * (SM count); the (dtype, D, G) instances
 * of rkv_paged_decode_attn; max_pages small enough for the compaction
 * scratch in shared memory (about 14 bytes per page on top of the
 * attention stages).  q, k_new, v_new, pos_pool and lb_pool 16-byte aligned.
 * Errors: RKV_ERR_INVALID_ARG, RKV_ERR_UNSUPPORTED,
 * RKV_ERR_WORKSPACE_TOO_SMALL, RKV_ERR_CUDA.  Device: RKV_DEV_BAD_INPUT,
 * RKV_DEV_POOL_EXHAUSTED, RKV_DEV_TABLE_OVERFLOW, RKV_DEV_TIMEOUT (then
 * re-initialise the workspace).  One cooperative launch, one CTA per SM.
 */
RKV_API int rkv_decode_step(const rkv_cache_t *cache, const int32_t *t, const int64_t *m_global,
                            const float *q, float scale, const void *k_new, const void *v_new,
                            const float *lb_new, const rkv_select_t *sel, float *out, float *lse_kept,
                            float *dropped, void *ws, size_t ws_bytes, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* RKV_H_ */
