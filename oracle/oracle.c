/*
 * oracle.c -- plain, slow CPU reference for one decode step of
 * retention-scored, globally budgeted KV-cache eviction followed by
 * attention over the kept entries.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the bench's
 * CPU-baseline / reference leg load this library.  The product (the CUDA
 * library librkv.so and its Python binding) never calls it, and the two share
 * no source file, header, table or helper.
 *
 * What it follows (web summaries of three papers):
 *   [DBTrimKV]  "Make Each Token Count: Towards Improving Long-Context
 *               Performance with KV Cache Eviction"
 *               - Methodology 2, geometric retention as future utility:
 *                 the retention weight of token i at step t is beta_i^(t-i).
 *               - Methodology 3, weight-tied global gate: one global budget
 *                 M_global; all cached entries of all layers and heads are
 *                 ranked together and the top M_global are kept.
 *               - Methodology 4, implementation: paged layout with a
 *                 variable-length KV sequence per head.
 *   [TRIM-KV]   "Cache What Lasts: Token Retention for Memory-Bounded KV
 *               Cache in LLMs", technical summary, core mechanisms 1, 2, 4:
 *               beta in [0,1] per token, layer and head; decay beta^(t-i);
 *               when over budget, evict the lowest beta^(t-i).
 *   [ContourKV] "Trust the Mass: Forced Weights in KV-Cache Eviction"
 *               - Problem definition: after selection the attention weights
 *                 are renormalised over the kept set (forced weights).
 *               - Methodology 2: the budget is enforced physically (ragged
 *                 storage), not as a mask over the full cache.
 *               - Methodology 3 / main contributions: dropped mass, the
 *                 summed dense attention weight of the discarded keys.
 *               - Methodology 1: the eviction error ||mu - m_A|| between
 *                 the dense output and the forced-weight output.
 *   [IndexMem]  "learned KV eviction with latent memory", Methodology B:
 *               evicted tokens folded into a decayed outer-product state
 *               that a gated read adds back to the attention output.
 *
 * Readings where the pages are silent:
 *   - score s = fl32(float(t - i) * log(beta_i)), one IEEE binary32 multiply
 *     (log beta^(t-i) = (t-i) log beta); -0 is the same score as +0;
 *   - ties broken by ascending (layer, kv head, position);
 *   - entries present at step t are those with position < t;
 *   - logits use scale = 1/sqrt(D) (passed in); K/V bf16 values are widened
 *     exactly; attention is accumulated in binary64;
 *   - the pages fix no paged layout: the hole-fill compaction and the
 *     free-page stack below are a layout rule of this implementation, stated
 *     so that tables and pools can be compared bit for bit.
 *
 * Build: gcc -O2 -std=c99 -ffp-contract=off -fexcess-precision=standard
 *        -fno-fast-math -shared -fPIC (no FMA contraction: the score must be
 *        exactly one rounded multiply).  The same source built with -fopenmp
 *        runs the attention's independent heads on several threads (each
 *        head's sums keep their order, so the results are the same bits);
 *        only the CPU timing of the benchmark uses that build.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORC_OK 0
#define ORC_ERR_INPUT (-1) /* NaN log-retention, age outside [1, 2^24), bad layout */
#define ORC_ERR_POOL (-2)  /* free-page stack empty on append */
#define ORC_ERR_TABLE (-3) /* append past the end of a block table */

/* The cache, in the layout both sides agree on.  C = B*L*H heads; head
 * c = (b*L + l)*H + h.  Logical slot k of head c lives in physical page
 * block_table[c*max_pages + k/P] at offset k%P. */
typedef struct {
    int32_t B, L, H, G, D, P;
    int32_t n_pages, max_pages;
    int32_t kv_f32;      /* 1: K/V stored as float; 0: bfloat16 bit patterns */
    void *k_pool;        /* [n_pages][P][D] */
    void *v_pool;        /* [n_pages][P][D] */
    int32_t *pos_pool;   /* [n_pages][P] token position i */
    float *lb_pool;      /* [n_pages][P] log retention log(beta_i) */
    int32_t *block_table;/* [C][max_pages], -1 where no page */
    int32_t *len;        /* [C] entries per head */
    int32_t *free_stack; /* [n_pages] free page ids, top at free_stack[*free_top-1] */
    int32_t *free_top;   /* scalar */
} orc_cache;

static int64_t n_heads(const orc_cache *cc) { return (int64_t)cc->B * cc->L * cc->H; }

/* Threads the attention may use: sets them when n > 0 (OpenMP builds only)
 * and returns the number in effect (1 in a build without OpenMP). */
int orc_threads(int n) {
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
    return omp_get_max_threads();
#else
    (void)n;
    return 1;
#endif
}

static int64_t phys_row(const orc_cache *cc, int64_t c, int32_t k) {
    int32_t page = cc->block_table[c * cc->max_pages + k / cc->P];
    return (int64_t)page * cc->P + k % cc->P;
}

/* Widen one stored K or V element to binary64 (bf16 -> f32 is a 16-bit shift). */
static double kv_elem(const orc_cache *cc, const void *pool, int64_t row, int32_t d) {
    if (cc->kv_f32) return (double)((const float *)pool)[row * cc->D + d];
    uint32_t bits = (uint32_t)((const uint16_t *)pool)[row * cc->D + d] << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return (double)f;
}

/* ---------------------------------------------------------------- score ---
 * [DBTrimKV] Methodology 2 / [TRIM-KV] core mechanism 2: r_{t,i} = beta_i^(t-i).
 * In log space log r = (t-i) * log beta_i; one binary32 multiply, round to
 * nearest even.  The age t-i is an exact integer in [1, 2^24), so its
 * conversion to float is exact.  -0 is returned as +0. */
float orc_score(int32_t t, int32_t pos, float lb) {
    float age = (float)(t - pos);
    float s = age * lb;
    if (s == 0.0f) s = 0.0f;
    return s;
}

/* Validity of one entry's inputs: NaN log-retention or an age outside
 * [1, 2^24) is refused. */
int orc_entry_ok(int32_t t, int32_t pos, float lb) {
    int64_t age = (int64_t)t - (int64_t)pos;
    if (isnan(lb)) return 0;
    if (age < 1 || age >= (1 << 24)) return 0;
    return 1;
}

/* Element-wise orc_score / orc_entry_ok over arrays (for the pins). */
void orc_score_many(int64_t n, const int32_t *t, const int32_t *pos, const float *lb,
                    float *s, uint8_t *ok) {
    for (int64_t e = 0; e < n; e++) {
        ok[e] = (uint8_t)orc_entry_ok(t[e], pos[e], lb[e]);
        s[e] = ok[e] ? orc_score(t[e], pos[e], lb[e]) : 0.0f;
    }
}

/* --------------------------------------------------------------- select ---
 * [DBTrimKV] Methodology 3: rank every cached entry of all layers and heads
 * of a sequence by its score and keep the top M_global (per sequence).
 * [TRIM-KV] core mechanism 4: the lowest scores are the ones evicted.
 * Order: higher score first; equal scores by ascending (l, h, i). */
typedef struct {
    float s;
    int32_t l, h, i;
    int64_t c;
    int32_t slot;
} orc_entry;

static int cmp_rank(const void *pa, const void *pb) {
    const orc_entry *a = (const orc_entry *)pa, *b = (const orc_entry *)pb;
    if (a->s > b->s) return -1;
    if (a->s < b->s) return 1;
    if (a->l != b->l) return a->l < b->l ? -1 : 1;
    if (a->h != b->h) return a->h < b->h ? -1 : 1;
    if (a->i != b->i) return a->i < b->i ? -1 : 1;
    return 0;
}

/* keep[c*max_pages*P + k] = 1 for kept slots (0 otherwise, also past len);
 * kept[c] = number kept in head c.  t[b], m_global[b] per sequence. */
int orc_select(const orc_cache *cc, const int32_t *t, const int64_t *m_global,
               uint8_t *keep, int32_t *kept) {
    const int64_t C = n_heads(cc);
    const int64_t slots_per_head = (int64_t)cc->max_pages * cc->P;
    memset(keep, 0, (size_t)(C * slots_per_head));
    for (int64_t c = 0; c < C; c++) kept[c] = 0;
    for (int32_t b = 0; b < cc->B; b++) {
        int64_t n = 0;
        for (int32_t l = 0; l < cc->L; l++)
            for (int32_t h = 0; h < cc->H; h++) n += cc->len[((int64_t)b * cc->L + l) * cc->H + h];
        orc_entry *e = (orc_entry *)malloc((size_t)(n > 0 ? n : 1) * sizeof(orc_entry));
        if (!e) return ORC_ERR_INPUT;
        int64_t w = 0;
        for (int32_t l = 0; l < cc->L; l++) {
            for (int32_t h = 0; h < cc->H; h++) {
                int64_t c = ((int64_t)b * cc->L + l) * cc->H + h;
                for (int32_t k = 0; k < cc->len[c]; k++) {
                    int64_t row = phys_row(cc, c, k);
                    int32_t pos = cc->pos_pool[row];
                    float lb = cc->lb_pool[row];
                    if (!orc_entry_ok(t[b], pos, lb)) { free(e); return ORC_ERR_INPUT; }
                    e[w].s = orc_score(t[b], pos, lb);
                    e[w].l = l; e[w].h = h; e[w].i = pos; e[w].c = c; e[w].slot = k;
                    w++;
                }
            }
        }
        qsort(e, (size_t)n, sizeof(orc_entry), cmp_rank);
        int64_t m = m_global[b] < 0 ? 0 : m_global[b];
        if (m > n) m = n;
        for (int64_t r = 0; r < m; r++) {
            keep[e[r].c * slots_per_head + e[r].slot] = 1;
            kept[e[r].c] += 1;
        }
        free(e);
    }
    return ORC_OK;
}

/* Query row of query head g of KV head c (grouped-query attention: query
 * head h*G + g of a layer reads KV head h). */
static const float *query_of(const float *q, int64_t c, int32_t g, int32_t G, int32_t D) {
    return q + (c * G + g) * D;
}

/* Logits z_k = scale * <q, k_k> of every entry (slot order) of head c, in
 * binary64 over the exactly widened K elements. */
static void head_logits(const orc_cache *cc, int64_t c, const float *qv, float scale, double *z) {
    const int32_t n = cc->len[c], D = cc->D;
    for (int32_t k = 0; k < n; k++) {
        int64_t row = phys_row(cc, c, k);
        double dot = 0.0;
        for (int32_t d = 0; d < D; d++) dot += (double)qv[d] * kv_elem(cc, cc->k_pool, row, d);
        z[k] = (double)scale * dot;
    }
}

/* ------------------------------------------------------- per-head budget ---
 * [TRIM-KV] core mechanism 4 (inference eviction) with a budget for each
 * head: a head over its budget drops the entries with the lowest current
 * retention beta^(t-i) (the pages' analogy, section 3: a backpack of fixed
 * size drops its least valuable item).  [DBTrimKV] Methodology 3 names this
 * fixed per-head allocation as what its single global budget replaces.
 * Head c keeps its top m_head[c] entries by score (negative = 0); equal
 * scores by ascending position. */
typedef struct {
    float s;
    int32_t i;
    int32_t slot;
} orc_head_entry;

static int cmp_head_rank(const void *pa, const void *pb) {
    const orc_head_entry *a = (const orc_head_entry *)pa, *b = (const orc_head_entry *)pb;
    if (a->s > b->s) return -1;
    if (a->s < b->s) return 1;
    if (a->i != b->i) return a->i < b->i ? -1 : 1;
    return 0;
}

static int cmp_recent(const void *pa, const void *pb) {
    const orc_head_entry *a = (const orc_head_entry *)pa, *b = (const orc_head_entry *)pb;
    if (a->i != b->i) return a->i > b->i ? -1 : 1;
    return 0;
}

/* The entries of head c (sequence b) with their scores; NULL on bad input. */
static orc_head_entry *head_entries(const orc_cache *cc, int64_t c, int32_t t, int32_t *n_out) {
    const int32_t n = cc->len[c];
    orc_head_entry *e = (orc_head_entry *)malloc((size_t)(n > 0 ? n : 1) * sizeof(orc_head_entry));
    if (!e) return NULL;
    for (int32_t k = 0; k < n; k++) {
        int64_t row = phys_row(cc, c, k);
        int32_t pos = cc->pos_pool[row];
        float lb = cc->lb_pool[row];
        if (!orc_entry_ok(t, pos, lb)) { free(e); return NULL; }
        e[k].s = orc_score(t, pos, lb);
        e[k].i = pos;
        e[k].slot = k;
    }
    *n_out = n;
    return e;
}

int orc_select_per_head(const orc_cache *cc, const int32_t *t, const int32_t *m_head, uint8_t *keep,
                        int32_t *kept) {
    const int64_t C = n_heads(cc);
    const int64_t LH = (int64_t)cc->L * cc->H;
    const int64_t slots_per_head = (int64_t)cc->max_pages * cc->P;
    memset(keep, 0, (size_t)(C * slots_per_head));
    for (int64_t c = 0; c < C; c++) {
        int32_t n = 0;
        orc_head_entry *e = head_entries(cc, c, t[c / LH], &n);
        if (!e) return ORC_ERR_INPUT;
        qsort(e, (size_t)n, sizeof(orc_head_entry), cmp_head_rank);
        int32_t m = m_head[c] < 0 ? 0 : m_head[c];
        if (m > n) m = n;
        for (int32_t r = 0; r < m; r++) keep[c * slots_per_head + e[r].slot] = 1;
        kept[c] = m;
        free(e);
    }
    return ORC_OK;
}

/* --------------------------------------------------- ContourKV allocation ---
 * [ContourKV] Methodology 3: the dropped-mass statistic predicts the cells
 * (attention heads) whose top-mass selection stays far from the dense
 * output; those "flat" cells get a fixed budget directly, every cell keeps a
 * recency floor, and the importance scores of an existing method are reused
 * with this allocation in place of its own (here the retention scores and
 * the global order of [DBTrimKV] Methodology 3).  Readings:
 *   - a cell is a KV head c; its statistic is the mean of its G query
 *     heads' dropped mass at the previous evicting step, dm_prev[c][g],
 *     summed in ascending g and divided by G in binary32; flat iff > tau;
 *   - 1. every head keeps its floor: its min(r, len) most recent entries
 *     (largest positions; positions within a head are distinct);
 *   - 2. a flat head also keeps the top flat_budget of its other entries
 *     (score descending, equal scores by ascending position);
 *   - 3. the rest of the sequence's budget, M_rest = max(0, M_global -
 *     entries kept by 1 and 2), goes to the global order (score descending,
 *     equal scores by ascending (layer, head, position)) over the remaining
 *     entries of the non-flat heads.
 * Floors and flat budgets are kept even when they exceed M_global.
 * flat_out[C] (may be NULL) receives 1 for the flat heads. */
int orc_select_contour(const orc_cache *cc, const int32_t *t, const int64_t *m_global, const float *dm_prev,
                       float tau, int32_t flat_budget, int32_t floor_r, uint8_t *keep, int32_t *kept,
                       uint8_t *flat_out) {
    const int64_t C = n_heads(cc);
    const int64_t LH = (int64_t)cc->L * cc->H;
    const int64_t slots_per_head = (int64_t)cc->max_pages * cc->P;
    memset(keep, 0, (size_t)(C * slots_per_head));
    for (int64_t c = 0; c < C; c++) kept[c] = 0;
    for (int32_t b = 0; b < cc->B; b++) {
        int64_t forced = 0, rest_n = 0;
        for (int64_t cl = 0; cl < LH; cl++) rest_n += cc->len[b * LH + cl];
        orc_entry *rest = (orc_entry *)malloc((size_t)(rest_n > 0 ? rest_n : 1) * sizeof(orc_entry));
        if (!rest) return ORC_ERR_INPUT;
        int64_t w = 0;
        for (int64_t cl = 0; cl < LH; cl++) {
            const int64_t c = b * LH + cl;
            float sum = 0.0f;
            for (int32_t g = 0; g < cc->G; g++) sum += dm_prev[c * cc->G + g];
            const float mean = sum / (float)cc->G;
            const int flat = mean > tau;
            if (flat_out) flat_out[c] = (uint8_t)flat;
            int32_t n = 0;
            orc_head_entry *e = head_entries(cc, c, t[b], &n);
            if (!e) { free(rest); return ORC_ERR_INPUT; }
            /* 1. the floor: the most recent entries */
            qsort(e, (size_t)n, sizeof(orc_head_entry), cmp_recent);
            int32_t nf = floor_r < 0 ? 0 : (floor_r > n ? n : floor_r);
            for (int32_t r = 0; r < nf; r++) keep[c * slots_per_head + e[r].slot] = 1;
            kept[c] += nf;
            /* 2. a flat head's fixed budget over its other entries */
            if (flat) {
                qsort(e + nf, (size_t)(n - nf), sizeof(orc_head_entry), cmp_head_rank);
                int32_t m = flat_budget < 0 ? 0 : flat_budget;
                if (m > n - nf) m = n - nf;
                for (int32_t r = nf; r < nf + m; r++) keep[c * slots_per_head + e[r].slot] = 1;
                kept[c] += m;
            } else {
                for (int32_t r = nf; r < n; r++) {
                    rest[w].s = e[r].s;
                    rest[w].l = (int32_t)(cl / cc->H);
                    rest[w].h = (int32_t)(cl % cc->H);
                    rest[w].i = e[r].i;
                    rest[w].c = c;
                    rest[w].slot = e[r].slot;
                    w++;
                }
            }
            forced += kept[c];
            free(e);
        }
        /* 3. the rest of the budget, globally over the non-flat heads */
        qsort(rest, (size_t)w, sizeof(orc_entry), cmp_rank);
        int64_t m = m_global[b] - forced;
        if (m < 0) m = 0;
        if (m > w) m = w;
        for (int64_t r = 0; r < m; r++) {
            keep[rest[r].c * slots_per_head + rest[r].slot] = 1;
            kept[rest[r].c] += 1;
        }
        free(rest);
    }
    return ORC_OK;
}

/* ------------------------------------------------------------ attention ---
 * [ContourKV] Problem definition: once the subset is chosen, the weights are
 * the softmax renormalised over the kept set (forced weights):
 *   o = sum_{j kept} exp(z_j - m) v_j / sum_{j kept} exp(z_j - m),
 *   z_j = scale * <q, k_j>.
 * [ContourKV] Methodology 3 / main contributions: dropped mass is the weight
 * the discarded keys held under dense attention over every entry present
 * before this step's eviction:
 *   dm = sum_{j evicted} exp(z_j - M) / sum_{j all} exp(z_j - M).
 * Query head qh = h*G + g of layer l reads KV head h (grouped-query attention
 * with consecutive query heads per group).  q, out: [C][G][D]; lse, dm: [C][G].
 * keep == NULL means every entry is kept.  A head with nothing kept gives
 * o = 0 and lse = -inf; a head with no entries has dm = 0. */
int orc_attention(const orc_cache *cc, const float *q, float scale, const uint8_t *keep,
                  float *out, float *lse_kept, float *dropped) {
    const int64_t C = n_heads(cc);
    const int64_t slots_per_head = (int64_t)cc->max_pages * cc->P;
    const int32_t D = cc->D, G = cc->G;
    int32_t max_len = 0;
    int failed = 0;
    for (int64_t c = 0; c < C; c++) if (cc->len[c] > max_len) max_len = cc->len[c];
    /* heads are independent: each thread has its own logit and sum buffers */
#pragma omp parallel
    {
        double *z = (double *)malloc((size_t)(max_len > 0 ? max_len : 1) * sizeof(double));
        double *acc = (double *)malloc((size_t)D * sizeof(double));
        if (!z || !acc) {
#pragma omp atomic write
            failed = 1;
        }
#pragma omp for schedule(dynamic, 1)
        for (int64_t c = 0; c < C; c++) {
            if (!z || !acc) continue;
            const int32_t n = cc->len[c];
            for (int32_t g = 0; g < G; g++) {
                head_logits(cc, c, query_of(q, c, g, G, D), scale, z);
                /* dense over all entries present before eviction */
                double m_all = -INFINITY;
                for (int32_t k = 0; k < n; k++) if (z[k] > m_all) m_all = z[k];
                double z_all = 0.0, z_ev = 0.0;
                for (int32_t k = 0; k < n; k++) {
                    double p = exp(z[k] - m_all);
                    z_all += p;
                    if (keep && !keep[c * slots_per_head + k]) z_ev += p;
                }
                if (dropped) dropped[c * G + g] = (float)(n > 0 ? z_ev / z_all : 0.0);
                /* forced weights over the kept set */
                double m_k = -INFINITY;
                int32_t n_kept = 0;
                for (int32_t k = 0; k < n; k++) {
                    if (keep && !keep[c * slots_per_head + k]) continue;
                    n_kept++;
                    if (z[k] > m_k) m_k = z[k];
                }
                double zk = 0.0;
                for (int32_t d = 0; d < D; d++) acc[d] = 0.0;
                for (int32_t k = 0; k < n; k++) {
                    if (keep && !keep[c * slots_per_head + k]) continue;
                    double p = exp(z[k] - m_k);
                    int64_t row = phys_row(cc, c, k);
                    zk += p;
                    for (int32_t d = 0; d < D; d++) acc[d] += p * kv_elem(cc, cc->v_pool, row, d);
                }
                float *o = out + (c * G + g) * D;
                for (int32_t d = 0; d < D; d++) o[d] = (float)(n_kept > 0 ? acc[d] / zk : 0.0);
                if (lse_kept) lse_kept[c * G + g] = (float)(n_kept > 0 ? m_k + log(zk) : -INFINITY);
            }
        }
        free(z);
        free(acc);
    }
    return failed ? ORC_ERR_INPUT : ORC_OK;
}

/* ------------------------------------------------------- eviction error ---
 * [ContourKV] Methodology 1 (theoretical analysis and enumeration): a kept
 * subset A is scored by the distance between the dense attention output mu
 * and the forced-weight output m_A over A:
 *   e(A) = || mu - m_A ||,
 *   mu  = sum_{j all}  exp(z_j) v_j / sum_{j all}  exp(z_j),
 *   m_A = sum_{j in A} exp(z_j) v_j / sum_{j in A} exp(z_j),
 * "all" = every entry of the head present before this step's eviction.
 * Readings: the norm is the Euclidean norm over the head dimension, per
 * query head; a head with no entries has e = 0; with nothing kept m_A = 0 (as
 * in orc_attention), so e = ||mu||; keep == NULL means A is every entry.
 * err [C][G]; mu_out [C][G][D] receives mu (may be NULL). */
int orc_eviction_error(const orc_cache *cc, const float *q, float scale, const uint8_t *keep,
                       float *err, float *mu_out) {
    const int64_t C = n_heads(cc);
    const int64_t slots_per_head = (int64_t)cc->max_pages * cc->P;
    const int32_t D = cc->D, G = cc->G;
    int32_t max_len = 0;
    int failed = 0;
    for (int64_t c = 0; c < C; c++) if (cc->len[c] > max_len) max_len = cc->len[c];
#pragma omp parallel
    {
        double *z = (double *)malloc((size_t)(max_len > 0 ? max_len : 1) * sizeof(double));
        double *mu = (double *)malloc((size_t)D * sizeof(double));
        double *ma = (double *)malloc((size_t)D * sizeof(double));
        if (!z || !mu || !ma) {
#pragma omp atomic write
            failed = 1;
        }
#pragma omp for schedule(dynamic, 1)
        for (int64_t c = 0; c < C; c++) {
            if (!z || !mu || !ma) continue;
            const int32_t n = cc->len[c];
            for (int32_t g = 0; g < G; g++) {
                head_logits(cc, c, query_of(q, c, g, G, D), scale, z);
                /* mu: softmax over every entry */
                double m_all = -INFINITY;
                for (int32_t k = 0; k < n; k++) if (z[k] > m_all) m_all = z[k];
                double s_all = 0.0;
                for (int32_t d = 0; d < D; d++) mu[d] = 0.0;
                for (int32_t k = 0; k < n; k++) {
                    double p = exp(z[k] - m_all);
                    int64_t row = phys_row(cc, c, k);
                    s_all += p;
                    for (int32_t d = 0; d < D; d++) mu[d] += p * kv_elem(cc, cc->v_pool, row, d);
                }
                for (int32_t d = 0; d < D; d++) mu[d] = n > 0 ? mu[d] / s_all : 0.0;
                /* m_A: softmax over the kept entries only */
                double m_k = -INFINITY;
                int32_t n_kept = 0;
                for (int32_t k = 0; k < n; k++) {
                    if (keep && !keep[c * slots_per_head + k]) continue;
                    n_kept++;
                    if (z[k] > m_k) m_k = z[k];
                }
                double s_k = 0.0;
                for (int32_t d = 0; d < D; d++) ma[d] = 0.0;
                for (int32_t k = 0; k < n; k++) {
                    if (keep && !keep[c * slots_per_head + k]) continue;
                    double p = exp(z[k] - m_k);
                    int64_t row = phys_row(cc, c, k);
                    s_k += p;
                    for (int32_t d = 0; d < D; d++) ma[d] += p * kv_elem(cc, cc->v_pool, row, d);
                }
                for (int32_t d = 0; d < D; d++) ma[d] = n_kept > 0 ? ma[d] / s_k : 0.0;
                double sq = 0.0;
                for (int32_t d = 0; d < D; d++) sq += (mu[d] - ma[d]) * (mu[d] - ma[d]);
                err[c * G + g] = (float)sqrt(sq);
                if (mu_out)
                    for (int32_t d = 0; d < D; d++) mu_out[(c * G + g) * D + d] = (float)mu[d];
            }
        }
        free(z);
        free(mu);
        free(ma);
    }
    return failed ? ORC_ERR_INPUT : ORC_OK;
}

/* -------------------------------------------------------- latent memory ---
 * IndexMem ("learned KV eviction with latent memory"), Methodology B: the
 * evicted tokens update a fixed-size state matrix M and a stabilising
 * vector b online, by outer-product accumulation with decay (fast
 * weights); learned projections and a gate g(q) read it (slow weights);
 * the output is o = o_attn + g(q) * m(q).  Readings (the page gives no
 * formulas; this is the linear-attention form those words describe):
 *   - one state per KV head c: M_c [D][D], b_c [D];
 *   - feature map phi(x) = elu(P_l x) + 1 with a per-layer projection P_l
 *     [D][D] (D*D*L parameters: 0.5M for an 8B-class model, the size the
 *     page quotes for the memory), elu(y) = y for y > 0, exp(y) - 1 else;
 *   - update at an evicting step, with this step's evicted entries j of
 *     head c:  M_c = decay * M_c + sum_j phi(k_j) v_j^T,
 *              b_c = decay * b_c + sum_j phi(k_j);
 *   - read for query head (c, g):  m = phi(q)^T M_c / (phi(q)^T b_c), and
 *     m = 0 when phi(q)^T b_c = 0 (nothing ever evicted);
 *   - gate g(q) = sigmoid(w_{l,hq} . q + beta_{l,hq});  out += g * m.
 * The update runs after the selection and before compaction (the evicted
 * rows are still in place); the read adds to the attention output. */
static double phi_of(double y) { return y > 0.0 ? y + 1.0 : exp(y); }

/* Features phi(P_l x) of one D-vector x (float or stored K element). */
static void features(const float *P, const double *x, int32_t D, double *f) {
    for (int32_t i = 0; i < D; i++) {
        double y = 0.0;
        for (int32_t d = 0; d < D; d++) y += (double)P[(int64_t)i * D + d] * x[d];
        f[i] = phi_of(y);
    }
}

int orc_memory_update(const orc_cache *cc, const uint8_t *keep, const float *proj, double decay, double *M,
                      double *bvec) {
    const int64_t C = n_heads(cc);
    const int64_t LH = (int64_t)cc->L * cc->H;
    const int64_t slots_per_head = (int64_t)cc->max_pages * cc->P;
    const int32_t D = cc->D;
    double *k = (double *)malloc((size_t)D * sizeof(double));
    double *f = (double *)malloc((size_t)D * sizeof(double));
    if (!k || !f) { free(k); free(f); return ORC_ERR_INPUT; }
    for (int64_t c = 0; c < C; c++) {
        const int32_t l = (int32_t)((c % LH) / cc->H);
        const float *P = proj + (int64_t)l * D * D;
        double *Mc = M + c * (int64_t)D * D, *bc = bvec + c * D;
        for (int64_t e = 0; e < (int64_t)D * D; e++) Mc[e] *= decay;
        for (int32_t i = 0; i < D; i++) bc[i] *= decay;
        for (int32_t s = 0; s < cc->len[c]; s++) {
            if (keep[c * slots_per_head + s]) continue;
            const int64_t row = phys_row(cc, c, s);
            for (int32_t d = 0; d < D; d++) k[d] = kv_elem(cc, cc->k_pool, row, d);
            features(P, k, D, f);
            for (int32_t i = 0; i < D; i++) {
                bc[i] += f[i];
                for (int32_t j = 0; j < D; j++) Mc[(int64_t)i * D + j] += f[i] * kv_elem(cc, cc->v_pool, row, j);
            }
        }
    }
    free(k);
    free(f);
    return ORC_OK;
}

int orc_memory_read(const orc_cache *cc, const float *q, const float *proj, const float *gate_w,
                    const float *gate_b, const double *M, const double *bvec, float *out) {
    const int64_t C = n_heads(cc);
    const int64_t LH = (int64_t)cc->L * cc->H;
    const int32_t D = cc->D, G = cc->G;
    double *x = (double *)malloc((size_t)D * sizeof(double));
    double *f = (double *)malloc((size_t)D * sizeof(double));
    if (!x || !f) { free(x); free(f); return ORC_ERR_INPUT; }
    for (int64_t c = 0; c < C; c++) {
        const int32_t l = (int32_t)((c % LH) / cc->H);
        const int32_t h = (int32_t)(c % cc->H);
        const float *P = proj + (int64_t)l * D * D;
        const double *Mc = M + c * (int64_t)D * D, *bc = bvec + c * D;
        for (int32_t g = 0; g < G; g++) {
            const float *qv = query_of(q, c, g, G, D);
            const int64_t hq = (int64_t)l * cc->H * G + (int64_t)h * G + g;  /* query head of the layer */
            for (int32_t d = 0; d < D; d++) x[d] = (double)qv[d];
            features(P, x, D, f);
            double den = 0.0, z = (double)gate_b[hq];
            for (int32_t i = 0; i < D; i++) den += f[i] * bc[i];
            for (int32_t d = 0; d < D; d++) z += (double)gate_w[hq * D + d] * x[d];
            const double gate = 1.0 / (1.0 + exp(-z));
            float *o = out + (c * G + g) * D;
            for (int32_t j = 0; j < D; j++) {
                double num = 0.0;
                for (int32_t i = 0; i < D; i++) num += f[i] * Mc[(int64_t)i * D + j];
                o[j] = (float)((double)o[j] + (den > 0.0 ? gate * num / den : 0.0));
            }
        }
    }
    free(x);
    free(f);
    return ORC_OK;
}

/* ------------------------------------------------------------ compaction ---
 * [ContourKV] Methodology 2: the kept set is stored physically (ragged
 * storage); evicted rows are really removed.  [DBTrimKV] Methodology 4: each
 * head keeps its own length in a paged layout.  The layout rule used here:
 * heads in ascending c; in head c with n entries and n_new kept,
 *   holes   = slots k < n_new that are not kept, ascending;
 *   sources = slots k >= n_new that are kept, ascending;
 * the j-th source's (K, V, position, log-retention) row is copied to the
 * j-th hole; the pages at table indices [ceil(n_new/P), ceil(n/P)) are pushed
 * onto the free stack in ascending table index, their table entries become
 * -1, and len = n_new. */
static void copy_row(const orc_cache *cc, int64_t dst, int64_t src) {
    size_t esz = cc->kv_f32 ? 4 : 2;
    memcpy((char *)cc->k_pool + dst * cc->D * esz, (char *)cc->k_pool + src * cc->D * esz, cc->D * esz);
    memcpy((char *)cc->v_pool + dst * cc->D * esz, (char *)cc->v_pool + src * cc->D * esz, cc->D * esz);
    cc->pos_pool[dst] = cc->pos_pool[src];
    cc->lb_pool[dst] = cc->lb_pool[src];
}

int orc_compact(orc_cache *cc, const uint8_t *keep) {
    const int64_t C = n_heads(cc);
    const int64_t slots_per_head = (int64_t)cc->max_pages * cc->P;
    for (int64_t c = 0; c < C; c++) {
        const uint8_t *f = keep + c * slots_per_head;
        const int32_t n = cc->len[c];
        int32_t n_new = 0;
        for (int32_t k = 0; k < n; k++) n_new += f[k] ? 1 : 0;
        int32_t hole = 0, src = n_new;
        for (;;) {
            while (hole < n_new && f[hole]) hole++;
            while (src < n && !f[src]) src++;
            if (hole >= n_new || src >= n) break;
            copy_row(cc, phys_row(cc, c, hole), phys_row(cc, c, src));
            hole++;
            src++;
        }
        const int32_t keep_pages = (n_new + cc->P - 1) / cc->P;
        const int32_t old_pages = (n + cc->P - 1) / cc->P;
        for (int32_t pi = keep_pages; pi < old_pages; pi++) {
            int32_t *slot = &cc->block_table[c * cc->max_pages + pi];
            cc->free_stack[(*cc->free_top)++] = *slot;
            *slot = -1;
        }
        cc->len[c] = n_new;
    }
    return ORC_OK;
}

/* --------------------------------------------------------------- append ---
 * Decoding writes token t's K, V, position t and log-retention into slot
 * len of every head, heads in ascending c.  When len is a multiple of P the
 * head first takes a page from the top of the free stack. */
int orc_append(orc_cache *cc, const int32_t *t, const void *k_new, const void *v_new,
               const float *lb_new) {
    const int64_t C = n_heads(cc);
    const size_t esz = cc->kv_f32 ? 4 : 2;
    for (int64_t c = 0; c < C; c++) {
        const int32_t b = (int32_t)(c / ((int64_t)cc->L * cc->H));
        const int32_t k = cc->len[c];
        if (k / cc->P >= cc->max_pages) return ORC_ERR_TABLE;
        if (k % cc->P == 0) {
            if (*cc->free_top <= 0) return ORC_ERR_POOL;
            cc->block_table[c * cc->max_pages + k / cc->P] = cc->free_stack[--(*cc->free_top)];
        }
        int64_t row = phys_row(cc, c, k);
        memcpy((char *)cc->k_pool + row * cc->D * esz, (const char *)k_new + c * cc->D * esz, cc->D * esz);
        memcpy((char *)cc->v_pool + row * cc->D * esz, (const char *)v_new + c * cc->D * esz, cc->D * esz);
        cc->pos_pool[row] = t[b];
        cc->lb_pool[row] = lb_new[c];
        cc->len[c] = k + 1;
    }
    return ORC_OK;
}
