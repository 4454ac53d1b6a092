// internal.h -- launch interfaces between the C ABI layer (api.cu) and the
// kernels.  Not installed; the public interface is include/rkv.h.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "../../include/rkv.h"
#include "common.cuh"

namespace rkv {

// Workspace layout, all offsets in bytes from the workspace base.
struct WsLayout {
    size_t status;        // int32, sticky RKV_DEV_* bits
    size_t done_compact;  // uint32, self-resetting completion counter
    size_t done_append;   // uint32, self-resetting completion counter
    size_t bar;           // uint32 grid-barrier counter (reset by the selection's last CTA)
    size_t leave;         // uint32 exit ticket of the selection
    size_t win;           // uint32 [B][4] threshold window per sequence (kept across calls)
    size_t cnt;           // uint32 [B][4] per-call counters: keys above the window, candidates, window outcome
    size_t kmax;          // uint64 [B] largest kept key (cleared at exit)
    size_t cand;          // uint2 [B][WIN_CAP] keys inside the window
    size_t more;          // uint32 [waves][NPASS] continuation flags (cleared at exit)
    size_t hist;          // uint32 [waves][NPASS][n_groups][NBINS] (cleared at exit)
    size_t head_cnt;      // uint32 [C], attention split-head arrival counters (self-resetting)
    size_t partial;       // float [MAX_ATTN_CTAS][2][rec], attention partial states
    // fused decode step (rkv_decode_step)
    size_t step_bar;      // uint32 grid-barrier counter (reset by the last CTA to leave)
    size_t step_leave;    // uint32 exit ticket
    size_t step_parity;   // uint32, which half of step_ctr this call uses (flipped at exit)
    size_t step_ctr;      // uint32 [2][ctr_words]: per-call counters, one half zeroed while the other is used
    size_t ckey;          // uint64 [B][WIN_CAP] keys of the window candidates
    size_t cslot;         // int32  [B][WIN_CAP] logical slot of each candidate in its head
    size_t cfate;         // int32  [B][WIN_CAP] 1 if the candidate is kept
    size_t cz;            // float  [B][WIN_CAP][G] base-2 logits of each candidate
    size_t cv;            // [B][WIN_CAP][row bytes] V row of each candidate (pool dtype)
    size_t ghist;         // uint32 [NPASS][B][NBINS] exact-select histograms (cleared after use)
    size_t hrec;          // float  [C][rec] state of whole heads that hold candidates
    size_t npre;          // int32  [C] pre-step lengths
    size_t pfx;           // int32  [C+1] page prefix of the pre-step lengths (own range of each CTA)
    size_t bmask;         // uint16 [C][max_pages] forced keep bits (ContourKV)
    size_t bkept;         // int32  [C] forced counts (ContourKV)
    size_t bfloor;        // int32  [C] oldest floor position (ContourKV)
    size_t bskip;         // uint8  [C] flat heads (ContourKV)
    size_t bseq;          // uint64 [B][2] forced entries, entries left to rank (ContourKV)
    size_t total;
};

// Per-call counters of the fused step: head_kept[C], head_flag[C],
// seq[B][4] (keys above the window, candidates), misc[16] (compaction arrivals).
inline size_t step_ctr_words(int64_t C, int B) { return (size_t)(2 * C + 4 * (int64_t)B + 16 + 63) / 64 * 64; }

// One int32 written on the device (compact.cu).
cudaError_t launch_set_word(int32_t *p, int32_t v, cudaStream_t s);

struct SelectGrid {
    int n_groups, cta_per_group, waves, threads, smem_bytes, cache_pages;
};

// Returns false if the shape cannot be laid out.
bool ws_layout(const rkv_cache_t &c, WsLayout *out);
SelectGrid select_grid_for(const rkv_cache_t &c, int sm_count);

struct SelectArgs {
    const int32_t *pos_pool;
    const float *lb_pool;
    const int32_t *block_table;
    const int32_t *len;
    const int32_t *free_top;
    int B, LH, C, max_pages, ibits;
    const int32_t *t;
    const int64_t *m_global;
    uint64_t *kappa;
    int32_t *kept;
    int32_t *n_pre;
    uint16_t *keep_mask;
    int32_t *plan;
    int32_t *status;
    uint32_t *bar;
    uint32_t *leave;
    uint32_t *win;
    uint32_t *cnt;
    unsigned long long *kmax;
    uint2 *cand;
    uint32_t *more;
    uint32_t *hist;
    int n_groups, cta_per_group, waves, cache_pages;
    // ContourKV's global part (all NULL otherwise): entries of heads with
    // skip[c] set and entries at positions >= floor_pos[c] are left out of
    // the ranking; pre_mask bits are ORed into the keep masks and pre_kept
    // added to the kept counts; the budget is min(max(0, m_global[b] -
    // seq[2b]), seq[2b+1]) (forced entries, entries left to rank); the
    // threshold window is neither read nor updated.
    const int32_t *floor_pos;
    const uint8_t *skip;
    const uint16_t *pre_mask;
    const int32_t *pre_kept;
    const unsigned long long *seq;
};
cudaError_t launch_select(const SelectArgs &a, const SelectGrid &g, cudaStream_t s);

// Budget variants (budget.cu): one CTA per head.
struct BudgetArgs {
    const int32_t *pos_pool;
    const float *lb_pool;
    const int32_t *block_table;
    const int32_t *len;
    const int32_t *t;
    int LH, C, G, max_pages;
    int mode;                  // RKV_BUDGET_PER_HEAD / RKV_BUDGET_CONTOUR
    const int32_t *m_head;     // [C] (per head)
    const float *dm_prev;      // [C][G] (ContourKV)
    float tau;
    int32_t flat_budget, floor_r;
    uint16_t *mask;            // keep masks (per head) / forced bits (ContourKV)
    int32_t *kept;             // kept (per head) / forced counts (ContourKV)
    int32_t *n_pre;            // per head
    int32_t *floor_pos;        // ContourKV: [C] oldest floor position (INT_MAX: none)
    uint8_t *skip;             // ContourKV: [C] flat heads
    unsigned long long *seq;   // ContourKV: [B][2] forced, entries left to rank (zeroed before)
    int32_t *status;
};
cudaError_t launch_head_budget(const BudgetArgs &a, cudaStream_t s);
cudaError_t launch_plan(const int32_t *n_pre, const int32_t *kept, int32_t *plan, const int32_t *free_top,
                        uint64_t *kappa, int C, int B, cudaStream_t s);

// Fixed scratch of the allocation-free selection (a __device__ array in
// select.cu): word offsets of its fields and its size.
constexpr int NOALLOC_MAX_B = 16;
constexpr int NOALLOC_MAX_DEVICES = 64;
constexpr size_t NOALLOC_STATUS = 0, NOALLOC_BAR = 16, NOALLOC_LEAVE = 32, NOALLOC_MORE = 64;
constexpr size_t NOALLOC_WIN = 192, NOALLOC_CNT = 256;     // [MAX_B][4] each
constexpr size_t NOALLOC_KMAX = 384;                        // uint64 [MAX_B]
constexpr size_t NOALLOC_HIST = 512;  // after the flags and counters, 2 KiB aligned
constexpr size_t NOALLOC_CAND = NOALLOC_HIST + (size_t)NOALLOC_MAX_B * NPASS * NBINS;
constexpr size_t NOALLOC_WORDS = NOALLOC_CAND + (size_t)NOALLOC_MAX_B * WIN_CAP * 2;
static_assert(NOALLOC_MORE + NOALLOC_MAX_B * NPASS <= NOALLOC_WIN, "flag region");
static_assert(NOALLOC_WIN + 4 * NOALLOC_MAX_B <= NOALLOC_CNT && NOALLOC_CNT + 4 * NOALLOC_MAX_B <= NOALLOC_KMAX &&
                  NOALLOC_KMAX + 2 * NOALLOC_MAX_B <= NOALLOC_HIST,
              "counter region");
// Device address of that array on the current device (looked up once per
// device); returns nonzero and sets *err on failure.
int noalloc_scratch(uint32_t **out, const char **err);
int select_max_smem();

struct AttnArgs {
    const void *k_pool;
    const void *v_pool;
    const int32_t *block_table;
    const int32_t *len;        // pre-compaction lengths
    const uint16_t *keep_mask; // NULL: every entry kept
    const float *q;
    float *out;                // NULL: dropped-mass only (V not read)
    float *lse;                // may be NULL
    float *dropped;            // may be NULL
    int32_t *status;
    uint32_t *head_cnt;
    float *partial;
    int C, max_pages;
    float qscale;              // scale * log2(e)
};
// Returns cudaErrorNotSupported if (dtype, D, G) is not instantiated.  bf16
// pools are read through the two tensor maps (64-column boxes of 16 rows,
// 128-byte swizzle); fp32 pools ignore them.
cudaError_t launch_attn(const AttnArgs &a, int dtype, int D, int G, int sm_count, cudaStream_t s,
                        const CUtensorMap &tk, const CUtensorMap &tv);
bool attn_supported(int dtype, int D, int G);
// Eviction error (evict_err.cu): per head, the forced-weight output of the
// evicted rows against the kept output: err = dropped * ||m_ev - out_kept||.
struct EvictErrArgs {
    const void *k_pool;
    const void *v_pool;
    const int32_t *block_table;
    const int32_t *n_pre;
    const uint16_t *keep_mask;
    const float *q;            // [C][G][D]
    const float *out_kept;     // [C][G][D]
    const float *dropped;      // [C][G]
    float *err;                // [C][G]
    float scale;
    int C, max_pages;
};
cudaError_t launch_evict_err(const EvictErrArgs &a, int dtype, int D, int G, cudaStream_t s);
bool attn_uses_tensor_maps(int dtype);
size_t attn_partial_rec_floats(int D, int G);

// Fused decode step: selection, attention with dropped mass, compaction and
// append in one cooperative launch (one CTA per SM).
constexpr int STEP_MAX_B = 64;      // sequences per call
constexpr int STEP_HEADS_PER_CTA = 384;  // C <= this * grid
struct StepArgs {
    void *k_pool;
    void *v_pool;
    int32_t *pos_pool;
    float *lb_pool;
    int32_t *block_table;
    int32_t *len;
    int32_t *free_stack;
    int32_t *free_top;
    int B, LH, C, max_pages, ibits, row_bytes;
    const int32_t *t;
    const int64_t *m_global;   // NULL: this step evicts nothing
    const float *q;
    float qscale;              // scale * log2(e)
    const void *k_new;
    const void *v_new;
    const float *lb_new;
    float *out;
    float *lse;                // may be NULL
    float *dropped;            // may be NULL
    uint64_t *kappa;           // selection outputs (evicting steps)
    int32_t *kept;
    int32_t *n_pre;
    uint16_t *keep_mask;
    int32_t *plan;
    int32_t *status;
    uint32_t *bar;
    uint32_t *leave;
    uint32_t *parity;
    uint32_t *ctr;             // [2][ctr_words]
    int ctr_words;
    uint32_t *win;             // [B][4], shared with the selection kernel
    uint64_t *ckey;
    int32_t *cslot;
    int32_t *cfate;
    float *cz;
    unsigned char *cv;
    uint32_t *ghist;
    float *partial;
    uint32_t *head_cnt;        // [C] cross-CTA merge tickets (self-resetting)
    float *hrec;
    int32_t *npre;
    int32_t *pfx;
};
bool step_supported(int dtype, int D, int G);
// Shared memory the step kernel needs for this shape (0: not supported).
size_t step_smem_bytes(int dtype, int D, int G, int max_pages);
cudaError_t launch_step(const StepArgs &a, int dtype, int D, int G, int grid, cudaStream_t s,
                        const CUtensorMap &tk, const CUtensorMap &tv);

// Latent memory (memory.cu).
struct MemUpdateArgs {
    const void *k_pool;
    const void *v_pool;
    const int32_t *block_table;
    const int32_t *n_pre;
    const uint16_t *keep_mask;
    const float *proj;         // [L][D][D]
    float decay;
    float *M;                  // [C][D][D]
    float *b;                  // [C][D]
    int C, LH, H, max_pages;
};
struct MemReadArgs {
    const float *q;            // [C][G][D]
    const float *proj;         // [L][D][D]
    const float *gate_w;       // [L][Hq][D]
    const float *gate_b;       // [L][Hq]
    const float *M;
    const float *b;
    float *out;                // [C][G][D], added to
    int C, LH, H, Hq;
};
bool memory_supported(int D, int G);
cudaError_t launch_memory_update(const MemUpdateArgs &a, int dtype, int D, cudaStream_t s);
cudaError_t launch_memory_read(const MemReadArgs &a, int D, int G, cudaStream_t s);

struct CompactArgs {
    void *k_pool;
    void *v_pool;
    int32_t *pos_pool;
    float *lb_pool;
    int32_t *block_table;
    int32_t *len;
    int32_t *free_stack;
    int32_t *free_top;
    const int32_t *kept;
    const int32_t *n_pre;
    const uint16_t *keep_mask;
    const int32_t *plan;
    uint32_t *done;
    int C, max_pages, row_bytes;
};
cudaError_t launch_compact(const CompactArgs &a, cudaStream_t s);

struct AppendArgs {
    void *k_pool;
    void *v_pool;
    int32_t *pos_pool;
    float *lb_pool;
    int32_t *block_table;
    int32_t *len;
    int32_t *free_stack;
    int32_t *free_top;
    const int32_t *t;
    const void *k_new;
    const void *v_new;
    const float *lb_new;
    int32_t *status;
    uint32_t *done;
    int C, LH, max_pages, row_bytes;
};
cudaError_t launch_append(const AppendArgs &a, cudaStream_t s);

}  // namespace rkv
