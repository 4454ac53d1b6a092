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
    size_t cnt;           // uint32 [B][4] per-call counters: keys above the window, candidates
    size_t cand;          // uint2 [B][WIN_CAP] keys inside the window
    size_t more;          // uint32 [waves][NPASS] continuation flags (cleared at exit)
    size_t hist;          // uint32 [waves][NPASS][n_groups][NBINS] (cleared at exit)
    size_t head_cnt;      // uint32 [C], attention split-head arrival counters (self-resetting)
    size_t partial;       // float [MAX_ATTN_CTAS][2][rec], attention partial states
    size_t total;
};

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
    uint2 *cand;
    uint32_t *more;
    uint32_t *hist;
    int n_groups, cta_per_group, waves, cache_pages;
};
cudaError_t launch_select(const SelectArgs &a, const SelectGrid &g, cudaStream_t s);

// Fixed scratch of the allocation-free selection (a __device__ array in
// select.cu): word offsets of its fields and its size.
constexpr int NOALLOC_MAX_B = 16;
constexpr int NOALLOC_MAX_DEVICES = 64;
constexpr size_t NOALLOC_STATUS = 0, NOALLOC_BAR = 16, NOALLOC_LEAVE = 32, NOALLOC_MORE = 64;
constexpr size_t NOALLOC_WIN = 192, NOALLOC_CNT = 256;     // [MAX_B][4] each
constexpr size_t NOALLOC_HIST = 512;  // after the flags and counters, 2 KiB aligned
constexpr size_t NOALLOC_CAND = NOALLOC_HIST + (size_t)NOALLOC_MAX_B * NPASS * NBINS;
constexpr size_t NOALLOC_WORDS = NOALLOC_CAND + (size_t)NOALLOC_MAX_B * WIN_CAP * 2;
static_assert(NOALLOC_MORE + NOALLOC_MAX_B * NPASS <= NOALLOC_WIN, "flag region");
static_assert(NOALLOC_WIN + 4 * NOALLOC_MAX_B <= NOALLOC_CNT && NOALLOC_CNT + 4 * NOALLOC_MAX_B <= NOALLOC_HIST,
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
bool attn_uses_tensor_maps(int dtype);
size_t attn_partial_rec_floats(int D, int G);

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
