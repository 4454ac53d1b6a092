// api.cu -- the C ABI of librkv (declared in include/rkv.h): argument
// validation, workspace layout and kernel launches on the caller's stream.
// No call allocates, frees or synchronises.
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <string>

#include <nvtx3/nvToolsExt.h>

#include "common.cuh"
#include "internal.h"

namespace rkv {
namespace {

thread_local std::string g_err;

int fail(int code, const char *fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof buf, fmt, ap);
    va_end(ap);
    g_err = buf;
    return code;
}

int cuda_fail(cudaError_t e, const char *what) {
    if (e == cudaErrorNotSupported) return fail(RKV_ERR_UNSUPPORTED, "%s: not supported for this shape", what);
    return fail(RKV_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int elt_bytes(int dtype) { return dtype == RKV_BF16 ? 2 : (dtype == RKV_F32 ? 4 : 0); }

// Shape and pointer checks shared by every entry point.
int check_cache(const rkv_cache_t *c, bool need_pools) {
    if (!c) return fail(RKV_ERR_INVALID_ARG, "cache is NULL");
    if (c->B <= 0 || c->L <= 0 || c->H <= 0 || c->Hq <= 0 || c->D <= 0)
        return fail(RKV_ERR_INVALID_ARG, "B, L, H, Hq, D must be positive");
    if (c->Hq % c->H != 0) return fail(RKV_ERR_INVALID_ARG, "Hq (%d) must be a multiple of H (%d)", c->Hq, c->H);
    if (c->P != PAGE) return fail(RKV_ERR_UNSUPPORTED, "page size must be 16 (got %d)", c->P);
    if (c->n_pages <= 0 || c->max_pages <= 0) return fail(RKV_ERR_INVALID_ARG, "n_pages and max_pages must be positive");
    if ((int64_t)c->n_pages * PAGE >= (1ll << 31)) return fail(RKV_ERR_UNSUPPORTED, "n_pages*16 must be < 2^31");
    if ((int64_t)c->max_pages * PAGE >= (1ll << 31)) return fail(RKV_ERR_UNSUPPORTED, "max_pages*16 must be < 2^31");
    const int64_t C = (int64_t)c->B * c->L * c->H;
    if (C >= (1ll << 31) || C * c->max_pages >= (1ll << 40)) return fail(RKV_ERR_UNSUPPORTED, "too many heads");
    const int eb = elt_bytes(c->dtype);
    if (!eb) return fail(RKV_ERR_INVALID_ARG, "dtype must be RKV_BF16 or RKV_F32");
    if ((c->D * eb) % 16 != 0) return fail(RKV_ERR_UNSUPPORTED, "row bytes D*elt must be a multiple of 16");
    if (!c->len || !c->block_table) return fail(RKV_ERR_INVALID_ARG, "len / block_table is NULL");
    if (need_pools) {
        if (!c->k_pool || !c->v_pool || !c->pos_pool || !c->lb_pool || !c->free_stack || !c->free_top)
            return fail(RKV_ERR_INVALID_ARG, "a cache pool pointer is NULL");
        if (!aligned16(c->k_pool) || !aligned16(c->v_pool))
            return fail(RKV_ERR_INVALID_ARG, "k_pool / v_pool must be 16-byte aligned");
    }
    return RKV_OK;
}

int check_sel(const rkv_select_t *s) {
    if (!s || !s->kappa || !s->kept || !s->n_pre || !s->keep_mask || !s->plan)
        return fail(RKV_ERR_INVALID_ARG, "selection buffers must all be non-NULL");
    return RKV_OK;
}

int lh_bits(int64_t LH) {
    int b = 0;
    while ((1ll << b) < LH) b++;
    return b;
}

// Select grid that depends only on the shape (upper bound for workspace sizing).
constexpr int MAX_SEL_CTAS = 1024;

void layout_for(const rkv_cache_t &c, int sel_groups_x_waves, WsLayout *L) {
    const int G = c.Hq / c.H;
    const int64_t C = (int64_t)c.B * c.L * c.H;
    size_t off = 0;
    auto take = [&](size_t bytes, size_t align) {
        off = (off + align - 1) / align * align;
        size_t at = off;
        off += bytes;
        return at;
    };
    L->status = take(32, 16);  // bits, first timeout site, fused steps in the window / exact, wait limit
    L->done_compact = take(4, 4);
    L->done_append = take(4, 4);
    L->bar = take(4, 64);
    L->leave = take(4, 64);
    L->win = take((size_t)c.B * 16, 16);
    L->cnt = take((size_t)c.B * 16, 16);
    L->kmax = take((size_t)c.B * 8, 16);
    L->cand = take((size_t)c.B * WIN_CAP * 8, 16);
    L->more = take((size_t)c.B * NPASS * 4, 16);
    L->hist = take((size_t)sel_groups_x_waves * NPASS * NBINS * 4, 256);
    L->head_cnt = take((size_t)C * 4, 256);
    L->partial = take((size_t)MAX_ATTN_CTAS * 2 * attn_partial_rec_floats(c.D, G) * 4, 256);
    // fused decode step (nothing when the batch is too large for it)
    const int SB = c.B <= STEP_MAX_B ? c.B : 0;
    const int64_t SC = SB ? C : 0;
    const size_t cw = SB ? step_ctr_words(SC, SB) : 0;
    L->step_bar = take(4, 64);
    L->step_leave = take(4, 64);
    L->step_parity = take(4, 64);
    L->step_ctr = take(2 * cw * 4, 256);
    L->ckey = take((size_t)SB * WIN_CAP * 8, 256);
    L->cslot = take((size_t)SB * WIN_CAP * 4, 256);
    L->cfate = take((size_t)SB * WIN_CAP * 4, 256);
    L->cz = take((size_t)SB * WIN_CAP * G * 4, 256);
    L->cv = take((size_t)SB * WIN_CAP * c.D * elt_bytes(c.dtype), 256);
    L->ghist = take((size_t)NPASS * SB * NBINS * 4, 256);
    L->hrec = take((size_t)SC * attn_partial_rec_floats(c.D, G) * 4, 256);
    L->npre = take((size_t)SC * 4, 256);
    L->pfx = take((size_t)(SC + 1) * 4, 256);
    L->bmask = take((size_t)C * c.max_pages * 2, 256);
    L->bkept = take((size_t)C * 4, 256);
    L->bfloor = take((size_t)C * 4, 256);
    L->bskip = take((size_t)C, 256);
    L->bseq = take((size_t)c.B * 16, 256);
    L->total = take(0, 256);
}

int sm_count_now(int *out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    e = cudaDeviceGetAttribute(out, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceGetAttribute");
    return RKV_OK;
}

int check_ws(const rkv_cache_t *c, void *ws, size_t ws_bytes, WsLayout *L) {
    if (!ws) return fail(RKV_ERR_INVALID_ARG, "workspace is NULL");
    if (!aligned16(ws)) return fail(RKV_ERR_INVALID_ARG, "workspace must be 16-byte aligned");
    ws_layout(*c, L);
    if (ws_bytes < L->total)
        return fail(RKV_ERR_WORKSPACE_TOO_SMALL, "workspace of %zu bytes < %zu needed", ws_bytes, L->total);
    return RKV_OK;
}

// cuTensorMapEncodeTiled, fetched once through the runtime's driver entry point.
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

int encode_pool_map(CUtensorMap *m, void *pool, int D, int n_pages) {
    if (D % 64 != 0) return fail(RKV_ERR_UNSUPPORTED, "bf16 pools need D a multiple of 64");
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q{};
        cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q);
        if (e != cudaSuccess || q != cudaDriverEntryPointSuccess || !p)
            return fail(RKV_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
        fn = reinterpret_cast<EncodeTiledFn>(p);
    }
    // the pool as a 3-D tensor (64 columns, n_pages*16 rows, D/64 halves) of
    // bf16: one box is a whole page and lands in shared memory as D/64 planes
    // of 16 rows x 128 bytes, 16-byte chunks XOR-swizzled by line mod 8
    const cuuint32_t nhalf = (cuuint32_t)(D / 64);
    const cuuint64_t dims[3] = {64, (cuuint64_t)n_pages * PAGE, nhalf};
    const cuuint64_t strides[2] = {(cuuint64_t)D * 2, 128};
    const cuuint32_t box[3] = {64, PAGE, nhalf};
    const cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, pool, dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(RKV_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
    return RKV_OK;
}

template <typename T>
T *at(void *ws, size_t off) {
    return reinterpret_cast<T *>(static_cast<unsigned char *>(ws) + off);
}

}  // namespace

bool ws_layout(const rkv_cache_t &c, WsLayout *out) {
    // groups x waves of the selection grid never exceed 2*B (groups <= B)
    layout_for(c, 2 * c.B, out);
    return true;
}

}  // namespace rkv

using namespace rkv;

// One NVTX range per call that enqueues work, named after the entry point
// (host side only; a no-op unless a profiler is attached).
namespace {
struct NvtxRange {
    explicit NvtxRange(const char *name) { nvtxRangePushA(name); }
    ~NvtxRange() { nvtxRangePop(); }
    NvtxRange(const NvtxRange &) = delete;
    NvtxRange &operator=(const NvtxRange &) = delete;
};
}  // namespace

extern "C" {

RKV_API const char *rkv_version(void) { return "librkv 0.1.0 (sm_100a)"; }

RKV_API const char *rkv_last_error(void) { return g_err.c_str(); }

RKV_API size_t rkv_workspace_size(const rkv_cache_t *cache) {
    if (check_cache(cache, false) != RKV_OK) return 0;
    WsLayout L;
    ws_layout(*cache, &L);
    return L.total;
}

RKV_API int rkv_workspace_init(void *ws, size_t ws_bytes, void *stream) {
    const NvtxRange nvtx_range("rkv_workspace_init");
    if (!ws || ws_bytes == 0) return fail(RKV_ERR_INVALID_ARG, "workspace is NULL or empty");
    cudaError_t e = cudaMemsetAsync(ws, 0, ws_bytes, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync(workspace)");
    return RKV_OK;
}

RKV_API int32_t *rkv_device_status(void *ws) { return ws ? reinterpret_cast<int32_t *>(ws) : nullptr; }

RKV_API int rkv_workspace_set_wait_limit(void *ws, size_t ws_bytes, uint32_t microseconds, void *stream) {
    const NvtxRange nvtx_range("rkv_workspace_set_wait_limit");
    if (!ws || ws_bytes < 32) return fail(RKV_ERR_INVALID_ARG, "workspace is NULL or too small");
    if (microseconds > 0x7FFFFFFFu) return fail(RKV_ERR_INVALID_ARG, "wait limit above 2^31 - 1 microseconds");
    cudaError_t e = launch_set_word(reinterpret_cast<int32_t *>(ws) + 4, (int32_t)microseconds,
                                    static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "rkv_workspace_set_wait_limit");
    return RKV_OK;
}

RKV_API int rkv_score_select(const rkv_cache_t *cache, const int32_t *t, const int64_t *m_global,
                             const rkv_select_t *sel, void *ws, size_t ws_bytes, void *stream) {
    const NvtxRange nvtx_range("rkv_score_select");
    int rc = check_cache(cache, true);
    if (rc) return rc;
    if ((rc = check_sel(sel))) return rc;
    if (!t || !m_global) return fail(RKV_ERR_INVALID_ARG, "t / m_global is NULL");
    WsLayout L;
    if ((rc = check_ws(cache, ws, ws_bytes, &L))) return rc;
    const int64_t LH = (int64_t)cache->L * cache->H;
    const int lb = lh_bits(LH);
    if (lb > 24) return fail(RKV_ERR_UNSUPPORTED, "L*H must be <= 2^24");
    int sms = 0;
    if ((rc = sm_count_now(&sms))) return rc;
    SelectGrid g = select_grid_for(*cache, sms < MAX_SEL_CTAS ? sms : MAX_SEL_CTAS);
    if (g.cache_pages < 0) return fail(RKV_ERR_UNSUPPORTED, "L*H too large for the selection kernel");
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    SelectArgs a{};
    a.pos_pool = cache->pos_pool;
    a.lb_pool = cache->lb_pool;
    a.block_table = cache->block_table;
    a.len = cache->len;
    a.free_top = cache->free_top;
    a.B = cache->B;
    a.LH = (int)LH;
    a.C = (int)(cache->B * LH);
    a.max_pages = cache->max_pages;
    a.ibits = 32 - lb;
    a.t = t;
    a.m_global = m_global;
    a.kappa = sel->kappa;
    a.kept = sel->kept;
    a.n_pre = sel->n_pre;
    a.keep_mask = sel->keep_mask;
    a.plan = sel->plan;
    a.status = at<int32_t>(ws, L.status);
    a.bar = at<uint32_t>(ws, L.bar);
    a.leave = at<uint32_t>(ws, L.leave);
    a.win = at<uint32_t>(ws, L.win);
    a.cnt = at<uint32_t>(ws, L.cnt);
    a.kmax = at<unsigned long long>(ws, L.kmax);
    a.cand = at<uint2>(ws, L.cand);
    a.more = at<uint32_t>(ws, L.more);
    a.hist = at<uint32_t>(ws, L.hist);
    a.n_groups = g.n_groups;
    a.cta_per_group = g.cta_per_group;
    a.waves = g.waves;
    a.cache_pages = g.cache_pages;
    cudaError_t e = launch_select(a, g, s);
    if (e != cudaSuccess) return cuda_fail(e, "select kernel launch");
    return RKV_OK;
}

// Allocation-free variant of rkv_score_select (no workspace argument): the
// selection scratch lives in a fixed device array of the library instead.
RKV_API int rkv_score_select_noalloc(const rkv_cache_t *cache, const int32_t *t, const int64_t *m_global,
                                     const rkv_select_t *sel, void *stream) {
    int rc = check_cache(cache, true);
    if (rc) return rc;
    if ((rc = check_sel(sel))) return rc;
    if (!t || !m_global) return fail(RKV_ERR_INVALID_ARG, "t / m_global is NULL");
    if (cache->B > NOALLOC_MAX_B)
        return fail(RKV_ERR_UNSUPPORTED,
                    "rkv_score_select_noalloc: batch %d exceeds its fixed scratch (at most %d sequences); "
                    "use rkv_score_select with a workspace",
                    cache->B, NOALLOC_MAX_B);
    const int64_t LH = (int64_t)cache->L * cache->H;
    const int lb = lh_bits(LH);
    if (lb > 24) return fail(RKV_ERR_UNSUPPORTED, "L*H must be <= 2^24");
    int sms = 0;
    if ((rc = sm_count_now(&sms))) return rc;
    const SelectGrid g = select_grid_for(*cache, sms < MAX_SEL_CTAS ? sms : MAX_SEL_CTAS);
    if (g.waves * g.n_groups > NOALLOC_MAX_B)
        return fail(RKV_ERR_UNSUPPORTED, "rkv_score_select_noalloc: too many sequences for its fixed scratch");
    uint32_t *scr = nullptr;
    const char *why = nullptr;
    if (noalloc_scratch(&scr, &why)) return fail(RKV_ERR_CUDA, "rkv_score_select_noalloc scratch: %s", why);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    // status, barrier counter, ticket, flags, counters, threshold windows and
    // this call's histograms start at zero (a cleared window means the exact
    // radix passes run; candidates need no clearing)
    const size_t words = NOALLOC_HIST + (size_t)g.waves * g.n_groups * NPASS * NBINS;
    cudaError_t e = cudaMemsetAsync(scr, 0, words * sizeof(uint32_t), s);
    if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync(noalloc scratch)");
    SelectArgs a{};
    a.pos_pool = cache->pos_pool;
    a.lb_pool = cache->lb_pool;
    a.block_table = cache->block_table;
    a.len = cache->len;
    a.free_top = cache->free_top;
    a.B = cache->B;
    a.LH = (int)LH;
    a.C = (int)(cache->B * LH);
    a.max_pages = cache->max_pages;
    a.ibits = 32 - lb;
    a.t = t;
    a.m_global = m_global;
    a.kappa = sel->kappa;
    a.kept = sel->kept;
    a.n_pre = sel->n_pre;
    a.keep_mask = sel->keep_mask;
    a.plan = sel->plan;
    a.status = reinterpret_cast<int32_t *>(scr + NOALLOC_STATUS);
    a.bar = scr + NOALLOC_BAR;
    a.leave = scr + NOALLOC_LEAVE;
    a.more = scr + NOALLOC_MORE;
    a.win = scr + NOALLOC_WIN;
    a.cnt = scr + NOALLOC_CNT;
    a.kmax = reinterpret_cast<unsigned long long *>(scr + NOALLOC_KMAX);
    a.cand = reinterpret_cast<uint2 *>(scr + NOALLOC_CAND);
    a.hist = scr + NOALLOC_HIST;
    a.n_groups = g.n_groups;
    a.cta_per_group = g.cta_per_group;
    a.waves = g.waves;
    a.cache_pages = g.cache_pages;
    e = launch_select(a, g, s);
    if (e != cudaSuccess) return cuda_fail(e, "select kernel launch (noalloc)");
    return RKV_OK;
}

static int attn_common(const rkv_cache_t *cache, const float *q, float scale, const rkv_select_t *sel,
                       float *out, float *lse, float *dropped, void *ws, size_t ws_bytes, void *stream,
                       const char *what) {
    int rc = check_cache(cache, true);
    if (rc) return rc;
    if (!q) return fail(RKV_ERR_INVALID_ARG, "%s: q is NULL", what);
    if (!aligned16(q)) return fail(RKV_ERR_INVALID_ARG, "%s: q must be 16-byte aligned", what);
    if (sel && !sel->keep_mask) return fail(RKV_ERR_INVALID_ARG, "%s: sel->keep_mask is NULL", what);
    const int G = cache->Hq / cache->H;
    if (!attn_supported(cache->dtype, cache->D, G))
        return fail(RKV_ERR_UNSUPPORTED, "%s: (dtype %d, D %d, G %d) not built", what, cache->dtype, cache->D, G);
    WsLayout L;
    if ((rc = check_ws(cache, ws, ws_bytes, &L))) return rc;
    int sms = 0;
    if ((rc = sm_count_now(&sms))) return rc;
    AttnArgs a{};
    a.k_pool = cache->k_pool;
    a.v_pool = cache->v_pool;
    a.block_table = cache->block_table;
    a.len = cache->len;
    a.keep_mask = sel ? sel->keep_mask : nullptr;
    a.q = q;
    a.out = out;
    a.lse = lse;
    a.dropped = dropped;
    a.status = at<int32_t>(ws, L.status);
    a.head_cnt = at<uint32_t>(ws, L.head_cnt);
    a.partial = at<float>(ws, L.partial);
    a.C = cache->B * cache->L * cache->H;
    a.max_pages = cache->max_pages;
    a.qscale = scale * 1.4426950408889634f;
    CUtensorMap tk{}, tv{};
    if (attn_uses_tensor_maps(cache->dtype)) {
        if ((rc = encode_pool_map(&tk, cache->k_pool, cache->D, cache->n_pages))) return rc;
        if ((rc = encode_pool_map(&tv, cache->v_pool, cache->D, cache->n_pages))) return rc;
    }
    cudaError_t e = launch_attn(a, cache->dtype, cache->D, G, sms, static_cast<cudaStream_t>(stream), tk, tv);
    if (e != cudaSuccess) return cuda_fail(e, what);
    return RKV_OK;
}

RKV_API int rkv_paged_decode_attn(const rkv_cache_t *cache, const float *q, float scale, const rkv_select_t *sel,
                                  float *out, float *lse_kept, float *dropped, void *ws, size_t ws_bytes,
                                  void *stream) {
    const NvtxRange nvtx_range("rkv_paged_decode_attn");
    if (!out) return fail(RKV_ERR_INVALID_ARG, "rkv_paged_decode_attn: out is NULL");
    return attn_common(cache, q, scale, sel, out, lse_kept, dropped, ws, ws_bytes, stream, "rkv_paged_decode_attn");
}

RKV_API int rkv_dropped_mass(const rkv_cache_t *cache, const float *q, float scale, const rkv_select_t *sel,
                             float *dropped, void *ws, size_t ws_bytes, void *stream) {
    const NvtxRange nvtx_range("rkv_dropped_mass");
    if (!dropped) return fail(RKV_ERR_INVALID_ARG, "rkv_dropped_mass: dropped is NULL");
    if (!sel) return fail(RKV_ERR_INVALID_ARG, "rkv_dropped_mass: sel is NULL");
    return attn_common(cache, q, scale, sel, nullptr, nullptr, dropped, ws, ws_bytes, stream, "rkv_dropped_mass");
}

RKV_API int rkv_score_select_budget(const rkv_cache_t *cache, const int32_t *t, const rkv_budget_t *budget,
                                    const rkv_select_t *sel, void *ws, size_t ws_bytes, void *stream) {
    const NvtxRange nvtx_range("rkv_score_select_budget");
    int rc = check_cache(cache, true);
    if (rc) return rc;
    if ((rc = check_sel(sel))) return rc;
    if (!t || !budget) return fail(RKV_ERR_INVALID_ARG, "rkv_score_select_budget: t / budget is NULL");
    const bool contour = budget->mode == RKV_BUDGET_CONTOUR;
    if (!contour && budget->mode != RKV_BUDGET_PER_HEAD)
        return fail(RKV_ERR_INVALID_ARG, "rkv_score_select_budget: unknown mode %d", budget->mode);
    if (!contour && !budget->m_head) return fail(RKV_ERR_INVALID_ARG, "rkv_score_select_budget: m_head is NULL");
    if (contour && (!budget->m_global || !budget->dm_prev))
        return fail(RKV_ERR_INVALID_ARG, "rkv_score_select_budget: m_global / dm_prev is NULL");
    if (contour && budget->flat_threshold != budget->flat_threshold)
        return fail(RKV_ERR_INVALID_ARG, "rkv_score_select_budget: flat_threshold is NaN");
    WsLayout L;
    if ((rc = check_ws(cache, ws, ws_bytes, &L))) return rc;
    const int64_t LH = (int64_t)cache->L * cache->H;
    const int lb = lh_bits(LH);
    if (lb > 24) return fail(RKV_ERR_UNSUPPORTED, "L*H must be <= 2^24");
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    BudgetArgs b{};
    b.pos_pool = cache->pos_pool;
    b.lb_pool = cache->lb_pool;
    b.block_table = cache->block_table;
    b.len = cache->len;
    b.t = t;
    b.LH = (int)LH;
    b.C = (int)(cache->B * LH);
    b.G = cache->Hq / cache->H;
    b.max_pages = cache->max_pages;
    b.mode = budget->mode;
    b.m_head = budget->m_head;
    b.dm_prev = budget->dm_prev;
    b.tau = budget->flat_threshold;
    b.flat_budget = budget->flat_budget;
    b.floor_r = budget->recency_floor;
    b.status = at<int32_t>(ws, L.status);
    cudaError_t e;
    if (!contour) {
        // every head's own top-m: masks, counts and lengths, then the plan
        b.mask = sel->keep_mask;
        b.kept = sel->kept;
        b.n_pre = sel->n_pre;
        if ((e = launch_head_budget(b, s)) != cudaSuccess) return cuda_fail(e, "budget kernel launch");
        if ((e = launch_plan(sel->n_pre, sel->kept, sel->plan, cache->free_top, sel->kappa, b.C, cache->B, s)) !=
            cudaSuccess)
            return cuda_fail(e, "plan kernel launch");
        return RKV_OK;
    }
    // ContourKV: floors and flat heads' budgets first, then the global
    // selection over what is left with the rest of the budget
    b.mask = at<uint16_t>(ws, L.bmask);
    b.kept = at<int32_t>(ws, L.bkept);
    b.floor_pos = at<int32_t>(ws, L.bfloor);
    b.skip = at<uint8_t>(ws, L.bskip);
    b.seq = at<unsigned long long>(ws, L.bseq);
    if ((e = cudaMemsetAsync(b.seq, 0, (size_t)cache->B * 16, s)) != cudaSuccess)
        return cuda_fail(e, "cudaMemsetAsync(budget counters)");
    if ((e = launch_head_budget(b, s)) != cudaSuccess) return cuda_fail(e, "budget kernel launch");
    int sms = 0;
    if ((rc = sm_count_now(&sms))) return rc;
    SelectGrid g = select_grid_for(*cache, sms < MAX_SEL_CTAS ? sms : MAX_SEL_CTAS);
    if (g.cache_pages < 0) return fail(RKV_ERR_UNSUPPORTED, "L*H too large for the selection kernel");
    SelectArgs a{};
    a.pos_pool = cache->pos_pool;
    a.lb_pool = cache->lb_pool;
    a.block_table = cache->block_table;
    a.len = cache->len;
    a.free_top = cache->free_top;
    a.B = cache->B;
    a.LH = (int)LH;
    a.C = (int)(cache->B * LH);
    a.max_pages = cache->max_pages;
    a.ibits = 32 - lb;
    a.t = t;
    a.m_global = budget->m_global;
    a.kappa = sel->kappa;
    a.kept = sel->kept;
    a.n_pre = sel->n_pre;
    a.keep_mask = sel->keep_mask;
    a.plan = sel->plan;
    a.status = at<int32_t>(ws, L.status);
    a.bar = at<uint32_t>(ws, L.bar);
    a.leave = at<uint32_t>(ws, L.leave);
    a.win = at<uint32_t>(ws, L.win);
    a.cnt = at<uint32_t>(ws, L.cnt);
    a.kmax = at<unsigned long long>(ws, L.kmax);
    a.cand = at<uint2>(ws, L.cand);
    a.more = at<uint32_t>(ws, L.more);
    a.hist = at<uint32_t>(ws, L.hist);
    a.n_groups = g.n_groups;
    a.cta_per_group = g.cta_per_group;
    a.waves = g.waves;
    a.cache_pages = g.cache_pages;
    a.floor_pos = b.floor_pos;
    a.skip = b.skip;
    a.pre_mask = b.mask;
    a.pre_kept = b.kept;
    a.seq = b.seq;
    if ((e = launch_select(a, g, s)) != cudaSuccess) return cuda_fail(e, "select kernel launch");
    return RKV_OK;
}

static int check_memory(const rkv_cache_t *cache, const rkv_memory_t *mem, const char *what) {
    if (!mem || !mem->proj || !mem->M || !mem->b)
        return fail(RKV_ERR_INVALID_ARG, "%s: memory, proj, M and b must be non-NULL", what);
    if (!aligned16(mem->M)) return fail(RKV_ERR_INVALID_ARG, "%s: M must be 16-byte aligned", what);
    if (!memory_supported(cache->D, cache->Hq / cache->H))
        return fail(RKV_ERR_UNSUPPORTED, "%s: D %d, G %d not built", what, cache->D, cache->Hq / cache->H);
    return RKV_OK;
}

RKV_API int rkv_memory_update(const rkv_cache_t *cache, const rkv_select_t *sel, const rkv_memory_t *mem,
                              void *stream) {
    const NvtxRange nvtx_range("rkv_memory_update");
    int rc = check_cache(cache, true);
    if (rc) return rc;
    if ((rc = check_sel(sel))) return rc;
    if ((rc = check_memory(cache, mem, "rkv_memory_update"))) return rc;
    if (!(mem->decay >= 0.0f && mem->decay <= 1.0f))
        return fail(RKV_ERR_INVALID_ARG, "rkv_memory_update: decay must be in [0, 1]");
    MemUpdateArgs a{};
    a.k_pool = cache->k_pool;
    a.v_pool = cache->v_pool;
    a.block_table = cache->block_table;
    a.n_pre = sel->n_pre;
    a.keep_mask = sel->keep_mask;
    a.proj = mem->proj;
    a.decay = mem->decay;
    a.M = mem->M;
    a.b = mem->b;
    a.C = cache->B * cache->L * cache->H;
    a.LH = cache->L * cache->H;
    a.H = cache->H;
    a.max_pages = cache->max_pages;
    cudaError_t e = launch_memory_update(a, cache->dtype, cache->D, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "rkv_memory_update");
    return RKV_OK;
}

RKV_API int rkv_memory_read(const rkv_cache_t *cache, const float *q, const rkv_memory_t *mem, float *out,
                            void *stream) {
    const NvtxRange nvtx_range("rkv_memory_read");
    int rc = check_cache(cache, false);
    if (rc) return rc;
    if (!q || !out) return fail(RKV_ERR_INVALID_ARG, "rkv_memory_read: q / out is NULL");
    if ((rc = check_memory(cache, mem, "rkv_memory_read"))) return rc;
    if (!mem->gate_w || !mem->gate_b) return fail(RKV_ERR_INVALID_ARG, "rkv_memory_read: gate_w / gate_b is NULL");
    MemReadArgs a{};
    a.q = q;
    a.proj = mem->proj;
    a.gate_w = mem->gate_w;
    a.gate_b = mem->gate_b;
    a.M = mem->M;
    a.b = mem->b;
    a.out = out;
    a.C = cache->B * cache->L * cache->H;
    a.LH = cache->L * cache->H;
    a.H = cache->H;
    a.Hq = cache->Hq;
    cudaError_t e = launch_memory_read(a, cache->D, cache->Hq / cache->H, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "rkv_memory_read");
    return RKV_OK;
}

RKV_API int rkv_eviction_error(const rkv_cache_t *cache, const float *q, float scale, const rkv_select_t *sel,
                               const float *out_kept, const float *dropped, float *err, void *ws, size_t ws_bytes,
                               void *stream) {
    const NvtxRange nvtx_range("rkv_eviction_error");
    if (!sel) return fail(RKV_ERR_INVALID_ARG, "rkv_eviction_error: sel is NULL");
    if (!out_kept || !dropped || !err || !q)
        return fail(RKV_ERR_INVALID_ARG, "rkv_eviction_error: q, out_kept, dropped and err must be non-NULL");
    int rc = check_cache(cache, true);
    if (rc) return rc;
    if ((rc = check_sel(sel))) return rc;
    WsLayout L;
    if ((rc = check_ws(cache, ws, ws_bytes, &L))) return rc;
    const int G = cache->Hq / cache->H;
    EvictErrArgs a{};
    a.k_pool = cache->k_pool;
    a.v_pool = cache->v_pool;
    a.block_table = cache->block_table;
    a.n_pre = sel->n_pre;
    a.keep_mask = sel->keep_mask;
    a.q = q;
    a.out_kept = out_kept;
    a.dropped = dropped;
    a.err = err;
    a.scale = scale;
    a.C = cache->B * cache->L * cache->H;
    a.max_pages = cache->max_pages;
    cudaError_t e = launch_evict_err(a, cache->dtype, cache->D, G, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "rkv_eviction_error");
    return RKV_OK;
}

RKV_API int rkv_decode_step(const rkv_cache_t *cache, const int32_t *t, const int64_t *m_global, const float *q,
                            float scale, const void *k_new, const void *v_new, const float *lb_new,
                            const rkv_select_t *sel, float *out, float *lse_kept, float *dropped, void *ws,
                            size_t ws_bytes, void *stream) {
    const NvtxRange nvtx_range("rkv_decode_step");
    int rc = check_cache(cache, true);
    if (rc) return rc;
    if (!t || !q || !k_new || !v_new || !lb_new || !out)
        return fail(RKV_ERR_INVALID_ARG, "rkv_decode_step: t, q, k_new, v_new, lb_new and out must be non-NULL");
    if (!aligned16(q) || !aligned16(k_new) || !aligned16(v_new) || !aligned16(cache->pos_pool) ||
        !aligned16(cache->lb_pool))
        return fail(RKV_ERR_INVALID_ARG, "rkv_decode_step: q, k_new, v_new, pos_pool and lb_pool must be 16-byte aligned");
    if (m_global && (rc = check_sel(sel))) return rc;
    if (cache->B > STEP_MAX_B)
        return fail(RKV_ERR_UNSUPPORTED, "rkv_decode_step: at most %d sequences per call (B = %d)", STEP_MAX_B,
                    cache->B);
    const int G = cache->Hq / cache->H;
    if (!step_supported(cache->dtype, cache->D, G))
        return fail(RKV_ERR_UNSUPPORTED, "rkv_decode_step: (dtype %d, D %d, G %d) not built", cache->dtype, cache->D, G);
    const int64_t LH = (int64_t)cache->L * cache->H;
    const int lb = lh_bits(LH);
    if (lb > 24) return fail(RKV_ERR_UNSUPPORTED, "L*H must be <= 2^24");
    WsLayout L;
    if ((rc = check_ws(cache, ws, ws_bytes, &L))) return rc;
    int sms = 0;
    if ((rc = sm_count_now(&sms))) return rc;
    const int grid = sms < MAX_ATTN_CTAS ? sms : MAX_ATTN_CTAS;
    const int64_t C = (int64_t)cache->B * LH;
    if (C > (int64_t)STEP_HEADS_PER_CTA * grid)
        return fail(RKV_ERR_UNSUPPORTED, "rkv_decode_step: %lld heads exceed %d per SM", (long long)C,
                    STEP_HEADS_PER_CTA);
    const size_t smem = step_smem_bytes(cache->dtype, cache->D, G, cache->max_pages);
    if (smem == 0 || smem > 227 * 1024)
        return fail(RKV_ERR_UNSUPPORTED, "rkv_decode_step: max_pages %d needs %zu bytes of shared memory",
                    cache->max_pages, smem);
    StepArgs a{};
    a.k_pool = cache->k_pool;
    a.v_pool = cache->v_pool;
    a.pos_pool = cache->pos_pool;
    a.lb_pool = cache->lb_pool;
    a.block_table = cache->block_table;
    a.len = cache->len;
    a.free_stack = cache->free_stack;
    a.free_top = cache->free_top;
    a.B = cache->B;
    a.LH = (int)LH;
    a.C = (int)C;
    a.max_pages = cache->max_pages;
    a.ibits = 32 - lb;
    a.row_bytes = cache->D * elt_bytes(cache->dtype);
    a.t = t;
    a.m_global = m_global;
    a.q = q;
    a.qscale = scale * 1.4426950408889634f;
    a.k_new = k_new;
    a.v_new = v_new;
    a.lb_new = lb_new;
    a.out = out;
    a.lse = lse_kept;
    a.dropped = dropped;
    if (m_global) {
        a.kappa = sel->kappa;
        a.kept = sel->kept;
        a.n_pre = sel->n_pre;
        a.keep_mask = sel->keep_mask;
        a.plan = sel->plan;
    }
    a.status = at<int32_t>(ws, L.status);
    a.bar = at<uint32_t>(ws, L.step_bar);
    a.leave = at<uint32_t>(ws, L.step_leave);
    a.parity = at<uint32_t>(ws, L.step_parity);
    a.ctr = at<uint32_t>(ws, L.step_ctr);
    a.ctr_words = (int)step_ctr_words(C, cache->B);
    a.win = at<uint32_t>(ws, L.win);
    a.ckey = at<uint64_t>(ws, L.ckey);
    a.cslot = at<int32_t>(ws, L.cslot);
    a.cfate = at<int32_t>(ws, L.cfate);
    a.cz = at<float>(ws, L.cz);
    a.cv = at<unsigned char>(ws, L.cv);
    a.ghist = at<uint32_t>(ws, L.ghist);
    a.partial = at<float>(ws, L.partial);
    a.head_cnt = at<uint32_t>(ws, L.head_cnt);
    a.hrec = at<float>(ws, L.hrec);
    a.npre = at<int32_t>(ws, L.npre);
    a.pfx = at<int32_t>(ws, L.pfx);
    CUtensorMap tk{}, tv{};
    if (attn_uses_tensor_maps(cache->dtype)) {
        if ((rc = encode_pool_map(&tk, cache->k_pool, cache->D, cache->n_pages))) return rc;
        if ((rc = encode_pool_map(&tv, cache->v_pool, cache->D, cache->n_pages))) return rc;
    }
    cudaError_t e = launch_step(a, cache->dtype, cache->D, G, grid, static_cast<cudaStream_t>(stream), tk, tv);
    if (e != cudaSuccess) return cuda_fail(e, "rkv_decode_step");
    return RKV_OK;
}

RKV_API int rkv_compact_pages(const rkv_cache_t *cache, const rkv_select_t *sel, void *ws, size_t ws_bytes,
                              void *stream) {
    const NvtxRange nvtx_range("rkv_compact_pages");
    int rc = check_cache(cache, true);
    if (rc) return rc;
    if ((rc = check_sel(sel))) return rc;
    WsLayout L;
    if ((rc = check_ws(cache, ws, ws_bytes, &L))) return rc;
    CompactArgs a{};
    a.k_pool = cache->k_pool;
    a.v_pool = cache->v_pool;
    a.pos_pool = cache->pos_pool;
    a.lb_pool = cache->lb_pool;
    a.block_table = cache->block_table;
    a.len = cache->len;
    a.free_stack = cache->free_stack;
    a.free_top = cache->free_top;
    a.kept = sel->kept;
    a.n_pre = sel->n_pre;
    a.keep_mask = sel->keep_mask;
    a.plan = sel->plan;
    a.done = at<uint32_t>(ws, L.done_compact);
    a.C = cache->B * cache->L * cache->H;
    a.max_pages = cache->max_pages;
    a.row_bytes = cache->D * elt_bytes(cache->dtype);
    cudaError_t e = launch_compact(a, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "compact kernel launch");
    return RKV_OK;
}

RKV_API int rkv_append(const rkv_cache_t *cache, const int32_t *t, const void *k_new, const void *v_new,
                       const float *lb_new, void *ws, size_t ws_bytes, void *stream) {
    const NvtxRange nvtx_range("rkv_append");
    int rc = check_cache(cache, true);
    if (rc) return rc;
    if (!t || !k_new || !v_new || !lb_new) return fail(RKV_ERR_INVALID_ARG, "rkv_append: an input is NULL");
    if (!aligned16(k_new) || !aligned16(v_new))
        return fail(RKV_ERR_INVALID_ARG, "rkv_append: k_new / v_new must be 16-byte aligned");
    WsLayout L;
    if ((rc = check_ws(cache, ws, ws_bytes, &L))) return rc;
    AppendArgs a{};
    a.k_pool = cache->k_pool;
    a.v_pool = cache->v_pool;
    a.pos_pool = cache->pos_pool;
    a.lb_pool = cache->lb_pool;
    a.block_table = cache->block_table;
    a.len = cache->len;
    a.free_stack = cache->free_stack;
    a.free_top = cache->free_top;
    a.t = t;
    a.k_new = k_new;
    a.v_new = v_new;
    a.lb_new = lb_new;
    a.status = at<int32_t>(ws, L.status);
    a.done = at<uint32_t>(ws, L.done_append);
    a.C = cache->B * cache->L * cache->H;
    a.LH = cache->L * cache->H;
    a.max_pages = cache->max_pages;
    a.row_bytes = cache->D * elt_bytes(cache->dtype);
    cudaError_t e = launch_append(a, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "append kernel launch");
    return RKV_OK;
}

}  // extern "C"
