// select.cu -- fused score + exact global top-M radix select (sm_100a).
//
// Make Each Token Count (DBTrimKV), Methodology 2-3: every cached entry of
// all layers and heads of a sequence gets the retention score
// log(beta_i^(t-i)) = (t-i) * log(beta_i), and the top M_global are kept.
// Cache What Lasts (TRIM-KV), core mechanism 4: the lowest are evicted.
//
// One cooperative persistent launch.  CTAs form one group per sequence (in
// waves when B exceeds the group count); a group splits its sequence's pages
// evenly.  Phase 0 computes each entry's 64-bit rank key
//   hi = order-preserving map of s = fl32(float(t - i) * lb) (smaller = better)
//   lo = (l*H + h) << ib | i                                (tie rule)
// and caches it in shared memory (pages past the cache capacity are
// recomputed from global memory on later passes).  Each radix pass
// histograms one digit (11, 11, 10 | 11, 11, 10 bits) of the keys that match
// the prefix found so far, flushes non-empty bins to a per-group global
// histogram, and after a bounded grid barrier every CTA of the group scans
// that histogram to pick the digit holding the M-th key.  A group stops as
// soon as the chosen bucket is kept whole.  The result is an exclusive
// threshold kappa (kept <=> key < kappa), per-page keep masks built with
// warp ballots, per-head kept counts, and the free-page plan that the
// compaction kernel consumes.
#include <cooperative_groups.h>

#include "common.cuh"
#include "internal.h"

namespace rkv {

namespace {

constexpr int SEL_THREADS = 512;
constexpr int SEL_MAX_LH = 8192;

struct SelSmem {
    int32_t *pfx;     // [LH + 1] page prefix of the group's sequence
    int32_t *lens;    // [LH]
    uint32_t *hist;   // [NBINS]
    uint32_t *scan;   // [40]
    uint2 *keys;      // [cache_pages * 16]
    int *flag;        // barrier / misc flags
    uint32_t *bcast;  // [4] broadcast words
};

struct SeqState {
    int b;
    bool active;
    int32_t t;
    int64_t n, m;            // entries, clamped budget
    uint32_t rank;           // 1-based rank of the threshold key among matching keys
    uint64_t pk, pm;         // prefix bits found so far and their mask
    bool done;
    uint64_t kappa;          // exclusive threshold once done
    int x0, x1;              // page range of this CTA within the sequence
};

// Head (local index) of flattened page x: largest c with pfx[c] <= x.
__device__ __forceinline__ int page_head(const int32_t *pfx, int LH, int x) {
    int lo = 0, hi = LH - 1;
    while (lo < hi) {
        int mid = (lo + hi + 1) >> 1;
        if (pfx[mid] <= x) lo = mid; else hi = mid - 1;
    }
    return lo;
}

// Rank key of slot (x, r) of the sequence.  Invalid slots (past len, or bad
// input, which is also recorded) get hi = KEY_INVALID.
__device__ __forceinline__ uint2 entry_key(const SelectArgs &a, const SelSmem &sm, const SeqState &st, int x,
                                           int r) {
    const int cl = page_head(sm.pfx, a.LH, x);
    const int pidx = x - sm.pfx[cl];
    const int k = pidx * PAGE + r;
    uint2 key = make_uint2(KEY_INVALID, 0u);
    if (k < sm.lens[cl]) {
        const int64_t c = (int64_t)st.b * a.LH + cl;
        const int32_t page = __ldg(a.block_table + c * a.max_pages + pidx);
        const int64_t row = (int64_t)page * PAGE + r;
        const int32_t pos = __ldg(a.pos_pool + row);
        const float lb = __ldg(a.lb_pool + row);
        const int64_t age = (int64_t)st.t - pos;
        const bool bad = (lb != lb) || age < 1 || age >= (1 << 24) || pos < 0 ||
                         (a.ibits < 32 && (uint32_t)pos >= (1u << a.ibits));
        if (bad) {
            set_status(a.status, RKV_DEV_BAD_INPUT);
        } else {
            float s = __fmul_rn((float)(int32_t)age, lb);
            if (s == 0.0f) s = 0.0f;
            key.x = score_key_desc(s);
            key.y = (uint32_t)(((uint64_t)cl << a.ibits) | (uint32_t)pos);
        }
    }
    return key;
}

__device__ __forceinline__ uint2 cached_key(const SelectArgs &a, const SelSmem &sm, const SeqState &st, int x,
                                            int r) {
    const int off = x - st.x0;
    if (off < a.cache_pages) return sm.keys[off * PAGE + r];
    return entry_key(a, sm, st, x, r);
}

__device__ __forceinline__ bool key_matches(uint2 k, const SeqState &st) {
    const uint64_t K = ((uint64_t)k.x << 32) | k.y;
    return k.x != KEY_INVALID && ((K ^ st.pk) & st.pm) == 0;
}

// Histogram digit p of this CTA's matching keys into the group's global bins.
// When `fill` is set (phase 0) the keys are computed and cached on the way.
__device__ void hist_pass(const SelectArgs &a, const SelSmem &sm, const SeqState &st, int p, int g, int wave,
                          bool fill, bool count) {
    for (int i = threadIdx.x; i < NBINS; i += blockDim.x) sm.hist[i] = 0u;
    __syncthreads();
    const int r = threadIdx.x & 15;
    for (int x = st.x0 + (int)(threadIdx.x >> 4); x < st.x1; x += blockDim.x >> 4) {
        uint2 k;
        if (fill) {
            k = entry_key(a, sm, st, x, r);
            const int off = x - st.x0;
            if (off < a.cache_pages) sm.keys[off * PAGE + r] = k;
        } else {
            k = cached_key(a, sm, st, x, r);
        }
        if (count && key_matches(k, st)) atomicAdd(&sm.hist[key_digit(k.x, k.y, p)], 1u);
    }
    __syncthreads();
    if (count) {
        uint32_t *gh = a.hist + ((size_t)(wave * NPASS + p) * a.n_groups + g) * NBINS;
        for (int i = threadIdx.x; i < NBINS; i += blockDim.x) {
            const uint32_t v = sm.hist[i];
            if (v) atomicAdd(gh + i, v);
        }
    }
}

// Pick digit p of the threshold from the group's completed histogram.
__device__ void scan_pass(const SelectArgs &a, const SelSmem &sm, SeqState &st, int p, int g, int wave) {
    const uint32_t *gh = a.hist + ((size_t)(wave * NPASS + p) * a.n_groups + g) * NBINS;
    constexpr int PER = NBINS / SEL_THREADS;  // 4
    uint32_t v[PER];
    uint32_t loc = 0;
#pragma unroll
    for (int j = 0; j < PER; j++) {
        v[j] = __ldcg(gh + threadIdx.x * PER + j);
        loc += v[j];
    }
    uint32_t total;
    const uint32_t ex = block_exclusive_scan(loc, sm.scan, &total);
    if (ex < st.rank && st.rank <= ex + loc) {
        uint32_t cum = ex;
#pragma unroll
        for (int j = 0; j < PER; j++) {
            if (cum < st.rank && st.rank <= cum + v[j]) {
                sm.bcast[0] = threadIdx.x * PER + j;  // digit
                sm.bcast[1] = st.rank - cum;          // new rank within the bucket
                sm.bcast[2] = v[j];                   // bucket size
            }
            cum += v[j];
        }
    }
    __syncthreads();
    const uint32_t d = sm.bcast[0], nr = sm.bcast[1], h = sm.bcast[2];
    __syncthreads();
    const int sh = digit_shift(p);
    const uint64_t dm = ((1ull << digit_bits(p)) - 1ull) << sh;
    st.pk |= (uint64_t)d << sh;
    st.pm |= dm;
    st.rank = nr;
    if (h == nr || p == NPASS - 1) {
        st.done = true;
        st.kappa = (st.pk | ~st.pm) + 1ull;
    }
}

// Keep masks (warp ballots over the 16 slots of a page) and kept counts.
__device__ void final_pass(const SelectArgs &a, const SelSmem &sm, const SeqState &st) {
    const int lane = threadIdx.x & 31, r = lane & 15;
    const int nwarp = blockDim.x >> 5, warp = threadIdx.x >> 5;
    for (int xb = st.x0 + warp * 2; xb < st.x1; xb += nwarp * 2) {
        const int x = xb + (lane >> 4);
        bool keep = false;
        if (x < st.x1) {
            const uint2 k = cached_key(a, sm, st, x, r);
            const uint64_t K = ((uint64_t)k.x << 32) | k.y;
            keep = k.x != KEY_INVALID && K < st.kappa;
        }
        const uint32_t ball = __ballot_sync(0xFFFFFFFFu, keep);
        if (r == 0 && x < st.x1) {
            const uint32_t m16 = (ball >> (lane & 16)) & 0xFFFFu;
            const int cl = page_head(sm.pfx, a.LH, x);
            const int pidx = x - sm.pfx[cl];
            const int64_t c = (int64_t)st.b * a.LH + cl;
            a.keep_mask[c * a.max_pages + pidx] = (uint16_t)m16;
            if (m16) atomicAdd(a.kept + c, __popc(m16));
        }
    }
}

__global__ void __launch_bounds__(SEL_THREADS, 1) select_kernel(SelectArgs a) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    SelSmem sm;
    {
        unsigned char *p = smem_raw;
        sm.keys = reinterpret_cast<uint2 *>(p);
        p += (size_t)a.cache_pages * PAGE * sizeof(uint2);
        sm.hist = reinterpret_cast<uint32_t *>(p);
        p += NBINS * sizeof(uint32_t);
        sm.scan = reinterpret_cast<uint32_t *>(p);
        p += 40 * sizeof(uint32_t);
        sm.bcast = reinterpret_cast<uint32_t *>(p);
        p += 4 * sizeof(uint32_t);
        sm.flag = reinterpret_cast<int *>(p);
        p += 4 * sizeof(int);
        sm.pfx = reinterpret_cast<int32_t *>(p);
        p += (size_t)(a.LH + 1) * sizeof(int32_t);
        sm.lens = reinterpret_cast<int32_t *>(p);
    }
    const int g = blockIdx.x / a.cta_per_group;
    const int rr = blockIdx.x % a.cta_per_group;
    uint32_t epoch = 0;
    bool alive = true;

    for (int wave = 0; wave < a.waves && alive; wave++) {
        SeqState st;
        st.b = wave * a.n_groups + g;
        st.active = g < a.n_groups && st.b < a.B;
        st.done = true;
        st.kappa = 0;
        st.x0 = st.x1 = 0;
        bool finalized = false;
        if (st.active) {
            // page prefix and lengths of this sequence's heads
            uint32_t carry = 0;
            int64_t nsum = 0;
            for (int base = 0; base < a.LH; base += blockDim.x) {
                const int cl = base + threadIdx.x;
                int32_t n = cl < a.LH ? __ldcg(a.len + (int64_t)st.b * a.LH + cl) : 0;
                if (n < 0) n = 0;
                if (cl < a.LH) sm.lens[cl] = n;
                uint32_t tot;
                const uint32_t ex = block_exclusive_scan((uint32_t)((n + PAGE - 1) / PAGE), sm.scan, &tot);
                if (cl < a.LH) sm.pfx[cl] = (int32_t)(carry + ex);
                carry += tot;
            }
            if (threadIdx.x == 0) sm.pfx[a.LH] = (int32_t)carry;
            __syncthreads();
            for (int cl = threadIdx.x; cl < a.LH; cl += blockDim.x) nsum += sm.lens[cl];
            // block sum of entries
            uint32_t tot_lo;
            block_exclusive_scan((uint32_t)nsum, sm.scan, &tot_lo);
            st.n = tot_lo;
            const int TP = (int)carry;
            st.x0 = (int)(((int64_t)rr * TP) / a.cta_per_group);
            st.x1 = (int)(((int64_t)(rr + 1) * TP) / a.cta_per_group);
            // per-head outputs of this sequence: n_pre copy, kept zeroed
            for (int cl = rr * blockDim.x + threadIdx.x; cl < a.LH; cl += a.cta_per_group * blockDim.x) {
                const int64_t c = (int64_t)st.b * a.LH + cl;
                a.n_pre[c] = sm.lens[cl];
                a.kept[c] = 0;
            }
            st.t = __ldg(a.t + st.b);
            int64_t m = __ldg(a.m_global + st.b);
            st.m = m < 0 ? 0 : (m > st.n ? st.n : m);
            st.rank = (uint32_t)st.m;
            st.pk = 0;
            st.pm = 0;
            st.done = (st.m == 0) || (st.m == st.n);
            st.kappa = st.m == 0 ? 0ull : ~0ull;
            hist_pass(a, sm, st, 0, g, wave, /*fill=*/true, /*count=*/!st.done);
        }
        alive = grid_barrier(a.bar, ++epoch, a.status, sm.flag);
        for (int p = 0; alive; p++) {
            if (st.active && !st.done) scan_pass(a, sm, st, p, g, wave);
            if (st.active && st.done && !finalized) {
                final_pass(a, sm, st);
                if (rr == 0 && threadIdx.x == 0) a.kappa[st.b] = st.kappa;
                finalized = true;
            }
            if (st.active && !st.done) {
                if (rr == 0 && threadIdx.x == 0) atomicOr(a.more + wave * NPASS + p, 1u);
                hist_pass(a, sm, st, p + 1, g, wave, false, true);
            }
            alive = grid_barrier(a.bar, ++epoch, a.status, sm.flag);
            if (!alive) break;
            if (__ldcg(a.more + wave * NPASS + p) == 0u) break;
        }
    }
    // Free-page plan over all heads (after the last barrier every kept count
    // and n_pre is final): plan[c] = pages freed in heads < c.
    if (!alive || blockIdx.x != 0) return;
    uint32_t carry = 0;
    for (int base = 0; base < a.C; base += blockDim.x) {
        const int c = base + threadIdx.x;
        uint32_t f = 0;
        if (c < a.C) {
            const int32_t np = __ldcg(a.n_pre + c), nk = __ldcg(a.kept + c);
            f = (uint32_t)((np + PAGE - 1) / PAGE - (nk + PAGE - 1) / PAGE);
        }
        uint32_t tot;
        const uint32_t ex = block_exclusive_scan(f, sm.scan, &tot);
        if (c < a.C) a.plan[c] = (int32_t)(carry + ex);
        carry += tot;
    }
    if (threadIdx.x == 0) {
        a.plan[a.C] = (int32_t)carry;
        a.plan[a.C + 1] = __ldcg(a.free_top);
    }
}

}  // namespace

int select_max_smem() { return 227 * 1024; }

SelectGrid select_grid_for(const rkv_cache_t &c, int sm_count) {
    SelectGrid g{};
    const int LH = c.L * c.H;
    g.threads = SEL_THREADS;
    const int ctas = sm_count;  // one CTA per SM (large shared-memory key cache)
    g.n_groups = c.B < ctas ? c.B : ctas;
    g.cta_per_group = ctas / g.n_groups;
    g.waves = (c.B + g.n_groups - 1) / g.n_groups;
    const int fixed = NBINS * 4 + 40 * 4 + 16 + 16 + (2 * LH + 1) * 4;
    const int avail = select_max_smem() - fixed - 1024;
    g.cache_pages = avail > 0 ? avail / (PAGE * (int)sizeof(uint2)) : 0;
    // no point caching more pages than the largest per-CTA share could hold
    const int64_t total_pages = (int64_t)c.n_pages;
    const int64_t share = total_pages / (g.cta_per_group > 0 ? g.cta_per_group : 1) + 2;
    if (g.cache_pages > share) g.cache_pages = (int)share;
    g.smem_bytes = fixed + g.cache_pages * PAGE * (int)sizeof(uint2);
    return g;
}

cudaError_t launch_select(const SelectArgs &a, const SelectGrid &g, cudaStream_t s) {
    if (a.LH > SEL_MAX_LH) return cudaErrorNotSupported;
    cudaError_t e = cudaFuncSetAttribute(select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, g.smem_bytes);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(g.n_groups * g.cta_per_group);
    cfg.blockDim = dim3(g.threads);
    cfg.dynamicSmemBytes = g.smem_bytes;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, select_kernel, a);
}

}  // namespace rkv
