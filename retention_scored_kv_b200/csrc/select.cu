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

#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace rkv {

namespace {

constexpr int SEL_THREADS = 512;
constexpr int SEL_MAX_LH = 8192;

struct SelSmem {
    int32_t *pfx;     // [LH + 1] page prefix of the group's sequence
    int32_t *lens;    // [LH]
    int32_t *kc;      // [LH] kept counts of this CTA's pages, per head
    uint32_t *hist;   // [4][NBINS] sub-histograms
    uint32_t *scan;   // [40]
    uint2 *keys;      // [cache_pages * 16]
    int *flag;        // barrier / misc flags
    uint32_t *bcast;  // [4] broadcast words
    unsigned long long *kmax;  // largest kept key of this CTA's pages
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
    bool wv;                 // threshold window of the previous call is usable
    uint32_t wlo, whi;       // window [wlo, whi) in score-key (hi word) space
    int wres;                // 0 unused, 1 resolved in the window, 2 missed, 3 overflowed
    uint32_t wn;             // candidates found in the window
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

// Rank key of one slot from its position and log-retention.  Invalid slots
// (past len, or bad input, which is also recorded) get hi = KEY_INVALID.
__device__ __forceinline__ uint2 make_key(const SelectArgs &a, const SeqState &st, int cl, int32_t pos, float lb) {
    const int64_t age = (int64_t)st.t - pos;
    const bool bad = (lb != lb) || age < 1 || age >= (1 << 24) || pos < 0 ||
                     (a.ibits < 32 && (uint32_t)pos >= (1u << a.ibits));
    if (bad) {
        set_status(a.status, RKV_DEV_BAD_INPUT);
        return make_uint2(KEY_INVALID, 0u);
    }
    if (a.skip) {
        // ContourKV's global part: flat heads and floor entries are not ranked
        const int64_t c = (int64_t)st.b * a.LH + cl;
        if (__ldg(a.skip + c) || pos >= __ldg(a.floor_pos + c)) return make_uint2(KEY_INVALID, 0u);
    }
    float s = __fmul_rn((float)(int32_t)age, lb);
    if (s == 0.0f) s = 0.0f;
    return make_uint2(score_key_desc(s), (uint32_t)(((uint64_t)cl << a.ibits) | (uint32_t)pos));
}

constexpr int UNR = 8;  // pages per thread per round (loads issued together)

// Computes the keys of pages [xa, xb) of this CTA's range from global memory
// and calls f(x, r, key) for each slot.  Warp w covers pages xa + 2w +
// (lane >> 4) + 32*j; each lane owns slot r = lane & 15 of its page, so a
// warp's two half-warps hold two whole pages.  Each round issues the block
// table loads of UNR pages, then their position / log-retention loads, so a
// round costs two dependent memory latencies.  Loop bounds are warp-uniform.
template <typename F>
__device__ __forceinline__ void keys_from_global(const SelectArgs &a, const SelSmem &sm, const SeqState &st, int xa,
                                                 int xb_end, F &&f) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarp = blockDim.x >> 5;
    const int r = lane & 15;
    const int step = 2 * nwarp;
    int cur = -1;  // head of the previous page looked up (pages ascend per thread)
    for (int xb = xa + 2 * warp; xb < xb_end; xb += step * UNR) {
        int32_t pg[UNR];
        int cl[UNR];
        bool ld[UNR];
#pragma unroll
        for (int u = 0; u < UNR; u++) {
            const int x = xb + (lane >> 4) + u * step;
            ld[u] = false;
            cl[u] = 0;
            pg[u] = 0;
            if (x < xb_end) {
                if (cur < 0) cur = page_head(sm.pfx, a.LH, x);
                while (cur + 1 < a.LH && sm.pfx[cur + 1] <= x) cur++;
                cl[u] = cur;
                const int pidx = x - sm.pfx[cur];
                if (pidx * PAGE + r < sm.lens[cur]) {
                    ld[u] = true;
                    pg[u] = __ldg(a.block_table + ((int64_t)st.b * a.LH + cur) * a.max_pages + pidx);
                }
            }
        }
        int32_t pos[UNR];
        float lb[UNR];
#pragma unroll
        for (int u = 0; u < UNR; u++) {
            pos[u] = 0;
            lb[u] = 0.0f;
            if (ld[u]) {
                const int64_t row = (int64_t)pg[u] * PAGE + r;
                pos[u] = __ldg(a.pos_pool + row);
                lb[u] = __ldg(a.lb_pool + row);
            }
        }
#pragma unroll
        for (int u = 0; u < UNR; u++) {
            const int x = xb + (lane >> 4) + u * step;
            f(x, r, (x < xb_end && ld[u]) ? make_key(a, st, cl[u], pos[u], lb[u]) : make_uint2(KEY_INVALID, 0u));
        }
    }
}

// Calls f(x, r, key) for every slot r of every page x of this CTA's range:
// cached pages from shared memory (a flat loop, 32 keys = two pages per warp
// per step), the rest recomputed from global memory.  With `fill` every key
// is computed from global memory and the cacheable ones are stored.
template <typename F>
__device__ __forceinline__ void for_keys(const SelectArgs &a, const SelSmem &sm, const SeqState &st, bool fill,
                                         F &&f) {
    const int ncache = min(st.x1 - st.x0, a.cache_pages);
    if (fill) {
        keys_from_global(a, sm, st, st.x0, st.x1, [&](int x, int r, uint2 k) {
            if (x - st.x0 < a.cache_pages && x < st.x1) sm.keys[(x - st.x0) * PAGE + r] = k;
            f(x, r, k);
        });
        return;
    }
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int nk = ncache * PAGE;
    for (int base = warp * 32; base < nk; base += blockDim.x) {
        const int i = base + lane;
        const uint2 k = i < nk ? sm.keys[i] : make_uint2(KEY_INVALID, 0u);
        f(i < nk ? st.x0 + (i >> 4) : st.x1, i & 15, k);
    }
    if (st.x0 + ncache < st.x1) keys_from_global(a, sm, st, st.x0 + ncache, st.x1, f);
}

__device__ __forceinline__ bool key_matches(uint2 k, const SeqState &st) {
    const uint64_t K = ((uint64_t)k.x << 32) | k.y;
    return k.x != KEY_INVALID && ((K ^ st.pk) & st.pm) == 0;
}

// Histogram digit p of this CTA's matching keys into the group's global bins.
// When `fill` is set (first pass) the keys are computed and cached on the way.
// Lanes update NSUB interleaved sub-histograms (lane mod NSUB) to spread the
// shared-memory atomics of keys that share a digit; they are summed on flush.
constexpr int NSUB = 4;
__device__ void hist_pass(const SelectArgs &a, const SelSmem &sm, const SeqState &st, int p, int g, int wave,
                          bool fill, bool count) {
    for (int i = threadIdx.x; i < NSUB * NBINS; i += blockDim.x) sm.hist[i] = 0u;
    __syncthreads();
    const int lane = threadIdx.x & 31;
    uint32_t *hsub = sm.hist + (lane & (NSUB - 1)) * NBINS;
    // first pass only: keys above the previous threshold's window are
    // counted, keys inside it are appended to the candidate list
    const bool win = fill && count && st.wv;
    uint32_t above = 0;
    uint32_t *ncand = a.cnt + (size_t)st.b * 4 + 1;
    uint2 *cand = a.cand + (size_t)st.b * WIN_CAP;
    for_keys(a, sm, st, fill, [&](int x, int r, uint2 k) {
        if (!count) return;
        const bool hit = x < st.x1 && key_matches(k, st);
        if (hit) atomicAdd(&hsub[key_digit(k.x, k.y, p)], 1u);
        if (win) {
            const bool valid = x < st.x1 && k.x != KEY_INVALID;
            above += (valid && k.x < st.wlo) ? 1u : 0u;
            const bool in = valid && k.x >= st.wlo && k.x < st.whi;
            const uint32_t ball = __ballot_sync(0xFFFFFFFFu, in);
            if (ball) {
                const int leader = __ffs(ball) - 1;
                uint32_t base = 0;
                if (lane == leader) base = atomicAdd(ncand, (uint32_t)__popc(ball));
                base = __shfl_sync(0xFFFFFFFFu, base, leader);
                const uint32_t idx = base + (uint32_t)__popc(ball & ((1u << lane) - 1u));
                if (in && idx < WIN_CAP) cand[idx] = k;
            }
        }
    });
    if (win) {
        uint32_t tot;
        block_exclusive_scan(above, sm.scan, &tot);
        if (threadIdx.x == 0 && tot) atomicAdd(a.cnt + (size_t)st.b * 4, tot);
    }
    __syncthreads();
    if (count) {
        uint32_t *gh = a.hist + ((size_t)(wave * NPASS + p) * a.n_groups + g) * NBINS;
        for (int i = threadIdx.x; i < NBINS; i += blockDim.x) {
            uint32_t v = 0;
#pragma unroll
            for (int j = 0; j < NSUB; j++) v += sm.hist[j * NBINS + i];
            if (v) atomicAdd(gh + i, v);
        }
    }
}

// Pick digit p of the threshold from the group's completed histogram.
__device__ void scan_pass(const SelectArgs &a, const SelSmem &sm, SeqState &st, int p, int g, int wave) {
    const uint32_t *gh = a.hist + ((size_t)(wave * NPASS + p) * a.n_groups + g) * NBINS;
    constexpr int PER = NBINS / SEL_THREADS;  // 4
    const uint4 v4 = __ldcg(reinterpret_cast<const uint4 *>(gh) + threadIdx.x);
    const uint32_t v[PER] = {v4.x, v4.y, v4.z, v4.w};
    const uint32_t loc = v[0] + v[1] + v[2] + v[3];
    if (threadIdx.x == 0) sm.bcast[3] = 0u;
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
                sm.bcast[3] = 1u;
            }
            cum += v[j];
        }
    }
    __syncthreads();
    const uint32_t d = sm.bcast[0], nr = sm.bcast[1], h = sm.bcast[2], found = sm.bcast[3];
    __syncthreads();
    if (!found) {
        // fewer matching keys than the rank (only when entries were rejected
        // as bad input): keep every key with the current prefix
        if (threadIdx.x == 0) set_status(a.status, RKV_DEV_BAD_INPUT);
        st.done = true;
        st.kappa = (st.pk | ~st.pm) + 1ull;
        return;
    }
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

// After the first barrier: if the previous threshold's window holds the
// M-th key (keys above the window < M <= above + candidates, and every
// candidate was stored), the threshold is the (M - above)-th smallest
// candidate -- found by counting, per candidate, the candidates below it
// (64-bit keys are distinct).  Otherwise the radix passes continue.
__device__ void try_window(const SelectArgs &a, const SelSmem &sm, SeqState &st) {
    if (!st.wv) return;
    const uint32_t above = __ldcg(a.cnt + (size_t)st.b * 4), nc = __ldcg(a.cnt + (size_t)st.b * 4 + 1);
    st.wn = nc;
    if (nc > WIN_CAP) { st.wres = 3; return; }
    if (!((int64_t)above < st.m && st.m <= (int64_t)above + nc)) { st.wres = 2; return; }
    const uint32_t r = (uint32_t)(st.m - above);  // 1-based rank among the candidates
    uint2 *cs = reinterpret_cast<uint2 *>(sm.hist);  // 4*NBINS words >= 2*WIN_CAP
    const uint2 *cand = a.cand + (size_t)st.b * WIN_CAP;
    for (uint32_t i = threadIdx.x; i < nc; i += blockDim.x) cs[i] = __ldcg(cand + i);
    __syncthreads();
    for (uint32_t i = threadIdx.x; i < nc; i += blockDim.x) {
        const uint64_t Ki = ((uint64_t)cs[i].x << 32) | cs[i].y;
        uint32_t less = 0;
        for (uint32_t j = 0; j < nc; j++) less += ((((uint64_t)cs[j].x << 32) | cs[j].y) < Ki) ? 1u : 0u;
        if (less == r - 1) {
            const uint64_t kap = Ki + 1ull;
            sm.bcast[0] = (uint32_t)kap;
            sm.bcast[1] = (uint32_t)(kap >> 32);
        }
    }
    __syncthreads();
    st.kappa = ((uint64_t)sm.bcast[1] << 32) | sm.bcast[0];
    st.done = true;
    st.wres = 1;
    __syncthreads();
}

// Head (local index) of a page from the key of its slot 0 (lo = cl << ib | i).
__device__ __forceinline__ int head_of(const SelectArgs &a, const SelSmem &sm, int x, uint2 k0) {
    if (k0.x != KEY_INVALID) return a.ibits >= 32 ? 0 : (int)(k0.y >> a.ibits);
    return page_head(sm.pfx, a.LH, x);
}

// Keep masks (half-warp ballots over the 16 slots of a page); kept counts are
// summed per head in shared memory and flushed with one atomic per head.
// The largest kept key goes to a.kmax[b]: the reported threshold is that key
// + 1 whichever way it was found (a radix bucket kept whole only bounds it).
__device__ void final_pass(const SelectArgs &a, const SelSmem &sm, const SeqState &st) {
    const int lane = threadIdx.x & 31;
    if (threadIdx.x == 0) *sm.kmax = 0ull;
    __syncthreads();
    unsigned long long kmx = 0ull;
    for_keys(a, sm, st, false, [&](int x, int r, uint2 k) {
        const uint64_t K = ((uint64_t)k.x << 32) | k.y;
        const bool keep = x < st.x1 && k.x != KEY_INVALID && K < st.kappa;
        if (keep && K > kmx) kmx = K;
        const uint32_t ball = __ballot_sync(0xFFFFFFFFu, keep);
        if (r == 0 && x < st.x1) {
            const uint32_t m16 = (ball >> (lane & 16)) & 0xFFFFu;
            const int cl = head_of(a, sm, x, k);
            const int pidx = x - sm.pfx[cl];
            const int64_t wi = ((int64_t)st.b * a.LH + cl) * a.max_pages + pidx;
            a.keep_mask[wi] = (uint16_t)(a.pre_mask ? (m16 | __ldg(a.pre_mask + wi)) : m16);
            if (m16) atomicAdd(&sm.kc[cl], __popc(m16));
        }
    });
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const unsigned long long y = __shfl_xor_sync(0xFFFFFFFFu, kmx, o);
        kmx = y > kmx ? y : kmx;
    }
    if (lane == 0 && kmx) atomicMax(sm.kmax, kmx);
    __syncthreads();
    if (threadIdx.x == 0 && *sm.kmax) atomicMax(a.kmax + st.b, *sm.kmax);
    if (st.x0 < st.x1) {
        const int c_lo = page_head(sm.pfx, a.LH, st.x0), c_hi = page_head(sm.pfx, a.LH, st.x1 - 1);
        for (int cl = c_lo + (int)threadIdx.x; cl <= c_hi; cl += blockDim.x) {
            const int v = sm.kc[cl];
            if (v) atomicAdd(a.kept + (int64_t)st.b * a.LH + cl, v);
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
        p += 4 * NBINS * sizeof(uint32_t);
        sm.scan = reinterpret_cast<uint32_t *>(p);
        p += 40 * sizeof(uint32_t);
        sm.kmax = reinterpret_cast<unsigned long long *>(p);
        p += 16;
        sm.bcast = reinterpret_cast<uint32_t *>(p);
        p += 4 * sizeof(uint32_t);
        sm.flag = reinterpret_cast<int *>(p);
        p += 4 * sizeof(int);
        sm.pfx = reinterpret_cast<int32_t *>(p);
        p += (size_t)(a.LH + 1) * sizeof(int32_t);
        sm.lens = reinterpret_cast<int32_t *>(p);
        p += (size_t)a.LH * sizeof(int32_t);
        sm.kc = reinterpret_cast<int32_t *>(p);
    }
    const int g = blockIdx.x / a.cta_per_group;
    const int rr = blockIdx.x % a.cta_per_group;
    const bool single = a.n_groups == 1 && a.waves == 1;
    uint32_t epoch = 0;
    bool alive = true;

    for (int wave = 0; wave < a.waves && alive; wave++) {
        SeqState st;
        st.b = wave * a.n_groups + g;
        st.active = g < a.n_groups && st.b < a.B;
        st.done = true;
        st.kappa = 0;
        st.x0 = st.x1 = 0;
        st.wv = false;
        st.wres = 0;
        st.wn = 0;
        bool finalized = false;
        if (st.active) {
            // page prefix and lengths of this sequence's heads
            uint32_t carry = 0;
            int64_t nsum = 0;
            for (int base = 0; base < a.LH; base += blockDim.x) {
                const int cl = base + threadIdx.x;
                const int32_t n =
                    cl < a.LH ? clamp_len(__ldcg(a.len + (int64_t)st.b * a.LH + cl), a.max_pages, a.status) : 0;
                if (cl < a.LH) { sm.lens[cl] = n; sm.kc[cl] = 0; }
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
                a.kept[c] = a.pre_kept ? __ldg(a.pre_kept + c) : 0;
            }
            st.t = __ldg(a.t + st.b);
            int64_t m = __ldg(a.m_global + st.b);
            if (a.seq) {
                // the budget left after the forced entries, at most the entries left to rank
                m -= (int64_t)__ldcg(a.seq + 2 * st.b);
                const int64_t left = (int64_t)__ldcg(a.seq + 2 * st.b + 1);
                if (m > left) m = left;
            }
            st.m = m < 0 ? 0 : (m > st.n ? st.n : m);
            st.rank = (uint32_t)st.m;
            st.pk = 0;
            st.pm = 0;
            st.done = (st.m == 0) || (st.m == st.n);
            st.kappa = st.m == 0 ? 0ull : ~0ull;
            {
                const uint32_t *w = a.win + (size_t)st.b * 4;
                st.wv = !a.seq && __ldcg(w) != 0u;
                st.wlo = __ldcg(w + 1);
                st.whi = __ldcg(w + 2);
            }
            hist_pass(a, sm, st, 0, g, wave, /*fill=*/true, /*count=*/!st.done);
        }
        alive = grid_barrier(a.bar, ++epoch, a.status, sm.flag);
        if (alive && st.active && !st.done) try_window(a, sm, st);
        for (int p = 0; alive; p++) {
            if (st.active && !st.done) scan_pass(a, sm, st, p, g, wave);
            if (st.active && st.done && !finalized) {
                final_pass(a, sm, st);
                if (rr == 0 && threadIdx.x == 0) {
                    // trivial budgets report kappa now; the others once every
                    // CTA's largest kept key is in (last CTA to leave)
                    if (st.m == 0 || st.m == st.n) {
                        a.kappa[st.b] = st.kappa;
                        a.cnt[(size_t)st.b * 4 + 2] = 0xFFFFFFFFu;
                    } else {
                        a.cnt[(size_t)st.b * 4 + 2] = (uint32_t)st.wres;
                        a.cnt[(size_t)st.b * 4 + 3] = st.wn;
                    }
                }
                finalized = true;
            }
            // one sequence: every CTA is resolved together, no closing barrier
            if (single && finalized) break;
            if (st.active && !st.done) {
                if (rr == 0 && threadIdx.x == 0) atomicOr(a.more + wave * NPASS + p, 1u);
                hist_pass(a, sm, st, p + 1, g, wave, false, true);
            }
            alive = grid_barrier(a.bar, ++epoch, a.status, sm.flag);
            if (!alive) break;
            if (__ldcg(a.more + wave * NPASS + p) == 0u) break;
        }
    }
    if (!alive) return;
    // Clear this launch's scratch for the next one.  With several groups the
    // closing barrier has passed, so every histogram read is done and the
    // CTAs clear slices in parallel; with one group CTAs leave without a
    // closing barrier and the last CTA to leave (ticket) clears them.  The
    // last CTA also resets the barrier counter and the window counters and
    // builds the free-page plan -- every kept count is final once all CTAs
    // have flushed and taken the ticket.  (A timed-out barrier skips this;
    // the workspace must then be re-initialised.)
    const size_t nh = (size_t)a.waves * NPASS * a.n_groups * NBINS;
    if (!single) {
        for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < nh; i += (size_t)gridDim.x * blockDim.x)
            a.hist[i] = 0u;
        for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < a.waves * NPASS; i += gridDim.x * blockDim.x)
            a.more[i] = 0u;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        __threadfence();
        *sm.flag = atomicAdd(a.leave, 1u) == gridDim.x - 1 ? 1 : 0;
    }
    __syncthreads();
    if (!*sm.flag) return;
    __threadfence();
    if (single) {
        for (size_t i = threadIdx.x; i < nh; i += blockDim.x) a.hist[i] = 0u;
        for (int i = threadIdx.x; i < a.waves * NPASS; i += blockDim.x) a.more[i] = 0u;
    }
    for (int b = threadIdx.x; b < a.B; b += blockDim.x) {
        const uint32_t wres = __ldcg(a.cnt + (size_t)b * 4 + 2);
        if (wres != 0xFFFFFFFFu) {
            const uint64_t kap = __ldcg(a.kmax + b) + 1ull;
            a.kappa[b] = kap;
            if (!a.seq) window_next(a.win + (size_t)b * 4, kap, (int)wres, __ldcg(a.cnt + (size_t)b * 4 + 3));
        }
        a.kmax[b] = 0ull;
    }
    __syncthreads();
    for (int i = threadIdx.x; i < 4 * a.B; i += blockDim.x) a.cnt[i] = 0u;
    // free-page plan over all heads: plan[c] = pages freed in heads < c
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
        *a.bar = 0u;
        *a.leave = 0u;
        __threadfence();
    }
}

// Scratch of the allocation-free selection entry point: status word, grid
// barrier counter, exit ticket, continuation flags, radix histograms and window candidates for up
// to NOALLOC_MAX_B sequences (about 0.9 MiB).  Every GPU that loads the
// library holds it until the process exits; all calls share it.
static __device__ __align__(256) uint32_t g_noalloc_scratch[NOALLOC_WORDS];

}  // namespace

// Device address of g_noalloc_scratch on the current device, looked up once
// per device (the host-side name is only a stand-in, not a device address).
int noalloc_scratch(uint32_t **out, const char **err) {
    static std::mutex mu;
    static uint32_t *ptrs[NOALLOC_MAX_DEVICES] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= NOALLOC_MAX_DEVICES) {
        *err = "no usable current CUDA device";
        return -1;
    }
    std::lock_guard<std::mutex> lock(mu);
    if (!ptrs[dev]) {
        void *p = nullptr;
        const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess || !p) {
            *err = cudaGetErrorString(e);
            return -1;
        }
        ptrs[dev] = static_cast<uint32_t *>(p);
    }
    *out = ptrs[dev];
    return 0;
}


int select_max_smem() { return 227 * 1024; }

SelectGrid select_grid_for(const rkv_cache_t &c, int sm_count) {
    SelectGrid g{};
    const int LH = c.L * c.H;
    g.threads = SEL_THREADS;
    const int ctas = sm_count;  // one CTA per SM (large shared-memory key cache)
    g.n_groups = c.B < ctas ? c.B : ctas;
    g.cta_per_group = ctas / g.n_groups;
    g.waves = (c.B + g.n_groups - 1) / g.n_groups;
    const int fixed = 4 * NBINS * 4 + 40 * 4 + 16 + 16 + 16 + (3 * LH + 1) * 4;
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
