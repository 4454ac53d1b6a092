// budget.cu -- budget-allocation variants of the selection (sm_100a): a
// budget per head, and the ContourKV allocation (recency floor in every
// head, a fixed budget for flat heads, the rest of the global budget ranked
// globally over the other heads).
//
// Cache What Lasts (TRIM-KV), core mechanism 4: a head over its budget drops
// its lowest retention beta^(t-i) (Make Each Token Count, Methodology 3,
// names this fixed per-head allocation as what its global budget replaces).
// Trust the Mass (ContourKV), Methodology 3: the dropped-mass statistic
// marks flat cells, which get a fixed budget; every cell keeps a recency
// floor; the importance scores are reused with this allocation.
//
// One CTA per head.  The head's entries are scored once (position and
// score key cached in shared memory up to HEAD_CACHE entries, recomputed
// from global memory beyond); exact in-CTA radix selects find the floor's
// oldest position (the r-th largest position) and the head's budget
// threshold among the entries outside the floor (64-bit key: score key,
// then position, so equal scores keep ascending positions); keep masks are
// written with one word per thread.  ContourKV's global part is the global
// selection kernel run over the remaining entries (see SelectArgs).
#include "common.cuh"
#include "internal.h"

namespace rkv {

namespace {

constexpr int BT = 256;              // threads per head CTA
constexpr int HEAD_CACHE = 12288;    // entries cached in shared memory (8 bytes each)
constexpr int PER_T = NBINS / BT;    // histogram bins per thread in a scan

struct HeadSm {
    uint32_t hist[NBINS];
    uint32_t scan[40];
    uint32_t bc[4];
    int32_t red[BT / 32];
    uint32_t key[HEAD_CACHE];        // score key (high word), KEY_INVALID for a bad entry
    int32_t pos[HEAD_CACHE];
};

// Score key and position of slot k of head c (validity as the global
// selection: NaN log-retention, age outside [1, 2^24) or a negative
// position are bad input).
__device__ __forceinline__ void entry_of(const BudgetArgs &a, int64_t c, int k, int32_t t, uint32_t *hi,
                                         int32_t *pos) {
    const int32_t pg = __ldg(a.block_table + c * a.max_pages + k / PAGE);
    const int64_t row = (int64_t)pg * PAGE + k % PAGE;
    const int32_t p = __ldg(a.pos_pool + row);
    const float lb = __ldg(a.lb_pool + row);
    const int64_t age = (int64_t)t - p;
    *pos = p;
    if ((lb != lb) || age < 1 || age >= (1 << 24) || p < 0) {
        set_status(a.status, RKV_DEV_BAD_INPUT);
        *hi = KEY_INVALID;
        return;
    }
    float s = __fmul_rn((float)(int32_t)age, lb);
    if (s == 0.0f) s = 0.0f;
    *hi = score_key_desc(s);
}

// Exact rank-th smallest (1-based) 64-bit key among the keys get(k, &K)
// accepts, k in [0, n): radix digits 11/11/10 | 11/11/10, stopping once the
// chosen bucket is taken whole.  Returns the exclusive threshold: exactly
// `rank` accepted keys are below it (keys are distinct).
template <typename Get>
__device__ uint64_t head_select(HeadSm &sm, int n, uint32_t rank, Get &&get) {
    uint64_t pk = 0ull, pm = 0ull;
    for (int p = 0; p < NPASS; p++) {
        for (int i = threadIdx.x; i < NBINS; i += BT) sm.hist[i] = 0u;
        __syncthreads();
        for (int k = threadIdx.x; k < n; k += BT) {
            uint64_t K;
            if (get(k, &K) && ((K ^ pk) & pm) == 0ull)
                atomicAdd(&sm.hist[key_digit((uint32_t)(K >> 32), (uint32_t)K, p)], 1u);
        }
        __syncthreads();
        uint32_t v[PER_T], loc = 0;
#pragma unroll
        for (int j = 0; j < PER_T; j++) {
            v[j] = sm.hist[threadIdx.x * PER_T + j];
            loc += v[j];
        }
        uint32_t tot;
        const uint32_t ex = block_exclusive_scan(loc, sm.scan, &tot);
        if (threadIdx.x == 0) sm.bc[3] = 0u;
        __syncthreads();
        if (ex < rank && rank <= ex + loc) {
            uint32_t cum = ex;
#pragma unroll
            for (int j = 0; j < PER_T; j++) {
                if (cum < rank && rank <= cum + v[j]) {
                    sm.bc[0] = threadIdx.x * PER_T + j;
                    sm.bc[1] = rank - cum;
                    sm.bc[2] = v[j];
                    sm.bc[3] = 1u;
                }
                cum += v[j];
            }
        }
        __syncthreads();
        const uint32_t d = sm.bc[0], nr = sm.bc[1], h = sm.bc[2], found = sm.bc[3];
        __syncthreads();
        if (!found) return (pk | ~pm) + 1ull;  // fewer accepted keys than the rank: unreachable
        const int sh = digit_shift(p);
        pk |= (uint64_t)d << sh;
        pm |= ((1ull << digit_bits(p)) - 1ull) << sh;
        rank = nr;
        if (h == nr || p == NPASS - 1) return (pk | ~pm) + 1ull;
    }
    return (pk | ~pm) + 1ull;
}

__global__ void __launch_bounds__(BT) head_budget_kernel(BudgetArgs a) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    HeadSm &sm = *reinterpret_cast<HeadSm *>(smem_raw);
    const int64_t c = blockIdx.x;
    const int b = (int)(c / a.LH);
    const int n = clamp_len(__ldg(a.len + c), a.max_pages, a.status);
    const int32_t t = __ldg(a.t + b);
    const bool cached = n <= HEAD_CACHE;
    // ---- score every entry once (cache when it fits) ----
    int nvalid = 0;
    for (int k = threadIdx.x; k < n; k += BT) {
        uint32_t hi;
        int32_t pos;
        entry_of(a, c, k, t, &hi, &pos);
        if (cached) {
            sm.key[k] = hi;
            sm.pos[k] = pos;
        }
        nvalid += hi != KEY_INVALID ? 1 : 0;
    }
    {
        uint32_t tot;
        block_exclusive_scan((uint32_t)nvalid, sm.scan, &tot);
        nvalid = (int)tot;
    }
    auto get = [&](int k, uint32_t *hi, int32_t *pos) {
        if (cached) {
            *hi = sm.key[k];
            *pos = sm.pos[k];
        } else {
            entry_of(a, c, k, t, hi, pos);
        }
    };
    // ---- flat head (ContourKV): binary32 mean of the query heads' dropped mass ----
    bool flat = false;
    int32_t m;
    if (a.mode == RKV_BUDGET_CONTOUR) {
        float sum = 0.0f;
        for (int g = 0; g < a.G; g++) sum = __fadd_rn(sum, __ldg(a.dm_prev + c * a.G + g));
        flat = __fdiv_rn(sum, (float)a.G) > a.tau;
        m = flat ? max(a.flat_budget, 0) : 0;
    } else {
        m = max(__ldg(a.m_head + c), 0);
    }
    // ---- recency floor: entries at or after the r-th largest position ----
    const int r = a.mode == RKV_BUDGET_CONTOUR ? max(a.floor_r, 0) : 0;
    int32_t floor_pos = 0x7FFFFFFF;  // no floor
    int nfloor = 0;
    if (r > 0) {
        if (r >= nvalid) {
            floor_pos = (int32_t)0x80000000;  // every valid entry
            nfloor = nvalid;
        } else {
            // descending positions as ascending keys (0xFFFFFFFF - pos) << 32
            // (pos >= 0, distinct); the r smallest are the floor
            const uint64_t kf = head_select(sm, n, (uint32_t)r, [&](int k, uint64_t *K) {
                uint32_t hi;
                int32_t pos;
                get(k, &hi, &pos);
                *K = (uint64_t)(0xFFFFFFFFu - (uint32_t)pos) << 32;
                return hi != KEY_INVALID;
            });
            // key < kf  <=>  0xFFFFFFFF - pos < X  <=>  pos >= 2^32 - X
            const int64_t X = (int64_t)(kf >> 32) + ((kf & 0xFFFFFFFFull) != 0ull ? 1 : 0);
            floor_pos = (int32_t)((1ll << 32) - X);
            nfloor = r;
        }
    }
    // ---- the head's own budget over the entries outside the floor ----
    const int eligible = nvalid - nfloor;
    if (m > eligible) m = eligible;
    uint64_t kap = 0ull;  // entries outside the floor with key < kap are kept
    if (m == eligible) {
        kap = ~0ull;
    } else if (m > 0) {
        kap = head_select(sm, n, (uint32_t)m, [&](int k, uint64_t *K) {
            uint32_t hi;
            int32_t pos;
            get(k, &hi, &pos);
            *K = ((uint64_t)hi << 32) | (uint32_t)pos;
            return hi != KEY_INVALID && pos < floor_pos;
        });
    }
    // ---- keep words (one per thread) and the head's count ----
    const int W = (n + PAGE - 1) / PAGE;
    int cnt = 0;
    for (int w = threadIdx.x; w < W; w += BT) {
        uint32_t bits = 0u;
        for (int j = 0; j < PAGE; j++) {
            const int k = w * PAGE + j;
            if (k >= n) break;
            uint32_t hi;
            int32_t pos;
            get(k, &hi, &pos);
            if (hi == KEY_INVALID) continue;
            const bool fl = pos >= floor_pos;
            const bool own = !fl && ((((uint64_t)hi << 32) | (uint32_t)pos) < kap || kap == ~0ull);
            if (fl || own) bits |= 1u << j;
        }
        a.mask[c * a.max_pages + w] = (uint16_t)bits;
        cnt += __popc(bits);
    }
    uint32_t tot;
    block_exclusive_scan((uint32_t)cnt, sm.scan, &tot);
    if (threadIdx.x == 0) {
        a.kept[c] = (int32_t)tot;
        if (a.mode == RKV_BUDGET_CONTOUR) {
            a.floor_pos[c] = floor_pos;
            a.skip[c] = flat ? 1 : 0;
            // forced entries, and the entries left for the global ranking
            atomicAdd(a.seq + 2 * b, (unsigned long long)tot);
            if (!flat) atomicAdd(a.seq + 2 * b + 1, (unsigned long long)(nvalid - nfloor));
        } else {
            a.n_pre[c] = n;
        }
    }
}

// Free-page plan of a selection written by the per-head kernel: plan[c] =
// pages freed by compaction in heads < c, plan[C] = total, plan[C+1] = the
// stack top; kappa (no sequence-wide threshold) = 0.
__global__ void __launch_bounds__(1024) plan_kernel(const int32_t *n_pre, const int32_t *kept, int32_t *plan,
                                                    const int32_t *free_top, uint64_t *kappa, int C, int B) {
    __shared__ uint32_t scan[40];
    uint32_t carry = 0;
    for (int base = 0; base < C; base += blockDim.x) {
        const int c = base + threadIdx.x;
        uint32_t f = 0;
        if (c < C) {
            const int32_t np = __ldcg(n_pre + c), nk = __ldcg(kept + c);
            f = (uint32_t)((np + PAGE - 1) / PAGE - (nk + PAGE - 1) / PAGE);
        }
        uint32_t tot;
        const uint32_t ex = block_exclusive_scan(f, scan, &tot);
        if (c < C) plan[c] = (int32_t)(carry + ex);
        carry += tot;
    }
    for (int i = threadIdx.x; i < B; i += blockDim.x) kappa[i] = 0ull;
    if (threadIdx.x == 0) {
        plan[C] = (int32_t)carry;
        plan[C + 1] = __ldcg(free_top);
    }
}

}  // namespace

cudaError_t launch_head_budget(const BudgetArgs &a, cudaStream_t s) {
    if (a.C == 0) return cudaSuccess;
    const int smem = (int)sizeof(HeadSm);
    cudaError_t e = cudaFuncSetAttribute(head_budget_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    head_budget_kernel<<<a.C, BT, smem, s>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_plan(const int32_t *n_pre, const int32_t *kept, int32_t *plan, const int32_t *free_top,
                        uint64_t *kappa, int C, int B, cudaStream_t s) {
    plan_kernel<<<1, 1024, 0, s>>>(n_pre, kept, plan, free_top, kappa, C, B);
    return cudaGetLastError();
}

}  // namespace rkv
