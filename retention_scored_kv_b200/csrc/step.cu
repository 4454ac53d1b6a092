// step.cu -- one decode step in a single cooperative launch (sm_100a):
// retention scores and global top-M selection, paged grouped-query decode
// attention over the kept entries with the dropped mass, compaction of the
// kept entries and the append of the new token.
//
// Make Each Token Count (DBTrimKV), Methodology 2-4, and Cache What Lasts
// (TRIM-KV), core mechanism 4: every cached entry scores (t - i) * log(beta_i),
// the top M_global of a sequence over all layers and heads are kept, ties by
// ascending (layer, head, position), and each head keeps its own length.
// Trust the Mass (ContourKV), Problem definition and Methodology 2-3: the
// softmax is renormalised over the kept keys, the dropped mass is the dense
// weight of the evicted keys, and evicted rows are physically removed.
//
// The separate kernels (selection, attention, compaction, append) each pay
// a launch and a grid ramp, and in steady decoding the selection scans only
// ~8 bytes per entry against the ~512 bytes of K/V the attention streams.
// This kernel folds them into one launch:
//  * Speculative pass.  Each sequence keeps a threshold window across calls
//    (a score-key range around the previous threshold).  The attention pass
//    fetches every page's positions and log-retentions with its K/V, builds
//    each entry's 64-bit rank key and classifies it: below the window's low
//    key -> kept, at or above its high key -> evicted, inside -> candidate.
//    Kept and evicted rows go straight into the online softmax; candidates
//    are set aside with their logits and V row.
//  * Resolve.  After one grid barrier, per sequence: if the keys below the
//    window are fewer than M and the candidates reach M, the threshold is the
//    (M - below)-th smallest candidate; each candidate's fate follows from
//    its rank among the candidates alone.
//  * Exact path.  Without a usable window (the prefill eviction, a miss, too
//    many candidates) an exact radix select runs in the same launch (digits
//    11/11/10 per 32-bit key half, per-sequence histograms behind bounded
//    grid barriers), writes the keep masks and kept counts, and the attention
//    pass then reads the masks.
//  * Tail.  Heads are dealt to CTAs in contiguous chunks: heads split across
//    CTAs or holding candidates are merged (the kept candidates' keep bits
//    were set when their fates were found), each head compacted (hole-fill,
//    freed pages pushed at the plan's offsets) and the new rows appended; a
//    pop waits (bounded) only for a page pushed in this call.
// Selection, keep masks, block tables, lengths and the free stack come out
// identical to the separate calls; attention outputs agree within rounding.
#include <cuda.h>

#include "attn_core.cuh"
#include "common.cuh"
#include "internal.h"

namespace rkv {

namespace {

using namespace core;

constexpr int NTH = ATTN_THREADS;
constexpr int NWARP = NTH / 32;
constexpr int MAXB = STEP_MAX_B;
constexpr int PPT = 1;           // pages per thread per round of the exact select's sweeps
constexpr int HGRP = 8;          // sequences histogrammed together in the exact select
constexpr int CMP_PAIRS = 1024;  // hole/source pairs resolved per compaction round
static_assert(STEP_HEADS_PER_CTA == NTH, "tail chunk = one head per thread");

enum : uint32_t { SF_TRIVIAL = 1u, SF_WIN = 2u, SF_DONE = 4u };

// Tail scratch (offsets in the big region).
constexpr int T_STASH = 0;                       // int32 [6][NTH]
constexpr int T_CL = 6 * NTH * 4;                // int32 [WIN_CAP] candidate list of one head
constexpr int T_PAIRS = T_CL + WIN_CAP * 4;      // int2 [CMP_PAIRS]
constexpr int T_TBL = T_PAIRS + CMP_PAIRS * 8;   // int32 [mp], src [mp+1], hole [mp+1], uint16 msk [mp]
// Candidates of this CTA's own tail heads, listed once after the resolve
// ((head - first own head) << 16 | index in its sequence's list), in the
// block-wide compaction's pair buffer (unused until the heavy tasks); more
// than OWN_CAP and the warp merges scan their sequence's list instead.
constexpr int T_OWN = T_PAIRS;
constexpr int OWN_CAP = CMP_PAIRS * 8 / 4;
// Per-warp scratch of the warp-level merge and compaction (used before the
// block-wide fallbacks, which reuse the same bytes from T_TBL on).
constexpr int RCAP = 16;    // partial records a warp merges (CTAs a head spans)
constexpr int CCAP = 128;   // candidates of one head a warp merges
constexpr int HCAP = 64;    // evicted entries of one head a warp compacts
struct WarpScr {
    const float *recp[RCAP];
    float st[4][RCAP * 8];  // mk, lk, me, le of each record and query row
    float fk[RCAP * 8];     // record weights 2^(mk_rec - mk)
    float mk[8], lk[8];
    int32_t cidx[CCAP];     // candidate indices (within the sequence's list)
    int32_t cfate[CCAP];
    float cz[CCAP * 8];     // logits, then weights 2^(z - mk) (0 for evicted)
    int32_t holes[HCAP], srcs[HCAP];
};
constexpr int WARP_SCR = 9216;
static_assert(sizeof(WarpScr) <= WARP_SCR, "warp scratch");
constexpr int T_WARP = T_TBL;

__host__ __device__ constexpr size_t tail_bytes(int mp) {
    const size_t cmp = (size_t)T_TBL + (size_t)mp * 4 + 2 * ((size_t)mp + 1) * 4 + (size_t)mp * 2 + 16;
    const size_t wrp = (size_t)T_WARP + (size_t)NWARP * WARP_SCR;
    return cmp > wrp ? cmp : wrp;
}
constexpr size_t RADIX_BYTES = (size_t)HGRP * NBINS * 4;
constexpr int KT = NTH * PPT;                // pages per round of the exact select's sweeps
constexpr int T_SPFX = (int)RADIX_BYTES;     // int32 [KT + 1] page-prefix chunk, after the histograms
constexpr size_t RESOLVE_BYTES = (size_t)WIN_CAP * 8;

// Fixed part of shared memory (offsets from the 1024-aligned base, the same
// for every instance): per-sequence state, scan scratch, flags, the CTA range
// starts and the pipeline barriers; the big region follows at S_BIG.
constexpr int MAX_NBAR = 2 * NCW * 8 + 2 * QR;
// Local resolve: every CTA ranks all candidates itself when there are at
// most RES_CAP of them and at most CADD_CAP heads (their kept-candidate
// counts are tallied in shared memory), so no second grid barrier is needed.
constexpr int RES_CAP = 1024;

constexpr int CADD_CAP = 8192;
// Radix select of the local resolve (sequences, state, histograms; big region).
constexpr int RSEL_MAXB = 16;
constexpr int T_RSEL = T_WARP + RES_CAP * 8 + CADD_CAP * 4;  // [RSEL_MAXB] 32-byte states
constexpr int T_RHIST = T_RSEL + RSEL_MAXB * 32;             // uint32 [RSEL_MAXB][256]
constexpr int S_LO = 0, S_HI = S_LO + MAXB * 8, S_KAP = S_HI + MAXB * 8, S_PK = S_KAP + MAXB * 8,
              S_PM = S_PK + MAXB * 8, S_KMX = S_PM + MAXB * 8, S_M = S_KMX + MAXB * 8, S_T = S_M + MAXB * 8,
              S_N = S_T + MAXB * 4, S_RANK = S_N + MAXB * 4, S_FL = S_RANK + MAXB * 4, S_ABOVE = S_FL + MAXB * 4,
              S_NC = S_ABOVE + MAXB * 4, S_OFF = S_NC + MAXB * 4, S_WRES = S_OFF + MAXB * 4,
              S_H1 = S_WRES + MAXB * 4, S_SCAN = S_H1 + MAXB * 4, S_MISC = S_SCAN + 4 * 36 * 4, S_MISC64 = S_MISC + 64 * 4,
              S_RLO = S_MISC64 + 8 * 8, S_FATE = S_RLO + (MAX_ATTN_CTAS + 1) * 4,
              S_BAR = (S_FATE + RES_CAP + 15) / 16 * 16,
              S_BIG = (S_BAR + MAX_NBAR * 8 + 1023) / 1024 * 1024;

// Shared memory: the fixed part (pipeline barriers, per-sequence state, scan
// scratch) first, then the big region: attention stages, positions /
// log-retentions, query ring, merge slots and stage metadata during an
// attention pass; scratch of the other phases outside it.
template <class M, int D, int G>
struct StepLayout {
    static constexpr int STAGE_BYTES = M::PAGE_BYTES * 2;
    static constexpr int NSW0 = 131072 / (NCW * STAGE_BYTES);
    static constexpr int NSW = NSW0 < 1 ? 1 : (NSW0 > 8 ? 8 : NSW0);   // stages per consumer warp
    static constexpr int NST = NCW * NSW;
    static constexpr int QBYTES = G * D * 4;
    static constexpr int REC = G * (D + 4);                   // partial record floats
    static constexpr int WSLOT = G * D + 4 * G + 4;           // merge slot: acc, mk, lk, me, le, candidates
    static constexpr int NBAR = 2 * NST + 2 * QR;
    static constexpr int B_STAGE = 0;
    static constexpr int B_POSLB = NST * STAGE_BYTES;         // [NST][16 positions, 16 log-retentions]
    static constexpr int B_Q = B_POSLB + NST * 128;
    static constexpr int B_MERGE = B_Q + QR * QBYTES;
    static constexpr int MFAC = G * NCW + G;                  // per parity: weights [G][NCW], kept sums [G]
    static constexpr int B_MFAC = B_MERGE + 2 * NCW * WSLOT * 4;
    static constexpr int B_META = B_MFAC + 2 * MFAC * 4;
    static constexpr int BIG_ATTN = B_META + NST * 4;
    static_assert(STAGE_BYTES % M::STAGE_ALIGN == 0, "stage alignment");
    static_assert(QBYTES % 16 == 0, "query block must be a 16-byte multiple");
    static_assert(NBAR <= NTH && NBAR <= MAX_NBAR, "barrier init");
    static_assert(M::STAGE_ALIGN <= 1024, "big region alignment");
    static_assert(BIG_ATTN >= T_SPFX + (KT + 1) * 4 && BIG_ATTN >= (int)RESOLVE_BYTES, "scratch");
    static_assert(BIG_ATTN >= T_RHIST + RSEL_MAXB * 256 * 4, "local resolve scratch");
    static size_t smem(int mp) {
        const size_t big = tail_bytes(mp) > (size_t)BIG_ATTN ? tail_bytes(mp) : (size_t)BIG_ATTN;
        return (size_t)S_BIG + big + 1024;
    }
};

// Shared memory through one base pointer (offsets are constants, so no
// per-array pointers stay live across the attention pass).
struct Sm {
    unsigned char *base;
    template <typename T>
    __device__ __forceinline__ T *at(int off) const { return reinterpret_cast<T *>(base + off); }
    __device__ __forceinline__ uint64_t *bars() const { return at<uint64_t>(S_BAR); }
    __device__ __forceinline__ uint64_t *lo() const { return at<uint64_t>(S_LO); }
    __device__ __forceinline__ uint64_t *hi() const { return at<uint64_t>(S_HI); }
    __device__ __forceinline__ uint64_t *kap() const { return at<uint64_t>(S_KAP); }
    __device__ __forceinline__ uint64_t *pk() const { return at<uint64_t>(S_PK); }
    __device__ __forceinline__ uint64_t *pm() const { return at<uint64_t>(S_PM); }
    __device__ __forceinline__ unsigned long long *kmx() const { return at<unsigned long long>(S_KMX); }
    __device__ __forceinline__ int64_t *m() const { return at<int64_t>(S_M); }
    __device__ __forceinline__ int32_t *t() const { return at<int32_t>(S_T); }
    __device__ __forceinline__ uint32_t *n() const { return at<uint32_t>(S_N); }
    __device__ __forceinline__ uint32_t *rank() const { return at<uint32_t>(S_RANK); }
    __device__ __forceinline__ uint32_t *fl() const { return at<uint32_t>(S_FL); }
    __device__ __forceinline__ uint32_t *above() const { return at<uint32_t>(S_ABOVE); }
    __device__ __forceinline__ uint32_t *nc() const { return at<uint32_t>(S_NC); }
    __device__ __forceinline__ uint32_t *off() const { return at<uint32_t>(S_OFF); }
    __device__ __forceinline__ uint32_t *wres() const { return at<uint32_t>(S_WRES); }
    // keys in the threshold's 1024-wide score-key bucket (second radix pass)
    __device__ __forceinline__ uint32_t *h1() const { return at<uint32_t>(S_H1); }
    __device__ __forceinline__ uint32_t *scan() const { return at<uint32_t>(S_SCAN); }
    __device__ __forceinline__ int *misc() const { return at<int>(S_MISC); }
    __device__ __forceinline__ int64_t *misc64() const { return at<int64_t>(S_MISC64); }
    __device__ __forceinline__ int32_t *rlo() const { return at<int32_t>(S_RLO); }
    __device__ __forceinline__ int8_t *fate() const { return at<int8_t>(S_FATE); }
    __device__ __forceinline__ int32_t *own() const { return reinterpret_cast<int32_t *>(base + S_BIG + T_OWN); }
    __device__ __forceinline__ unsigned char *big() const { return base + S_BIG; }
};

// misc slots
enum { MS_CSTART = 0, MS_CLAST, MS_RADIX, MS_MISS, MS_BAR, MS_TOTAL, MS_NCL,
       MS_ACTIVE, MS_QN, MS_QH, MS_NOWN, MS_HNEXT };

struct Ctx {
    int32_t TP, x0, x1, pfx_start;  // flattened pages (< 2^27)
    int c_start, c_last;
    bool last, evict;
    int32_t top0;
    uint32_t par, epoch;
    bool exact;      // the exact selection ran (its thresholds are reported in the tail)
    int passes;      // exact-select passes run (histograms to clear)
    int attn_runs;   // attention passes run
    // The pipeline barriers are initialised once per launch; a later
    // attention pass continues their phases.  Round-robin passes number
    // their pages after the earlier passes' (pbase) and their query slots
    // after the earlier passes' heads (qbase); head-per-warp passes count
    // every consumer warp's pages over the launch (wcnt[0] in a consumer
    // warp; in a producer warp wcnt[0] and wcnt[1] for the two consumer
    // warps it feeds).  Every pass of a launch takes the same mode, and
    // producer and consumer count alike.
    int32_t pbase;
    int qbase;
    uint32_t wcnt[2];
};

// This call's half of the per-call counters: head_kept[C], head_flag[C],
// seq[B][4], arrivals.
__device__ __forceinline__ uint32_t *ctr_of(const StepArgs &a, const Ctx &cx) {
    return a.ctr + (size_t)cx.par * a.ctr_words;
}
__device__ __forceinline__ uint32_t *head_kept_of(const StepArgs &a, const Ctx &cx) { return ctr_of(a, cx); }
__device__ __forceinline__ uint32_t *head_flag_of(const StepArgs &a, const Ctx &cx) { return ctr_of(a, cx) + a.C; }
__device__ __forceinline__ uint32_t *seqc_of(const StepArgs &a, const Ctx &cx) {
    return ctr_of(a, cx) + 2 * (size_t)a.C;
}
__device__ __forceinline__ uint32_t *arrive_of(const StepArgs &a, const Ctx &cx) {
    return ctr_of(a, cx) + 2 * (size_t)a.C + 4 * (size_t)a.B;
}

template <int NSCAN>
__device__ __forceinline__ void block_scan_n(const uint32_t (&v)[NSCAN], uint32_t (&ex)[NSCAN],
                                             uint32_t (&tot)[NSCAN], uint32_t *scratch) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
    uint32_t x[NSCAN];
#pragma unroll
    for (int s = 0; s < NSCAN; s++) {
        x[s] = v[s];
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t y = __shfl_up_sync(0xFFFFFFFFu, x[s], o);
            if (lane >= o) x[s] += y;
        }
        if (lane == 31) scratch[s * 36 + warp] = x[s];
    }
    __syncthreads();
    if (warp == 0) {
#pragma unroll
        for (int s = 0; s < NSCAN; s++) {
            uint32_t w = lane < nw ? scratch[s * 36 + lane] : 0u;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const uint32_t y = __shfl_up_sync(0xFFFFFFFFu, w, o);
                if (lane >= o) w += y;
            }
            if (lane < nw) scratch[s * 36 + lane] = w;
            if (lane == 31) scratch[s * 36 + 32] = w;
        }
    }
    __syncthreads();
#pragma unroll
    for (int s = 0; s < NSCAN; s++) {
        ex[s] = (warp > 0 ? scratch[s * 36 + warp - 1] : 0u) + x[s] - v[s];
        tot[s] = scratch[s * 36 + 32];
    }
    __syncthreads();
}

// Rank key of one entry: hi = order-preserving map of s = fl32(float(t - i)
// * lb) (smaller = ranked first), lo = (l*H + h) << ibits | i.  Returns false
// for an entry the method cannot score (NaN log-retention, age outside
// [1, 2^24), position out of range).
__device__ __forceinline__ bool entry_key(int32_t t, uint32_t cl, int32_t pos, float lb, int ibits, uint64_t *K) {
    const int64_t age = (int64_t)t - pos;
    if ((lb != lb) || age < 1 || age >= (1 << 24) || pos < 0 || (ibits < 32 && (uint32_t)pos >= (1u << ibits)))
        return false;
    float s = __fmul_rn((float)(int32_t)age, lb);
    if (s == 0.0f) s = 0.0f;
    *K = ((uint64_t)score_key_desc(s) << 32) | (uint32_t)(((uint64_t)cl << ibits) | (uint32_t)pos);
    return true;
}

// The same key's hi word alone, under the same rejection rule, in 32-bit
// arithmetic: plim = 2^ibits (2^31 for ibits = 32), so one unsigned compare
// rejects negative and out-of-range positions; with pos >= 0, t > pos keeps
// t - pos from overflowing.  The lo word is (cl << ibits) | pos, truncated to
// 32 bits.
__device__ __forceinline__ bool entry_key_hi(int32_t t, int32_t pos, float lb, uint32_t plim, uint32_t *hi) {
    if ((uint32_t)pos >= plim || t <= pos || (uint32_t)t - (uint32_t)pos >= (1u << 24) || lb != lb) return false;
    float s = __fmul_rn((float)(int32_t)((uint32_t)t - (uint32_t)pos), lb);
    if (s == 0.0f) s = 0.0f;
    *hi = score_key_desc(s);
    return true;
}

__device__ __forceinline__ uint32_t below_bits(int w, int nn) {
    const int lo = w * PAGE;
    if (lo + PAGE <= nn) return 0xFFFFu;
    if (lo >= nn) return 0u;
    return (1u << (nn - lo)) - 1u;
}

// Exclusive prefix sums of two word arrays in place (va[W], vb[W] receive
// the totals): each thread sums a contiguous chunk, one block scan of the
// chunk sums, then the chunks are rewritten as running prefixes.
__device__ void scan_words2(int32_t *va, int32_t *vb, int W, uint32_t *scratch) {
    const int CH = (W + NTH - 1) / NTH;
    const int w0 = min(W, (int)threadIdx.x * CH), w1 = min(W, w0 + CH);
    uint32_t sum[2] = {0u, 0u};
    for (int w = w0; w < w1; w++) {
        sum[0] += (uint32_t)va[w];
        sum[1] += (uint32_t)vb[w];
    }
    uint32_t ex[2], tot[2];
    block_scan_n<2>(sum, ex, tot, scratch);
    for (int w = w0; w < w1; w++) {
        const uint32_t xa = (uint32_t)va[w], xb = (uint32_t)vb[w];
        va[w] = (int32_t)ex[0];
        vb[w] = (int32_t)ex[1];
        ex[0] += xa;
        ex[1] += xb;
    }
    if (threadIdx.x == 0) {
        va[W] = (int32_t)tot[0];
        vb[W] = (int32_t)tot[1];
    }
    __syncthreads();
}

// CTA whose page range holds flattened page x: the largest j with
// rlo[j] <= x (empty ranges share their start with the next one).
__device__ __forceinline__ int owner_rlo(const int32_t *rlo, int nct, int64_t x) {
    int lo = 0, hi = nct - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (rlo[mid] <= x) lo = mid; else hi = mid - 1;
    }
    return lo;
}

// ------------------------------------------------------------- prologue ----
template <class M, int D, int G>
__device__ __forceinline__ void prologue(const StepArgs &a, const Sm &sm, Ctx &cx, const CUtensorMap *tmk,
                                         const CUtensorMap *tmv) {
    const int tid = threadIdx.x, nct = gridDim.x;
    // every independent load first: the counter half, the stack top, this
    // thread's head lengths (LPT in registers) and its sequence's step inputs
    // and threshold window
    constexpr int LPT = 4;
    cx.evict = a.m_global != nullptr;
    cx.par = __ldcg(a.parity) & 1u;
    cx.top0 = __ldcg(a.free_top);
    const int CS = (a.C + NTH - 1) / NTH;
    const int h0 = min(a.C, tid * CS), h1 = min(a.C, h0 + CS);
    int32_t nl[LPT];
#pragma unroll
    for (int u = 0; u < LPT; u++) nl[u] = h0 + u < h1 ? clamp_len(__ldcg(a.len + h0 + u), a.max_pages, a.status) : 0;
    auto len_at = [&](int c) -> int32_t {
        const int u = c - h0;
        int32_t v = 0;
#pragma unroll
        for (int q = 0; q < LPT; q++)
            if (u == q) v = nl[q];
        return u < LPT ? v : clamp_len(__ldcg(a.len + c), a.max_pages, a.status);
    };
    int32_t seq_t = 0;
    int64_t seq_m = 0;
    uint32_t seq_w[3] = {0u, 0u, 0u};
    if (tid < a.B) {
        seq_t = __ldg(a.t + tid);
        if (cx.evict) {
            seq_m = __ldg(a.m_global + tid);
            seq_w[0] = __ldcg(a.win + (size_t)tid * 4);
            seq_w[1] = __ldcg(a.win + (size_t)tid * 4 + 1);
            seq_w[2] = __ldcg(a.win + (size_t)tid * 4 + 2);
        }
    }
    uint32_t *other = a.ctr + (size_t)(cx.par ^ 1u) * a.ctr_words;
    // the other half is the next call's: clear it now
    for (size_t i = (size_t)blockIdx.x * NTH + tid; i < (size_t)a.ctr_words; i += (size_t)nct * NTH) other[i] = 0u;
    cx.epoch = 0;
    cx.exact = false;
    cx.passes = 0;
    cx.attn_runs = 0;
    cx.pbase = 0;
    cx.qbase = 0;
    cx.wcnt[0] = cx.wcnt[1] = 0u;
    if (tid < MAXB) sm.n()[tid] = 0u;
    if (tid < 64) sm.misc()[tid] = 0;
    if (tid == 0) {
        sm.misc()[MS_CSTART] = a.C;
        sm.misc()[MS_CLAST] = -1;
    }
    if (M::USES_TMAP && tid == 0) {
        prefetch_tensormap(tmk);
        prefetch_tensormap(tmv);
    }
    __syncthreads();
    uint32_t my_pages = 0;
    for (int c = h0; c < h1; c++) {
        const int32_t n = len_at(c);
        my_pages += (uint32_t)((n + PAGE - 1) / PAGE);
        atomicAdd(&sm.n()[c / a.LH], (uint32_t)n);
        if (c % nct == (int)blockIdx.x) {
            a.npre[c] = n;
            if (cx.evict) a.n_pre[c] = n;
        }
    }
    uint32_t TPu;
    const uint32_t my_pfx = block_exclusive_scan(my_pages, sm.scan(), &TPu);
    cx.TP = (int32_t)TPu;
    cx.x0 = (int32_t)range_lo(blockIdx.x, cx.TP, nct);
    cx.x1 = (int32_t)range_lo(blockIdx.x + 1, cx.TP, nct);
    // every CTA's range start, once (the tail looks them up instead of dividing)
    for (int j = tid; j <= nct; j += NTH) sm.rlo()[j] = (int32_t)range_lo(j, cx.TP, nct);
    cx.last = blockIdx.x == nct - 1;
    // first head of the range (first c with pfx + max(pages, 1) > x0) and
    // the last head the range visits (last c with pfx < x1; every head for
    // the last CTA)
    int first = a.C, lastc = -1;
    int64_t first_pfx = 0;
    {
        int64_t p = my_pfx;
        for (int c = h0; c < h1; c++) {
            const int64_t pg = (len_at(c) + PAGE - 1) / PAGE;
            if (first == a.C && p + (pg > 0 ? pg : 1) > cx.x0) {
                first = c;
                first_pfx = p;
            }
            if (p < cx.x1 || cx.last) lastc = c;
            p += pg;
        }
    }
    if (first < a.C) atomicMin(&sm.misc()[MS_CSTART], first);
    if (lastc >= 0) atomicMax(&sm.misc()[MS_CLAST], lastc);
    __syncthreads();
    if (first < a.C && first == sm.misc()[MS_CSTART]) sm.misc64()[0] = first_pfx;
    // per-sequence setup
    if (tid < a.B) {
        const int b = tid;
        sm.t()[b] = seq_t;
        const int64_t N = sm.n()[b];
        uint32_t fl = SF_TRIVIAL | SF_DONE;
        uint64_t lo = ~0ull, hi = ~0ull, kap = ~0ull;
        int64_t m = N;
        if (cx.evict) {
            m = seq_m < 0 ? 0 : (seq_m > N ? N : seq_m);
            if (m == 0 || m == N) {
                kap = m == 0 ? 0ull : ~0ull;
                lo = hi = kap;
            } else {
                if (seq_w[0] != 0u) {
                    fl = SF_WIN;
                    lo = (uint64_t)seq_w[1] << 32;
                    hi = (uint64_t)seq_w[2] << 32;
                } else {
                    fl = 0u;
                    atomicOr(&sm.misc()[MS_RADIX], 1);
                }
                kap = 0ull;
            }
        }
        sm.m()[b] = m;
        sm.fl()[b] = fl;
        sm.lo()[b] = lo;
        sm.hi()[b] = hi;
        sm.kap()[b] = kap;
        sm.wres()[b] = 0u;
        sm.above()[b] = 0u;
        sm.nc()[b] = 0u;
    }
    __syncthreads();
    cx.c_start = sm.misc()[MS_CSTART];
    cx.c_last = sm.misc()[MS_CLAST];
    cx.pfx_start = cx.c_start < a.C ? (int32_t)sm.misc64()[0] : cx.TP;
}

// -------------------------------------------------------- attention pass ----
// Head-per-warp mode: when this CTA's range holds at least NCW heads and
// they are short (at most HPW_PAGES pages per head on average), each head
// goes to one consumer warp whole (head c_start + j to warp j mod NCW), so no
// head needs a merge across warps; otherwise pages are dealt to the warps
// round-robin.
constexpr int HPW_PAGES = 64;
__device__ __forceinline__ bool head_per_warp(const Ctx &cx) {
    const int64_t heads = (int64_t)cx.c_last - cx.c_start + 1;
    return heads >= NCW && (int64_t)(cx.x1 - cx.x0) <= (int64_t)HPW_PAGES * heads;
}

// The heads of one consumer warp in the head-per-warp mode: c_start + w,
// then every NCW-th head while c <= c_last, each with its page prefix (the
// pages of the heads stepped over are summed from one warp-wide round of
// length loads).  Every lane of the calling warp runs it.
struct HeadCursor {
    int c, n, pages;
    int64_t pfx;
    __device__ void step(const StepArgs &a, int from, int64_t pfx_from, int skip) {
        const int lane = threadIdx.x & 31;
        const int h = from + lane;
        const int32_t ln = (lane <= skip && h < a.C) ? clamp_len(__ldcg(a.len + h), a.max_pages, nullptr) : 0;
        int pg = lane < skip ? (ln + PAGE - 1) / PAGE : 0;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) pg += __shfl_xor_sync(0xFFFFFFFFu, pg, o);
        c = from + skip;
        pfx = pfx_from + pg;
        n = __shfl_sync(0xFFFFFFFFu, ln, skip);
        pages = (n + PAGE - 1) / PAGE;
    }
    __device__ void init(const StepArgs &a, const Ctx &cx, int w) { step(a, cx.c_start, cx.pfx_start, w); }
    __device__ void next(const StepArgs &a) { step(a, c, pfx, NCW); }
    __device__ bool valid(const Ctx &cx) const { return c <= cx.c_last; }
};

// Warms L1 with a head's query block (G*D floats), 128 bytes per lane.
template <int G, int D>
__device__ __forceinline__ void prefetch_q(const float *q, int lane) {
    constexpr int LINES = (G * D * 4 + 127) / 128;
    if (lane < LINES) asm volatile("prefetch.global.L1 [%0];" ::"l"(q + lane * 32));
}

// Pages are dealt to consumer warps round-robin (page li -> warp li % NCW);
// each consumer warp owns a private ring filled in order by producer warp
// (warp % NPW), so every mbarrier has one producer and one consumer.  SPEC
// classifies entries against the sequences' windows; otherwise the keep
// masks come from memory (or every entry is kept when nothing is evicted).
template <class M, int D, int G, bool SPEC>
__device__ __forceinline__ void attn_pass(const StepArgs &a, const Sm &sm, Ctx &cx, const CUtensorMap *tmk,
                                          const CUtensorMap *tmv) {
    using LY = StepLayout<M, D, G>;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    uint64_t *full = sm.bars(), *empty = full + LY::NST, *qfull = empty + LY::NST, *qempty = qfull + QR;
    unsigned char *stage = sm.big() + LY::B_STAGE;
    unsigned char *poslb = sm.big() + LY::B_POSLB;
    float *qring = reinterpret_cast<float *>(sm.big() + LY::B_Q);
    float *merge = reinterpret_cast<float *>(sm.big() + LY::B_MERGE);
    uint32_t *meta = reinterpret_cast<uint32_t *>(sm.big() + LY::B_META);
    __syncthreads();
    if (cx.attn_runs == 0) {
        if (tid < LY::NBAR) {
            // full: producer; empty: the owning consumer warp; qfull: producer 0; qempty: every consumer warp
            mbar_init(full + tid, tid >= 2 * LY::NST + QR ? NCW : 1);
        }
        fence_mbar_init();
        __syncthreads();
    }
    const int64_t pb0 = cx.pbase;
    // timeout site codes: 0x10 (speculative pass) / 0x20 (mask pass) + wait kind
    const int32_t site = SPEC ? 0x10 : 0x20;
    cx.attn_runs++;
    const bool masks = !SPEC && cx.evict;

    if (warp >= NCW) {
        // =============================== producers ===============================
        if constexpr (REG_SPLIT) setmaxnreg_dec<PRODUCER_REGS>();
        const int pw = warp - NCW;
        Walker w;
        w.init(a.len, a.C, a.max_pages, cx.x1, cx.last, cx.c_start, cx.pfx_start);
        const uint64_t pol_kv = policy_evict_first();
        const uint64_t pol_keep = policy_evict_last();
        int nq = cx.qbase;
        int c, pages, n;
        int64_t pfx;
        while (w.next(&c, &pfx, &pages, &n)) {
            if (pages == 0) continue;
            const int64_t pa = max(pfx, (int64_t)cx.x0), pb = min(pfx + pages, (int64_t)cx.x1);
            if (pw == 0 && lane == 0) {
                const int slot = nq % QR;
                mbar_wait(&qempty[slot], ((nq / QR) & 1) ^ 1, a.status, site + 1);
                mbar_arrive_expect_tx(&qfull[slot], LY::QBYTES);
                bulk_g2s(qring + slot * G * D, a.q + (int64_t)c * G * D, LY::QBYTES, &qfull[slot], pol_keep);
            }
            nq++;
            // block-table entries (and keep words) of the next 32 pages are
            // loaded while this block's copies are issued
            int32_t phys_n = 0;
            uint32_t kp_n = 0xFFFFu;
            auto load_block = [&](int64_t base) {
                const int64_t i = base + lane;
                if (i < pb && ((int)((i - cx.x0 + pb0) % NCW)) % NPW == pw) {
                    phys_n = __ldg(a.block_table + (int64_t)c * a.max_pages + (i - pfx));
                    if (masks) kp_n = (uint32_t)__ldcg(a.keep_mask + (int64_t)c * a.max_pages + (i - pfx));
                }
            };
            load_block(pa);
            for (int64_t base = pa; base < pb; base += 32) {
                const int64_t i = base + lane;
                const bool mine = i < pb && ((int)((i - cx.x0 + pb0) % NCW)) % NPW == pw;
                const int32_t phys = phys_n;
                uint32_t m = 0;
                if (mine) {
                    const int64_t pidx = i - pfx;
                    const int nv = min(PAGE, n - (int)pidx * PAGE);
                    const uint32_t valid = nv >= PAGE ? 0xFFFFu : ((1u << nv) - 1u);
                    m = SPEC ? (valid << 16) : ((kp_n & valid) | (valid << 16));
                }
                if (base + 32 < pb) load_block(base + 32);
                uint32_t todo = __ballot_sync(0xFFFFFFFFu, mine);
                while (todo) {
                    const int j = __ffs(todo) - 1;
                    todo &= todo - 1;
                    const int32_t pj = __shfl_sync(0xFFFFFFFFu, phys, j);
                    const uint32_t mj = __shfl_sync(0xFFFFFFFFu, m, j);
                    if (lane == 0) {
                        const int64_t li = base + j - cx.x0 + pb0;
                        const int cw = (int)(li % NCW);
                        const int64_t nw = li / NCW;
                        const int sg = cw * LY::NSW + (int)(nw % LY::NSW);
                        mbar_wait(&empty[sg], (uint32_t)((nw / LY::NSW) & 1) ^ 1u, a.status, site + 2);
                        meta[sg] = mj;
                        const bool load_v = SPEC || (mj & 0xFFFFu);
                        mbar_arrive_expect_tx(&full[sg], M::PAGE_BYTES * (load_v ? 2 : 1) + (SPEC ? 128u : 0u));
                        M::issue(stage + sg * LY::STAGE_BYTES, load_v, pj, &full[sg], a.k_pool, a.v_pool, tmk, tmv,
                                 pol_kv);
                        if (SPEC) {
                            bulk_g2s(poslb + sg * 128, a.pos_pool + (int64_t)pj * PAGE, 64, &full[sg], pol_keep);
                            bulk_g2s(poslb + sg * 128 + 64, a.lb_pool + (int64_t)pj * PAGE, 64, &full[sg], pol_keep);
                        }
                    }
                    __syncwarp();
                }
            }
        }
        cx.qbase = nq;
    } else {
        // ================================ consumers ================================
        if constexpr (REG_SPLIT) setmaxnreg_inc<CONSUMER_REGS>();
        Walker w;
        w.init(a.len, a.C, a.max_pages, cx.x1, cx.last, cx.c_start, cx.pfx_start);
        int nq = cx.qbase;
        int c, pages, n;
        int64_t pfx;
        typename M::State st;
        while (w.next(&c, &pfx, &pages, &n)) {
            if (pages == 0) {
                // a head with no entries: o = 0, lse = -inf, dropped = 0
                if (warp == 0) {
                    for (int e = lane; e < G * D; e += 32) a.out[(int64_t)c * G * D + e] = 0.0f;
                    if (lane < G) {
                        if (a.lse) a.lse[(int64_t)c * G + lane] = -INFINITY;
                        if (a.dropped) a.dropped[(int64_t)c * G + lane] = 0.0f;
                    }
                }
                continue;
            }
            const int64_t pa = max(pfx, (int64_t)cx.x0), pb = min(pfx + pages, (int64_t)cx.x1);
            const bool whole = (pfx >= cx.x0) && (pfx + pages <= cx.x1);
            {
                const int slot = nq % QR;
                mbar_wait(&qfull[slot], (nq / QR) & 1, a.status, site + 3);
                M::load_q(st, qring + slot * G * D, a.qscale, lane);
                __syncwarp();
                if (lane == 0) mbar_arrive(&qempty[slot]);
            }
            int b = 0;
            uint32_t cl = 0;
            uint64_t wlo = 0, whi = 0;
            int32_t tb = 0;
            if constexpr (SPEC) {
                b = c / a.LH;
                cl = (uint32_t)(c - b * a.LH);
                wlo = sm.lo()[b];
                whi = sm.hi()[b];
                tb = sm.t()[b];
            }
            uint32_t kc = 0, ncw = 0;
            // virtual page index v = li + pb0 (this pass's pages follow the earlier passes')
            const int64_t la = pa - cx.x0 + pb0, lb = pb - cx.x0 + pb0;
            for (int64_t v = la + (((int64_t)warp - la) % NCW + NCW) % NCW; v < lb; v += NCW) {
                const int64_t li = v - pb0;
                const int64_t nw = v / NCW;
                const int sg = warp * LY::NSW + (int)(nw % LY::NSW);
                mbar_wait(&full[sg], (uint32_t)((nw / LY::NSW) & 1), a.status, site + 4);
                const uint32_t mt = meta[sg];
                const unsigned char *sk = stage + sg * LY::STAGE_BYTES;
                uint32_t keepm, evm, candm = 0u, cbase = 0u;
                float *zdst = nullptr;
                int zcap = 0;
                if constexpr (SPEC) {
                    const uint32_t valid = mt >> 16;
                    const int r = lane & 15;
                    const unsigned char *pl = poslb + sg * 128;
                    const int32_t pos = reinterpret_cast<const int32_t *>(pl)[r];
                    const float lbv = reinterpret_cast<const float *>(pl + 64)[r];
                    bool kept = false, cand = false, bad = false;
                    uint64_t K = 0ull;
                    if ((valid >> r) & 1u) {
                        bad = !entry_key(tb, cl, pos, lbv, a.ibits, &K);
                        kept = !bad && K < wlo;
                        cand = !bad && !kept && K < whi;
                    }
                    keepm = __ballot_sync(0xFFFFFFFFu, kept) & 0xFFFFu;
                    candm = __ballot_sync(0xFFFFFFFFu, cand) & 0xFFFFu;
                    if (__ballot_sync(0xFFFFFFFFu, bad) && lane == 0) set_status(a.status, RKV_DEV_BAD_INPUT);
                    evm = valid & ~keepm & ~candm;
                    const int64_t pidx = li + cx.x0 - pfx;
                    if (lane == 0) a.keep_mask[(int64_t)c * a.max_pages + pidx] = (uint16_t)keepm;
                    kc += (uint32_t)__popc(keepm);
                    if (candm) {
                        if (lane == 0) {
                            cbase = atomicAdd(seqc_of(a, cx) + (size_t)b * 4 + 1, (uint32_t)__popc(candm));
                            atomicOr(head_flag_of(a, cx) + c, 1u);
                        }
                        cbase = __shfl_sync(0xFFFFFFFFu, cbase, 0);
                        if (lane < 16 && cand) {
                            const uint32_t idx = cbase + (uint32_t)__popc(candm & ((1u << r) - 1u));
                            if (idx < (uint32_t)WIN_CAP) {
                                a.ckey[(size_t)b * WIN_CAP + idx] = K;
                                a.cslot[(size_t)b * WIN_CAP + idx] = (int32_t)(pidx * PAGE + r);
                            }
                        }
                        zdst = a.cz + ((size_t)b * WIN_CAP + cbase) * G;
                        zcap = cbase < (uint32_t)WIN_CAP ? (int)(WIN_CAP - cbase) : 0;
                        ncw += (uint32_t)__popc(candm);
                    }
                } else {
                    keepm = mt & 0xFFFFu;
                    evm = (mt >> 16) & ~keepm;
                }
                M::template page<SPEC>(st, sk, sk + M::PAGE_BYTES, keepm, evm, lane, candm, zdst, zcap);
                if constexpr (SPEC) {
                    if (candm) {
                        // set the candidates' V rows aside
                        uint32_t bits = candm;
                        uint32_t k = cbase;
                        while (bits) {
                            const int j = __ffs(bits) - 1;
                            bits &= bits - 1;
                            if (k < (uint32_t)WIN_CAP)
                                M::copy_row(sk + M::PAGE_BYTES, j, a.cv + ((size_t)b * WIN_CAP + k) * a.row_bytes, lane);
                            k++;
                        }
                    }
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&empty[sg]);
            }
            if constexpr (SPEC) {
                if (lane == 0 && kc) {
                    atomicAdd(head_kept_of(a, cx) + c, kc);
                    atomicAdd(seqc_of(a, cx) + (size_t)b * 4, kc);
                }
            }
            const int par = nq & 1;
            float *slot = merge + (par * NCW + warp) * LY::WSLOT;
            M::flush(st, slot, lane);
            if (lane == 0) slot[G * D + 4 * G] = (float)ncw;
            nq++;
            named_bar_sync(1, NCW * 32);

            // ---- merge the warps (consumer threads) ----
            // per query row g (eight lanes, one per warp part): merged
            // statistics by 8-lane shuffles, and each warp's weight
            // 2^(mk_w - mk) in a table; then every output element is the
            // weighted sum of the warps' parts
            static_assert(NCW == 8 && G <= 8, "eight lanes per query row in two warps");
            const float *mb = merge + par * NCW * LY::WSLOT;
            float *fac = reinterpret_cast<float *>(sm.big() + LY::B_MFAC) + par * LY::MFAC;
            float hc = 0.0f;
#pragma unroll
            for (int wi = 0; wi < NCW; wi++) hc += mb[wi * LY::WSLOT + G * D + 4 * G];
            // whole head without candidates: final; else a record for the tail
            const int dest = whole ? (hc > 0.0f ? 1 : 0) : 2;
            float *rec = dest == 1 ? a.hrec + (int64_t)c * LY::REC
                                   : a.partial + ((int64_t)blockIdx.x * 2 + ((pfx < cx.x0) ? 0 : 1)) * LY::REC;
            if (tid < 64) {
                const int g = tid >> 3, wi = tid & 7;
                const bool on = g < G;
                const float *src = mb + wi * LY::WSLOT;
                const float mkw = on ? src[G * D + g] : -INFINITY, mew = on ? src[G * D + 2 * G + g] : -INFINITY;
                const float lkw = on ? src[G * D + G + g] : 0.0f, lew = on ? src[G * D + 3 * G + g] : 0.0f;
                Merged s;
                s.mk = mkw;
                s.me = mew;
#pragma unroll
                for (int o = 1; o < 8; o <<= 1) {
                    s.mk = fmaxf(s.mk, __shfl_xor_sync(0xFFFFFFFFu, s.mk, o));
                    s.me = fmaxf(s.me, __shfl_xor_sync(0xFFFFFFFFu, s.me, o));
                }
                const float fk = (mkw == -INFINITY) ? 0.0f : ex2(mkw - s.mk);
                const float fe = (mew == -INFINITY) ? 0.0f : ex2(mew - s.me);
                s.lk = lkw * fk;
                s.le = lew * fe;
#pragma unroll
                for (int o = 1; o < 8; o <<= 1) {
                    s.lk += __shfl_xor_sync(0xFFFFFFFFu, s.lk, o);
                    s.le += __shfl_xor_sync(0xFFFFFFFFu, s.le, o);
                }
                if (on) fac[g * NCW + wi] = fk;
                if (on && wi == 0) {
                    fac[G * NCW + g] = s.lk;
                    if (dest == 0) {
                        if (a.lse) a.lse[(int64_t)c * G + g] = s.lk > 0.0f ? (s.mk + __log2f(s.lk)) * LN2 : -INFINITY;
                        if (a.dropped) a.dropped[(int64_t)c * G + g] = dm_of(s);
                    } else {
                        rec[G * D + g] = s.mk;
                        rec[G * D + G + g] = s.lk;
                        rec[G * D + 2 * G + g] = s.me;
                        rec[G * D + 3 * G + g] = s.le;
                    }
                }
            }
            named_bar_sync(1, NCW * 32);
            // four consecutive elements per thread (16-byte loads and stores:
            // slots, records and rows of outputs are 16-byte multiples)
            static_assert((G * D) % 4 == 0 && LY::WSLOT % 4 == 0 && LY::REC % 4 == 0, "16-byte groups");
            for (int e = tid * 4; e < G * D; e += NCW * 32 * 4) {
                const int g = e / D;
                float4 av = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
#pragma unroll
                for (int wi = 0; wi < NCW; wi++) {
                    const float4 x = *reinterpret_cast<const float4 *>(mb + wi * LY::WSLOT + e);
                    const float f = fac[g * NCW + wi];
                    av.x += x.x * f;
                    av.y += x.y * f;
                    av.z += x.z * f;
                    av.w += x.w * f;
                }
                if (dest == 0) {
                    const float lk = fac[G * NCW + g];
                    float4 o = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
                    if (lk > 0.0f) o = make_float4(av.x / lk, av.y / lk, av.z / lk, av.w / lk);
                    *reinterpret_cast<float4 *>(a.out + (int64_t)c * G * D + e) = o;
                } else {
                    *reinterpret_cast<float4 *>(rec + e) = av;
                }
            }
            if (dest == 1 && tid == 0) atomicOr(head_flag_of(a, cx) + c, 2u);
        }
        cx.qbase = nq;
        if constexpr (REG_SPLIT) setmaxnreg_dec<LAUNCH_REGS>();
    }
    cx.pbase = pb0 + (cx.x1 - cx.x0);
    __syncthreads();
    if (warp >= NCW) {
        if constexpr (REG_SPLIT) setmaxnreg_inc<LAUNCH_REGS>();
    }
}

template <class M, int D, int G, bool SPEC>
__device__ __forceinline__ void attn_pass_hpw(const StepArgs &a, const Sm &sm, Ctx &cx, const CUtensorMap *tmk,
                                          const CUtensorMap *tmv) {
    using LY = StepLayout<M, D, G>;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    uint64_t *full = sm.bars(), *empty = full + LY::NST;
    unsigned char *stage = sm.big() + LY::B_STAGE;
    unsigned char *poslb = sm.big() + LY::B_POSLB;
    float *qring = reinterpret_cast<float *>(sm.big() + LY::B_Q);
    float *merge = reinterpret_cast<float *>(sm.big() + LY::B_MERGE);
    uint32_t *meta = reinterpret_cast<uint32_t *>(sm.big() + LY::B_META);
    __syncthreads();
    if (cx.attn_runs == 0) {
        if (tid < LY::NBAR) {
            // full: producer; empty: the owning consumer warp; qfull: producer 0; qempty: every consumer warp
            mbar_init(full + tid, tid >= 2 * LY::NST + QR ? NCW : 1);
        }
        fence_mbar_init();
        __syncthreads();
    }
    // timeout site codes: 0x10 (speculative pass) / 0x20 (mask pass) + wait kind
    const int32_t site = SPEC ? 0x10 : 0x20;
    cx.attn_runs++;
    const bool masks = !SPEC && cx.evict;

    if (warp >= NCW) {
        // =============================== producers ===============================
        if constexpr (REG_SPLIT) setmaxnreg_dec<PRODUCER_REGS>();
        const int pw = warp - NCW;
        const uint64_t pol_kv = policy_evict_first();
        const uint64_t pol_keep = policy_evict_last();
        uint32_t cnt0 = cx.wcnt[0], cnt1 = cx.wcnt[1];  // pages issued to consumer warps pw, pw + NPW
        // one page to consumer warp cw (lane 0): its next stage, once free
        auto issue = [&](int cw, uint32_t k, int32_t pj, uint32_t mj) {
            const int sg = cw * LY::NSW + (int)(k % LY::NSW);
            mbar_wait(&empty[sg], ((k / LY::NSW) & 1u) ^ 1u, a.status, site + 2);
            meta[sg] = mj;
            const bool load_v = SPEC || (mj & 0xFFFFu);
            mbar_arrive_expect_tx(&full[sg], M::PAGE_BYTES * (load_v ? 2 : 1) + (SPEC ? 128u : 0u));
            M::issue(stage + sg * LY::STAGE_BYTES, load_v, pj, &full[sg], a.k_pool, a.v_pool, tmk, tmv, pol_kv);
            if (SPEC) {
                bulk_g2s(poslb + sg * 128, a.pos_pool + (int64_t)pj * PAGE, 64, &full[sg], pol_keep);
                bulk_g2s(poslb + sg * 128 + 64, a.lb_pool + (int64_t)pj * PAGE, 64, &full[sg], pol_keep);
            }
        };
        // the keep word (bit 16+ valid slots) of page pidx of a head of n entries
        auto page_meta = [&](int n, int64_t pidx, uint32_t kp) -> uint32_t {
            const int nv = min(PAGE, n - (int)pidx * PAGE);
            const uint32_t valid = nv >= PAGE ? 0xFFFFu : ((1u << nv) - 1u);
            return SPEC ? (valid << 16) : ((kp & valid) | (valid << 16));
        };
        {
            // head per warp: two cursors (the heads of consumer warps pw and
            // pw + NPW); a page is issued to whichever warp has a free stage,
            // so one warp's head end does not hold up the other
            HeadCursor hc[2];
            int64_t ip[2], pe[2], bb[2];
            int32_t bph[2];
            uint32_t bkp[2];
            bool on[2];
            // first page of the cursor's next head with pages in this range
            // (the consumer warp finishes the others by itself)
            auto seek = [&](int k) {
                for (;;) {
                    on[k] = hc[k].valid(cx);
                    if (!on[k]) break;
                    ip[k] = max(hc[k].pfx, (int64_t)cx.x0);
                    pe[k] = min(hc[k].pfx + hc[k].pages, (int64_t)cx.x1);
                    if (ip[k] < pe[k]) break;
                    hc[k].next(a);
                }
            };
            auto load_blk = [&](int k) {
                bb[k] = ip[k];
                const int64_t i = ip[k] + lane;
                bph[k] = 0;
                bkp[k] = 0xFFFFu;
                if (i < pe[k]) {
                    const int64_t pidx = i - hc[k].pfx;
                    bph[k] = __ldg(a.block_table + (int64_t)hc[k].c * a.max_pages + pidx);
                    if (masks) bkp[k] = (uint32_t)__ldcg(a.keep_mask + (int64_t)hc[k].c * a.max_pages + pidx);
                }
            };
#pragma unroll
            for (int k = 0; k < 2; k++) {
                hc[k].init(a, cx, pw + k * NPW);
                seek(k);
                if (on[k]) load_blk(k);
            }
            const uint64_t t0 = globaltimer_ns();
            uint32_t spins = 0;
            while (on[0] || on[1]) {
                bool moved = false;
#pragma unroll
                for (int k = 0; k < 2; k++) {
                    if (!on[k]) continue;
                    const int cw = pw + k * NPW;
                    const uint32_t kk = k == 0 ? cnt0 : cnt1;
                    const int sg = cw * LY::NSW + (int)(kk % LY::NSW);
                    int ok = 0;
                    if (lane == 0) ok = mbar_try_wait(&empty[sg], ((kk / LY::NSW) & 1u) ^ 1u) ? 1 : 0;
                    ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
                    if (!ok) continue;
                    const int j = (int)(ip[k] - bb[k]);
                    const int32_t pj = __shfl_sync(0xFFFFFFFFu, bph[k], j);
                    const uint32_t kp = __shfl_sync(0xFFFFFFFFu, bkp[k], j);
                    const uint32_t mj = page_meta(hc[k].n, ip[k] - hc[k].pfx, kp);
                    if (lane == 0) issue(cw, kk, pj, mj);  // the stage is free: no wait
                    __syncwarp();
                    if (k == 0) cnt0 = kk + 1u; else cnt1 = kk + 1u;
                    moved = true;
                    if (++ip[k] >= pe[k]) {
                        hc[k].next(a);
                        seek(k);
                        if (on[k]) load_blk(k);
                    } else if (ip[k] - bb[k] == 32) {
                        load_blk(k);
                    }
                }
                if (!moved && (++spins & 255u) == 0 && globaltimer_ns() - t0 > 2000000000ull) {
                    if (lane == 0) record_timeout(a.status, site + 5);
                    break;
                }
            }
        }
        cx.wcnt[0] = cnt0;
        cx.wcnt[1] = cnt1;
    } else {
        // ================================ consumers ================================
        if constexpr (REG_SPLIT) setmaxnreg_inc<CONSUMER_REGS>();
        uint32_t cnt = cx.wcnt[0];  // pages this warp has taken in the launch
        typename M::State st;
        // per head: the window classification inputs, kept count and
        // candidate count of this warp's share of the head
        int c = 0, b = 0, n = 0;
        int64_t pfx = 0;
        uint32_t cl = 0;
        uint64_t wlo = 0, whi = 0;
        int32_t tb = 0;
        uint32_t kc = 0, ncw = 0;
        auto head_setup = [&]() {
            if constexpr (SPEC) {
                b = c / a.LH;
                cl = (uint32_t)(c - b * a.LH);
                wlo = sm.lo()[b];
                whi = sm.hi()[b];
                tb = sm.t()[b];
            }
            kc = 0;
            ncw = 0;
        };
        // page li of the range in stage sg, the k-th page of this warp
        auto take_page = [&](int64_t li, int sg, uint32_t k) {
            mbar_wait(&full[sg], (k / LY::NSW) & 1u, a.status, site + 4);
            const uint32_t mt = meta[sg];
            const unsigned char *sk = stage + sg * LY::STAGE_BYTES;
            uint32_t keepm, evm, candm = 0u, cbase = 0u;
            float *zdst = nullptr;
            int zcap = 0;
            if constexpr (SPEC) {
                const uint32_t valid = mt >> 16;
                const int r = lane & 15;
                const unsigned char *pl = poslb + sg * 128;
                const int32_t pos = reinterpret_cast<const int32_t *>(pl)[r];
                const float lbv = reinterpret_cast<const float *>(pl + 64)[r];
                bool kept = false, cand = false, bad = false;
                uint64_t K = 0ull;
                if ((valid >> r) & 1u) {
                    bad = !entry_key(tb, cl, pos, lbv, a.ibits, &K);
                    kept = !bad && K < wlo;
                    cand = !bad && !kept && K < whi;
                }
                keepm = __ballot_sync(0xFFFFFFFFu, kept) & 0xFFFFu;
                candm = __ballot_sync(0xFFFFFFFFu, cand) & 0xFFFFu;
                if (__ballot_sync(0xFFFFFFFFu, bad) && lane == 0) set_status(a.status, RKV_DEV_BAD_INPUT);
                evm = valid & ~keepm & ~candm;
                const int64_t pidx = li + cx.x0 - pfx;
                if (lane == 0) a.keep_mask[(int64_t)c * a.max_pages + pidx] = (uint16_t)keepm;
                kc += (uint32_t)__popc(keepm);
                if (candm) {
                    if (lane == 0) {
                        cbase = atomicAdd(seqc_of(a, cx) + (size_t)b * 4 + 1, (uint32_t)__popc(candm));
                        atomicOr(head_flag_of(a, cx) + c, 1u);
                    }
                    cbase = __shfl_sync(0xFFFFFFFFu, cbase, 0);
                    if (lane < 16 && cand) {
                        const uint32_t idx = cbase + (uint32_t)__popc(candm & ((1u << r) - 1u));
                        if (idx < (uint32_t)WIN_CAP) {
                            a.ckey[(size_t)b * WIN_CAP + idx] = K;
                            a.cslot[(size_t)b * WIN_CAP + idx] = (int32_t)(pidx * PAGE + r);
                        }
                    }
                    zdst = a.cz + ((size_t)b * WIN_CAP + cbase) * G;
                    zcap = cbase < (uint32_t)WIN_CAP ? (int)(WIN_CAP - cbase) : 0;
                    ncw += (uint32_t)__popc(candm);
                }
            } else {
                keepm = mt & 0xFFFFu;
                evm = (mt >> 16) & ~keepm;
            }
            M::template page<SPEC>(st, sk, sk + M::PAGE_BYTES, keepm, evm, lane, candm, zdst, zcap);
            if constexpr (SPEC) {
                if (candm) {
                    // set the candidates' V rows aside
                    uint32_t bits = candm;
                    uint32_t ck = cbase;
                    while (bits) {
                        const int j = __ffs(bits) - 1;
                        bits &= bits - 1;
                        if (ck < (uint32_t)WIN_CAP)
                            M::copy_row(sk + M::PAGE_BYTES, j, a.cv + ((size_t)b * WIN_CAP + ck) * a.row_bytes, lane);
                        ck++;
                    }
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[sg]);
        };
        auto zero_head = [&]() {
            // a head with no entries: o = 0, lse = -inf, dropped = 0
            for (int e = lane; e < G * D; e += 32) a.out[(int64_t)c * G * D + e] = 0.0f;
            if (lane < G) {
                if (a.lse) a.lse[(int64_t)c * G + lane] = -INFINITY;
                if (a.dropped) a.dropped[(int64_t)c * G + lane] = 0.0f;
            }
        };
        {
            HeadCursor hcur;
            hcur.init(a, cx, warp);
            for (; hcur.valid(cx); hcur.next(a)) {
                c = hcur.c;
                n = hcur.n;
                pfx = hcur.pfx;
                const int pages = hcur.pages;
                if (pages == 0) {
                    zero_head();
                    continue;
                }
                const int64_t pa = max(pfx, (int64_t)cx.x0), pb = min(pfx + pages, (int64_t)cx.x1);
                const bool whole = (pfx >= cx.x0) && (pfx + pages <= cx.x1);
                M::load_q(st, a.q + (int64_t)c * G * D, a.qscale, lane);
                if (c + NCW <= cx.c_last) prefetch_q<G, D>(a.q + (int64_t)(c + NCW) * G * D, lane);
                head_setup();
                for (int64_t i = pa; i < pb; i++) {
                    take_page(i - cx.x0, warp * LY::NSW + (int)(cnt % LY::NSW), cnt);
                    cnt++;
                }
                if constexpr (SPEC) {
                    if (lane == 0 && kc) {
                        atomicAdd(head_kept_of(a, cx) + c, kc);
                        atomicAdd(seqc_of(a, cx) + (size_t)b * 4, kc);
                    }
                }
                // this warp holds the whole head (or this CTA's part of it)
                float *slot = merge + warp * LY::WSLOT;
                M::flush(st, slot, lane);
                __syncwarp();
                const int dest = whole ? (ncw > 0 ? 1 : 0) : 2;
                float *rec = dest == 1 ? a.hrec + (int64_t)c * LY::REC
                                       : a.partial + ((int64_t)blockIdx.x * 2 + ((pfx < cx.x0) ? 0 : 1)) * LY::REC;
                if (lane < G) {
                    const int g = lane;
                    Merged s;
                    s.mk = slot[G * D + g];
                    s.lk = slot[G * D + G + g];
                    s.me = slot[G * D + 2 * G + g];
                    s.le = slot[G * D + 3 * G + g];
                    if (dest == 0) {
                        if (a.lse) a.lse[(int64_t)c * G + g] = s.lk > 0.0f ? (s.mk + __log2f(s.lk)) * LN2 : -INFINITY;
                        if (a.dropped) a.dropped[(int64_t)c * G + g] = dm_of(s);
                    } else {
                        rec[G * D + g] = s.mk;
                        rec[G * D + G + g] = s.lk;
                        rec[G * D + 2 * G + g] = s.me;
                        rec[G * D + 3 * G + g] = s.le;
                    }
                }
                for (int e = lane * 4; e < G * D; e += 32 * 4) {  // 16-byte groups
                    const float4 x = *reinterpret_cast<const float4 *>(slot + e);
                    if (dest == 0) {
                        const float lk = slot[G * D + G + e / D];
                        float4 o = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
                        if (lk > 0.0f) o = make_float4(x.x / lk, x.y / lk, x.z / lk, x.w / lk);
                        *reinterpret_cast<float4 *>(a.out + (int64_t)c * G * D + e) = o;
                    } else {
                        *reinterpret_cast<float4 *>(rec + e) = x;
                    }
                }
                if (dest == 1 && lane == 0) atomicOr(head_flag_of(a, cx) + c, 2u);
                __syncwarp();
            }
        }
        cx.wcnt[0] = cnt;
        if constexpr (REG_SPLIT) setmaxnreg_dec<LAUNCH_REGS>();
    }
    __syncthreads();
    if (warp >= NCW) {
        if constexpr (REG_SPLIT) setmaxnreg_inc<LAUNCH_REGS>();
    }
}


// --------------------------------------------------------------- resolve ----
// After the speculative pass: per sequence, is the M-th key inside the
// window with every candidate stored?  If so every candidate's fate is its
// rank among the candidates (keys are distinct) and the M-th key gives the
// exclusive threshold.  Few candidates (RES_MODE_LOCAL): every CTA ranks all
// of them in shared memory, tallies kept candidates per head (sm.big() +
// T_WARP + RES_CAP*8, read by the tail's scan), keeps the fates in sm.fate()
// (indexed by the sequence's candidate offset + index) and sets the keep bits
// of its own heads; nothing crosses CTAs, so no barrier follows.  Otherwise
// (RES_MODE_GRID) each CTA ranks a slice, writes fates and kept counts to
// global memory, and a grid barrier must follow.  RES_MISS: some sequence
// missed (the exact path runs instead).
enum { RES_MISS = 0, RES_MODE_LOCAL = 1, RES_MODE_GRID = 2 };

// Local resolve, up to RSEL_MAXB sequences: the threshold of each sequence
// (its r-th smallest candidate key, r = m - above, 1 <= r <= nc) by a radix
// select in shared memory.  Digits of 8 bits start at the highest bit in
// which the sequence's candidates differ; each pass histograms the
// candidates still matching the chosen prefix and keeps the bucket holding
// the remaining rank, until that bucket holds one key (keys are distinct).
// Afterwards a candidate K is kept iff (K & mask) <= prefix, and is the
// threshold iff (K & mask) == prefix.
struct RselSeq {
    uint64_t prefix, mask;
    uint32_t rank, shift, done, pad;
};
static_assert(sizeof(RselSeq) == 32, "radix select state");

__device__ __forceinline__ int cand_seq(const Sm &sm, int B, int g) {
    int b = 0;
    while (b + 1 < B && (int)sm.off()[b + 1] <= g) b++;
    return b;
}

__device__ void resolve_radix(const StepArgs &a, const Sm &sm, const uint64_t *keys, int total) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    RselSeq *rs = reinterpret_cast<RselSeq *>(sm.big() + T_RSEL);
    uint32_t *hist = reinterpret_cast<uint32_t *>(sm.big() + T_RHIST);
    // bits in which each sequence's candidates differ from its first one
    if (tid < 2 * a.B) hist[tid] = 0u;
    __syncthreads();
    for (int g = tid; g < total; g += NTH) {
        const int b = cand_seq(sm, a.B, g);
        const uint64_t d = keys[g] ^ keys[sm.off()[b]];
        if (d >> 32) atomicOr(&hist[2 * b], (uint32_t)(d >> 32));
        if ((uint32_t)d) atomicOr(&hist[2 * b + 1], (uint32_t)d);
    }
    __syncthreads();
    if (tid < a.B) {
        const int b = tid;
        const uint32_t nb = sm.nc()[b];
        RselSeq r{};
        r.done = nb <= 1u ? 1u : 0u;
        r.rank = nb ? (uint32_t)(sm.m()[b] - (int64_t)sm.above()[b]) : 0u;
        const uint64_t d = ((uint64_t)hist[2 * b] << 32) | hist[2 * b + 1];
        const int hb = d ? 63 - __clzll((long long)d) : 0;  // highest differing bit
        r.shift = hb >= 7 ? (uint32_t)(hb - 7) : 0u;
        r.mask = hb >= 63 ? 0ull : ~((2ull << hb) - 1ull);    // bits above hb are common
        r.prefix = nb ? (keys[sm.off()[b]] & (r.done ? ~0ull : r.mask)) : 0ull;
        if (r.done) r.mask = ~0ull;
        rs[b] = r;
    }
    __syncthreads();
    for (int pass = 0; pass < 9; pass++) {
        if (tid == 0) {
            int act = 0;
            for (int b = 0; b < a.B; b++) act |= rs[b].done ? 0 : 1;
            sm.misc()[MS_ACTIVE] = act;
        }
        for (int i = tid; i < a.B * 256; i += NTH) hist[i] = 0u;
        __syncthreads();
        if (!sm.misc()[MS_ACTIVE]) break;
        for (int g = tid; g < total; g += NTH) {
            const int b = cand_seq(sm, a.B, g);
            const RselSeq &r = rs[b];
            const uint64_t K = keys[g];
            if (!r.done && (K & r.mask) == r.prefix) atomicAdd(&hist[b * 256 + (uint32_t)((K >> r.shift) & 255u)], 1u);
        }
        __syncthreads();
        for (int b = warp; b < a.B; b += NWARP) {
            RselSeq &r = rs[b];
            if (r.done) continue;
            const uint32_t *hb = hist + b * 256 + lane * 8;
            uint32_t loc = 0;
#pragma unroll
            for (int j = 0; j < 8; j++) loc += hb[j];
            uint32_t inc = loc;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const uint32_t y = __shfl_up_sync(0xFFFFFFFFu, inc, o);
                if (lane >= o) inc += y;
            }
            const uint32_t rank = r.rank;
            const bool mine = inc - loc < rank && rank <= inc;
            __syncwarp();
            if (mine) {
                // the bucket holding the rank, and the keys below it
                uint32_t cum = inc - loc, below = 0, h = 0;
                int dig = -1;
#pragma unroll
                for (int j = 0; j < 8; j++) {
                    const uint32_t e = hb[j];
                    if (dig < 0) {
                        if (rank <= cum + e) {
                            dig = lane * 8 + j;
                            h = e;
                            below = cum;
                        } else {
                            cum += e;
                        }
                    }
                }
                const uint32_t sh = r.shift;
                r.prefix = (r.prefix & ~(255ull << sh)) | ((uint64_t)dig << sh);
                r.mask |= 255ull << sh;
                r.rank = rank - below;
                if (h <= 1u || sh == 0u) {
                    r.done = 1u;
                } else {
                    r.shift = sh >= 8u ? sh - 8u : 0u;
                }
            }
            __syncwarp();
        }
        __syncthreads();
    }
}

__device__ int resolve(const StepArgs &a, const Sm &sm, const Ctx &cx) {
    const int tid = threadIdx.x, nct = gridDim.x;
    if (tid < a.B) {
        const int b = tid;
        if (!(sm.fl()[b] & SF_TRIVIAL)) {
            const uint32_t above = __ldcg(seqc_of(a, cx) + (size_t)b * 4), nc = __ldcg(seqc_of(a, cx) + (size_t)b * 4 + 1);
            const int64_t m = sm.m()[b];
            const bool hit = nc <= (uint32_t)WIN_CAP && (int64_t)above < m && m <= (int64_t)above + nc;
            sm.above()[b] = above;
            sm.nc()[b] = hit ? nc : 0u;
            // window outcome, used to resize it even if another sequence
            // sends the call down the exact path
            sm.wres()[b] = hit ? 1u : (nc > (uint32_t)WIN_CAP ? 3u : 2u);
            if (!hit) atomicOr(&sm.misc()[MS_MISS], 1);
        }
    }
    __syncthreads();
    if (sm.misc()[MS_MISS]) return RES_MISS;
    if (tid == 0) {
        uint32_t o = 0;
        for (int b = 0; b < a.B; b++) {
            sm.off()[b] = o;
            o += sm.nc()[b];
        }
        sm.misc()[MS_TOTAL] = (int)o;
    }
    __syncthreads();
    const int64_t total = sm.misc()[MS_TOTAL];
    if (total <= RES_CAP && a.C <= CADD_CAP) {
        uint64_t *keys = reinterpret_cast<uint64_t *>(sm.big() + T_WARP);
        uint32_t *cadd = reinterpret_cast<uint32_t *>(sm.big() + T_WARP + RES_CAP * 8);
        const int hc0 = (int)((int64_t)blockIdx.x * a.C / nct), hc1 = (int)((int64_t)(blockIdx.x + 1) * a.C / nct);
        for (int i = tid; i < a.C; i += NTH) cadd[i] = 0u;
        for (int g = tid; g < total; g += NTH) {
            int b = 0;
            while (b + 1 < a.B && (int64_t)sm.off()[b + 1] <= g) b++;
            keys[g] = __ldcg(a.ckey + (size_t)b * WIN_CAP + (g - sm.off()[b]));
        }
        __syncthreads();
        const bool radix = a.B <= RSEL_MAXB;
        if (radix) resolve_radix(a, sm, keys, (int)total);
        const RselSeq *rs = reinterpret_cast<const RselSeq *>(sm.big() + T_RSEL);
        if (tid == 0) sm.misc()[MS_NOWN] = 0;
        __syncthreads();
        for (int g = tid; g < total; g += NTH) {
            const int b = cand_seq(sm, a.B, g);
            const int ob = (int)sm.off()[b], nb = (int)sm.nc()[b];
            const uint64_t K = keys[g];
            bool kept, thr;
            if (radix) {
                const uint64_t km = K & rs[b].mask;
                kept = km <= rs[b].prefix;
                thr = km == rs[b].prefix;
            } else {
                // rank among the sequence's candidates: four independent
                // counts so the shared-memory loads overlap
                const uint64_t *kb = keys + ob;
                uint32_t l0 = 0, l1 = 0, l2 = 0, l3 = 0;
                int i = 0;
                for (; i + 4 <= nb; i += 4) {
                    l0 += kb[i] < K ? 1u : 0u;
                    l1 += kb[i + 1] < K ? 1u : 0u;
                    l2 += kb[i + 2] < K ? 1u : 0u;
                    l3 += kb[i + 3] < K ? 1u : 0u;
                }
                for (; i < nb; i++) l0 += kb[i] < K ? 1u : 0u;
                const uint32_t less = (l0 + l1) + (l2 + l3);
                const uint32_t r = (uint32_t)(sm.m()[b] - (int64_t)sm.above()[b]);
                kept = less < r;
                thr = less == r - 1;
            }
            sm.fate()[g] = kept ? 1 : 0;
            {
                const int cl = a.ibits >= 32 ? 0 : (int)((uint32_t)K >> a.ibits);
                const int c = b * a.LH + cl;
                if (c >= hc0 && c < hc1) {
                    const int at = atomicAdd(&sm.misc()[MS_NOWN], 1);
                    if (at < OWN_CAP) sm.own()[at] = ((c - hc0) << 16) | (g - ob);
                }
            }
            if (kept) {
                const int cl = a.ibits >= 32 ? 0 : (int)((uint32_t)K >> a.ibits);
                const int c = b * a.LH + cl;
                atomicAdd(cadd + c, 1u);
                if (c >= hc0 && c < hc1) {
                    const int slot = __ldcg(a.cslot + (size_t)b * WIN_CAP + (g - ob));
                    const uintptr_t addr = reinterpret_cast<uintptr_t>(a.keep_mask + (int64_t)c * a.max_pages + slot / PAGE);
                    atomicOr(reinterpret_cast<unsigned int *>(addr & ~(uintptr_t)3),
                             (1u << (slot % PAGE)) << ((addr & 2) ? 16 : 0));
                }
            }
            if (blockIdx.x == 0 && thr) {
                const uint64_t kap = K + 1ull;
                a.kappa[b] = kap;
                window_next(a.win + (size_t)b * 4, kap, 1, (uint32_t)nb);
            }
        }
        if (blockIdx.x == 0 && tid < a.B && (sm.fl()[tid] & SF_TRIVIAL)) a.kappa[tid] = sm.kap()[tid];
        __syncthreads();
        return RES_MODE_LOCAL;
    }
    const int64_t s0 = (int64_t)blockIdx.x * total / nct, s1 = (int64_t)(blockIdx.x + 1) * total / nct;
    uint64_t *keys = reinterpret_cast<uint64_t *>(sm.big());
    for (int b = 0; b < a.B; b++) {
        const int64_t ob = sm.off()[b], nb = sm.nc()[b];
        const int64_t jlo = max(s0, ob) - ob, jhi = min(s1, ob + nb) - ob;
        if (jlo >= jhi) continue;
        for (int i = tid; i < nb; i += NTH) keys[i] = __ldcg(a.ckey + (size_t)b * WIN_CAP + i);
        __syncthreads();
        const uint32_t r = (uint32_t)(sm.m()[b] - (int64_t)sm.above()[b]);  // 1-based
        // one warp per candidate: lanes count the smaller keys in parallel
        const int lane = tid & 31, warp = tid >> 5;
        for (int64_t j = jlo + warp; j < jhi; j += NWARP) {
            const uint64_t K = keys[j];
            uint32_t less = 0;
            for (int i = lane; i < nb; i += 32) less += keys[i] < K ? 1u : 0u;
            less = __reduce_add_sync(0xFFFFFFFFu, less);
            if (lane == 0) {
                const bool kept = less < r;
                a.cfate[(size_t)b * WIN_CAP + j] = kept ? 1 : 0;
                if (kept) {
                    const int cl = a.ibits >= 32 ? 0 : (int)((uint32_t)K >> a.ibits);
                    const int64_t c = (int64_t)b * a.LH + cl;
                    atomicAdd(head_kept_of(a, cx) + c, 1u);
                    // its keep bit (several candidates may share a mask word)
                    const int slot = __ldcg(a.cslot + (size_t)b * WIN_CAP + j);
                    const uintptr_t addr = reinterpret_cast<uintptr_t>(a.keep_mask + c * a.max_pages + slot / PAGE);
                    atomicOr(reinterpret_cast<unsigned int *>(addr & ~(uintptr_t)3),
                             (1u << (slot % PAGE)) << ((addr & 2) ? 16 : 0));
                }
                if (less == r - 1) {
                    const uint64_t kap = K + 1ull;
                    a.kappa[b] = kap;
                    window_next(a.win + (size_t)b * 4, kap, 1, (uint32_t)nb);
                }
            }
        }
        __syncthreads();
    }
    if (blockIdx.x == 0 && tid < a.B && (sm.fl()[tid] & SF_TRIVIAL)) a.kappa[tid] = sm.kap()[tid];
    return RES_MODE_GRID;
}

// After a grid-mode resolve: the candidates of this CTA's own tail heads,
// read from the sequences those heads belong to (see OWN_CAP).
__device__ void own_list_grid(const StepArgs &a, const Sm &sm) {
    const int tid = threadIdx.x, nct = gridDim.x;
    const int hc0 = (int)((int64_t)blockIdx.x * a.C / nct), hc1 = (int)((int64_t)(blockIdx.x + 1) * a.C / nct);
    if (tid == 0) sm.misc()[MS_NOWN] = 0;
    __syncthreads();
    if (hc0 < hc1) {
        const int b0 = hc0 / a.LH, b1 = (hc1 - 1) / a.LH;
        const int g0 = (int)sm.off()[b0], g1 = (int)(sm.off()[b1] + sm.nc()[b1]);
        for (int g = g0 + tid; g < g1; g += NTH) {
            int b = b0;
            while (b < b1 && (int)sm.off()[b + 1] <= g) b++;
            const int j = g - (int)sm.off()[b];
            const uint64_t K = __ldcg(a.ckey + (size_t)b * WIN_CAP + j);
            const int c = b * a.LH + (a.ibits >= 32 ? 0 : (int)((uint32_t)K >> a.ibits));
            if (c >= hc0 && c < hc1) {
                const int at = atomicAdd(&sm.misc()[MS_NOWN], 1);
                if (at < OWN_CAP) sm.own()[at] = ((c - hc0) << 16) | j;
            }
        }
    }
    __syncthreads();
}

// --------------------------------------------------------- exact select ----
// Calls f(c, pidx, n, key) for every page of this CTA's range, one page per
// thread per round (lanes of a warp hold consecutive pages).  c = head (-1 for
// a thread without a page), pidx = page index in the head, n = valid slots of
// the page, khi(r, hi) = the hi word of slot r's entry key (r < n; false,
// with the status flagged, for an entry rejected as bad input) and klo(r) =
// its lo word (valid only where khi returned true).  Every thread calls f, so f
// may use warp collectives.  Loads are pipelined across rounds: a round's 16
// positions and 16 log-retentions per page (16-byte vectors) are in flight
// together with the next round's head lengths and block-table entries.  The
// head of a page comes from a binary search in a chunk of the range's page
// prefix (a.pfx) staged in shared memory, reloaded when a round leaves it.
__device__ __forceinline__ void range_page_head(const StepArgs &a, const Ctx &cx, const int32_t *spfx, int hcur,
                                                int32_t x, int &c, int &pidx) {
    c = -1;
    pidx = 0;
    if (x >= cx.x1) return;
    int32_t base;
    if (spfx[KT] > x) {
        int lo = 0, hi = KT - 1;  // last j with spfx[j] <= x
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (spfx[mid] <= x) lo = mid; else hi = mid - 1;
        }
        c = hcur + lo;
        base = spfx[lo];
    } else {
        // more heads start here than the chunk holds (empty heads): search
        // the prefix in global memory
        int lo = hcur + KT, hi = cx.c_last;
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (__ldcg(a.pfx + mid) <= x) lo = mid; else hi = mid - 1;
        }
        c = lo;
        base = __ldcg(a.pfx + c);
    }
    pidx = x - base;
}

template <typename F>
__device__ __forceinline__ void for_range_pages(const StepArgs &a, const Sm &sm, const Ctx &cx, F &&f) {
    const int tid = threadIdx.x;
    int32_t *spfx = reinterpret_cast<int32_t *>(sm.big() + T_SPFX);
    int *hnext = &sm.misc()[MS_HNEXT];
    int hcur = cx.c_start;
    auto load_chunk = [&]() {
        for (int j = tid; j <= KT; j += NTH) {
            const int c = hcur + j;
            spfx[j] = c <= cx.c_last + 1 ? __ldcg(a.pfx + c) : 0x7FFFFFFF;
        }
        __syncthreads();
    };
    load_chunk();
    int c, pidx;
    range_page_head(a, cx, spfx, hcur, cx.x0 + tid, c, pidx);
    int32_t ln = 0, pg = 0;
    if (c >= 0) {
        ln = __ldcg(a.len + c);
        pg = __ldcg(a.block_table + (int64_t)c * a.max_pages + pidx);
    }
    for (int32_t X0 = cx.x0; X0 < cx.x1; X0 += KT) {
        // this round's positions and log-retentions
        const int n = c >= 0 ? min(PAGE, max(0, clamp_len(ln, a.max_pages, nullptr) - pidx * PAGE)) : 0;
        int4 pv[4];
        float4 lv[4];
        {
            const int4 *pp = reinterpret_cast<const int4 *>(a.pos_pool + (int64_t)pg * PAGE);
            const float4 *lp = reinterpret_cast<const float4 *>(a.lb_pool + (int64_t)pg * PAGE);
#pragma unroll
            for (int q = 0; q < 4; q++) {
                pv[q] = make_int4(0, 0, 0, 0);
                lv[q] = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
                if (4 * q < n) {
                    pv[q] = __ldcg(pp + q);
                    lv[q] = __ldcg(lp + q);
                }
            }
        }
        // the next round's heads and pages (the chunk is reloaded from this
        // round's last head when it does not reach the next round's end)
        const int32_t Xn = X0 + KT;
        int cn = -1, pn = 0;
        int32_t lnn = 0, pgn = 0;
        if (Xn < cx.x1) {
            if (spfx[KT] <= min(Xn + KT, cx.x1) - 1) {
                if (tid == NTH - 1) *hnext = c >= 0 ? c : hcur;
                __syncthreads();
                hcur = *hnext;
                __syncthreads();
                load_chunk();
            }
            range_page_head(a, cx, spfx, hcur, Xn + tid, cn, pn);
            if (cn >= 0) {
                lnn = __ldcg(a.len + cn);
                pgn = __ldcg(a.block_table + (int64_t)cn * a.max_pages + pn);
            }
        }
        {
            const int b = c >= 0 ? c / a.LH : 0;
            const int32_t tb = sm.t()[b];
            const uint32_t cl = (uint32_t)(c - b * a.LH);
            const uint32_t plim = a.ibits < 32 ? (1u << a.ibits) : 0x80000000u;
            const uint32_t clsh = (uint32_t)((uint64_t)cl << a.ibits);
            auto pos_of = [&](int r) -> int32_t {
                const int4 &pq = pv[r >> 2];
                return (r & 3) == 0 ? pq.x : (r & 3) == 1 ? pq.y : (r & 3) == 2 ? pq.z : pq.w;
            };
            auto khi = [&](int r, uint32_t &hi) -> bool {
                const float4 &lq = lv[r >> 2];
                const float ls = (r & 3) == 0 ? lq.x : (r & 3) == 1 ? lq.y : (r & 3) == 2 ? lq.z : lq.w;
                if (entry_key_hi(tb, pos_of(r), ls, plim, &hi)) return true;
                set_status(a.status, RKV_DEV_BAD_INPUT);
                return false;
            };
            auto klo = [&](int r) -> uint32_t { return clsh | (uint32_t)pos_of(r); };
            f(c, pidx, n, khi, klo);
        }
        c = cn;
        pidx = pn;
        ln = lnn;
        pg = pgn;
    }
    __syncthreads();
}

// This call's largest kept key of sequence b (uint64 in the counter half).
__device__ __forceinline__ unsigned long long *kmax_of(const StepArgs &a, const Ctx &cx, int b) {
    return reinterpret_cast<unsigned long long *>(seqc_of(a, cx) + (size_t)b * 4 + 2);
}

// Digit p of every unfinished sequence's threshold from its completed global
// histogram, one warp per sequence (every CTA computes the same result):
// lane l sums bins [64 l, 64 l + 64), a warp scan of the sums finds the lane
// whose bins hold the rank, and that lane reads its bins again to find the bin.
__device__ void scan_digits(const StepArgs &a, const Sm &sm, int p) {
    constexpr int PER = NBINS / 32;
    static_assert(NBINS % 128 == 0, "bins per lane in 16-byte loads");
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    for (int b = warp; b < a.B; b += NWARP) {
        if (sm.fl()[b] & SF_DONE) continue;
        const uint4 *gh = reinterpret_cast<const uint4 *>(a.ghist + ((size_t)p * a.B + b) * NBINS + lane * PER);
        uint32_t loc = 0;
#pragma unroll 4
        for (int j = 0; j < PER / 4; j++) {
            const uint4 q = __ldcg(gh + j);
            loc += q.x + q.y + q.z + q.w;
        }
        uint32_t inc = loc;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t y = __shfl_up_sync(0xFFFFFFFFu, inc, o);
            if (lane >= o) inc += y;
        }
        const uint32_t rank = sm.rank()[b];
        const bool mine = inc - loc < rank && rank <= inc;
        if (__ballot_sync(0xFFFFFFFFu, mine) == 0u) {
            // fewer matching keys than the rank (entries rejected as bad input)
            if (lane == 0) {
                set_status(a.status, RKV_DEV_BAD_INPUT);
                sm.fl()[b] |= SF_DONE;
                sm.kap()[b] = (sm.pk()[b] | ~sm.pm()[b]) + 1ull;
            }
            continue;
        }
        if (mine) {
            uint32_t cum = inc - loc, nr = 0, h = 0;
            int dig = 0;
#pragma unroll 2
            for (int j = 0; j < PER / 4; j++) {
                const uint4 q = __ldcg(gh + j);
                const uint32_t e[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
                for (int u = 0; u < 4; u++) {
                    if (cum < rank && rank <= cum + e[u]) {
                        dig = lane * PER + 4 * j + u;
                        nr = rank - cum;
                        h = e[u];
                    }
                    cum += e[u];
                }
            }
            if (p == 1) sm.h1()[b] = h;
            const int sh = digit_shift(p);
            sm.pk()[b] |= (uint64_t)dig << sh;
            sm.pm()[b] |= ((1ull << digit_bits(p)) - 1ull) << sh;
            sm.rank()[b] = nr;
            if (h == nr || p == NPASS - 1) {
                sm.fl()[b] |= SF_DONE;
                sm.kap()[b] = (sm.pk()[b] | ~sm.pm()[b]) + 1ull;
            }
        }
    }
    __syncthreads();
}

// Exact threshold of every non-trivial sequence by radix passes over this
// CTA's page range, then keep masks and kept counts for every page of it.
__device__ bool exact_select(const StepArgs &a, const Sm &sm, Ctx &cx) {
    const int tid = threadIdx.x, lane = tid & 31;
    {
        // page prefix of the heads this CTA's range visits, for page -> head
        const int CS = (a.C + NTH - 1) / NTH;
        const int h0 = min(a.C, tid * CS), h1 = min(a.C, h0 + CS);
        uint32_t mine = 0, tot;
        for (int c = h0; c < h1; c++)
            mine += (uint32_t)((clamp_len(__ldcg(a.len + c), a.max_pages, nullptr) + PAGE - 1) / PAGE);
        int64_t p = block_exclusive_scan(mine, sm.scan(), &tot);
        for (int c = h0; c < h1; c++) {
            if (c >= cx.c_start && c <= cx.c_last + 1) a.pfx[c] = (int32_t)p;
            p += (clamp_len(__ldcg(a.len + c), a.max_pages, nullptr) + PAGE - 1) / PAGE;
        }
        if (tid == 0 && cx.c_last + 1 == a.C) a.pfx[a.C] = (int32_t)cx.TP;
    }
    cx.exact = true;
    if (tid < a.B && !(sm.fl()[tid] & SF_TRIVIAL)) {
        sm.fl()[tid] &= ~SF_DONE;
        sm.rank()[tid] = (uint32_t)sm.m()[tid];
        sm.pk()[tid] = 0ull;
        sm.pm()[tid] = 0ull;
        sm.h1()[tid] = 0u;
    }
    if (tid < MAXB) sm.kmx()[tid] = 0ull;
    __syncthreads();
    const int b_first = cx.c_start < a.C ? cx.c_start / a.LH : 0;
    const int b_last = cx.c_last >= 0 ? cx.c_last / a.LH : -1;
    uint32_t *hist = reinterpret_cast<uint32_t *>(sm.big());
    // digit p's histogram of the sequences [g0, g1) this sweep counts
    int p = 0, g0 = 0, g1 = 0;
    auto count = [&](int c, int, int n, auto &khi, auto &klo) {
        if (c < 0) return;
        const int b = c / a.LH;
        if (b < g0 || b >= g1 || (sm.fl()[b] & SF_DONE)) return;
        const uint64_t pk = sm.pk()[b], pm = sm.pm()[b];
        const uint32_t pkh = (uint32_t)(pk >> 32), pmh = (uint32_t)(pm >> 32);
        const uint32_t pkl = (uint32_t)pk, pml = (uint32_t)pm;
        // digit p lies in the hi word for p < 3 (the lo word is then not
        // needed: its prefix bits are still unset), else in the lo word
        const bool in_lo = p >= 3;
        const int sh = digit_shift(p) & 31;
        const uint32_t dmask = (1u << digit_bits(p)) - 1u;
        uint32_t *hb = hist + (b - g0) * NBINS;
        // a page's neighbouring entries mostly share a bin: add runs
        uint32_t run_bin = 0u, run_n = 0u;
#pragma unroll
        for (int r = 0; r < PAGE; r++) {
            uint32_t w;
            if (r >= n || !khi(r, w) || ((w ^ pkh) & pmh) != 0u) continue;
            if (in_lo) {
                w = klo(r);
                if (((w ^ pkl) & pml) != 0u) continue;
            }
            const uint32_t bin = (w >> sh) & dmask;
            if (run_n && bin == run_bin) {
                run_n++;
            } else {
                if (run_n) atomicAdd(hb + run_bin, run_n);
                run_bin = bin;
                run_n = 1u;
            }
        }
        if (run_n) atomicAdd(hb + run_bin, run_n);
    };
    for (p = 0; p < NPASS; p++) {
        if (tid == 0) {
            int act = 0;
            for (int b = 0; b < a.B; b++) act |= (sm.fl()[b] & SF_DONE) ? 0 : 1;
            sm.misc()[MS_ACTIVE] = act;
        }
        __syncthreads();
        if (!sm.misc()[MS_ACTIVE]) break;
        cx.passes = p + 1;
        for (g0 = b_first; g0 <= b_last; g0 += HGRP) {
            g1 = min(b_last + 1, g0 + HGRP);
            for (int i = tid; i < (g1 - g0) * NBINS; i += NTH) hist[i] = 0u;
            __syncthreads();
            for_range_pages(a, sm, cx, count);
            __syncthreads();
            for (int i = tid; i < (g1 - g0) * NBINS; i += NTH) {
                const uint32_t v = hist[i];
                const int b = g0 + i / NBINS;
                if (v) atomicAdd(a.ghist + ((size_t)p * a.B + b) * NBINS + (i % NBINS), v);
            }
            __syncthreads();
        }
        if (!grid_barrier(a.bar, ++cx.epoch, a.status, &sm.misc()[MS_BAR])) return false;
        scan_digits(a, sm, p);
    }
    // keep masks, kept counts (summed over each run of lanes holding the same
    // head) and the largest kept key of each sequence (the reported threshold
    // is that key + 1: a radix bucket kept whole only bounds it)
    int kb = -1;
    unsigned long long km = 0ull;
    auto mark = [&](int c, int pidx, int n, auto &khi, auto &klo) {
        uint32_t m16 = 0u;
        if (c >= 0) {
            const int b = c / a.LH;
            const uint64_t kap = sm.kap()[b];
            const uint32_t kaph = (uint32_t)(kap >> 32), kapl = (uint32_t)kap;
            if (b != kb) {
                if (kb >= 0) atomicMax(sm.kmx() + kb, km);
                kb = b;
                km = 0ull;
            }
#pragma unroll
            for (int r = 0; r < PAGE; r++) {
                // K < kap on the two words: the lo word only on a hi tie
                uint32_t hi;
                if (r < n && khi(r, hi) && hi <= kaph) {
                    const uint32_t lo = klo(r);
                    if (hi < kaph || lo < kapl) {
                        m16 |= 1u << r;
                        const uint64_t K = ((uint64_t)hi << 32) | lo;
                        km = K > km ? K : km;
                    }
                }
            }
            a.keep_mask[(int64_t)c * a.max_pages + pidx] = (uint16_t)m16;
        }
        // lanes hold consecutive pages, so a head's lanes are contiguous:
        // suffix sums within runs of equal c, the run's first lane adds
        uint32_t sum = (uint32_t)__popc(m16);
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t y = __shfl_down_sync(0xFFFFFFFFu, sum, o);
            const int cy = __shfl_down_sync(0xFFFFFFFFu, c, o);
            if (lane + o < 32 && cy == c) sum += y;
        }
        const int cprev = __shfl_up_sync(0xFFFFFFFFu, c, 1);
        if (c >= 0 && (lane == 0 || cprev != c) && sum) atomicAdd(head_kept_of(a, cx) + c, sum);
    };
    for_range_pages(a, sm, cx, mark);
    if (kb >= 0 && km) atomicMax(sm.kmx() + kb, km);
    __syncthreads();
    if (tid < a.B && sm.kmx()[tid]) atomicMax(kmax_of(a, cx, tid), sm.kmx()[tid]);
    if (blockIdx.x == 0 && tid < a.B && (sm.fl()[tid] & SF_TRIVIAL)) a.kappa[tid] = sm.kap()[tid];
    __syncthreads();
    return true;
}

// ------------------------------------------------------------------ tail ----
template <class M>
__device__ __forceinline__ float row_elt(const unsigned char *row, int d) {
    if constexpr (M::ROW_BYTES / M::DIM == 2) {
        return __uint_as_float((uint32_t)__ldcg(reinterpret_cast<const unsigned short *>(row) + d) << 16);
    } else {
        return __ldcg(reinterpret_cast<const float *>(row) + d);
    }
}

// Fate (1 = kept) of candidate j of sequence b: from shared memory after a
// local resolve, else from the workspace.
__device__ __forceinline__ int cand_fate(const StepArgs &a, const Sm &sm, bool local, int b, int j) {
    return local ? (int)sm.fate()[sm.off()[b] + j] : __ldcg(a.cfate + (size_t)b * WIN_CAP + j);
}

// Merge of a head's partial states: the records of the CTAs its pages span
// (or the record of the one CTA that held candidates of it) and its
// candidates, each kept (logit z, weight 1, value v) or evicted (logit z).
template <class M, int D, int G>
__device__ void combine_head(const StepArgs &a, const Sm &sm, const Ctx &cx, int c, int64_t pfx, int jf, int jl,
                             uint32_t flag, bool cands, bool local) {
    using LY = StepLayout<M, D, G>;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int b = c / a.LH;
    const int cl = c - b * a.LH;
    int32_t *clist = reinterpret_cast<int32_t *>(sm.big() + T_CL);
    int ncl = 0;
    if (cands) {
        if (warp == 0) {
            const int nb = (int)sm.nc()[b];
            int cnt = 0;
            for (int base = 0; base < nb; base += 32) {
                const int i = base + lane;
                bool mine = false;
                if (i < nb) {
                    const uint64_t K = __ldcg(a.ckey + (size_t)b * WIN_CAP + i);
                    mine = (a.ibits >= 32 ? 0 : (int)((uint32_t)K >> a.ibits)) == cl;
                }
                const uint32_t ball = __ballot_sync(0xFFFFFFFFu, mine);
                if (mine) clist[cnt + __popc(ball & ((1u << lane) - 1u))] = i;
                cnt += __popc(ball);
            }
            if (lane == 0) sm.misc()[MS_NCL] = cnt;
        }
        __syncthreads();
        ncl = sm.misc()[MS_NCL];
    }
    const bool split = jf != jl;
    const size_t cb = (size_t)b * WIN_CAP;
    for (int e = tid; e < G * D + G; e += NTH) {
        const bool is_stat = e >= G * D;
        const int g = is_stat ? e - G * D : e / D;
        Merged s;
        s.mk = -INFINITY;
        s.me = -INFINITY;
        if (split) {
            for (int j = jf; j <= jl; j++) {
                if (!(sm.rlo()[j] < sm.rlo()[j + 1])) continue;
                const float *r = a.partial + ((int64_t)j * 2 + ((pfx < sm.rlo()[j]) ? 0 : 1)) * LY::REC;
                s.mk = fmaxf(s.mk, __ldcg(r + G * D + g));
                s.me = fmaxf(s.me, __ldcg(r + G * D + 2 * G + g));
            }
        } else if (flag & 2u) {
            const float *r = a.hrec + (int64_t)c * LY::REC;
            s.mk = fmaxf(s.mk, __ldcg(r + G * D + g));
            s.me = fmaxf(s.me, __ldcg(r + G * D + 2 * G + g));
        }
        for (int i = 0; i < ncl; i++) {
            const size_t idx = cb + clist[i];
            const float z = __ldcg(a.cz + idx * G + g);
            if (cand_fate(a, sm, local, b, clist[i])) s.mk = fmaxf(s.mk, z); else s.me = fmaxf(s.me, z);
        }
        s.lk = 0.0f;
        s.le = 0.0f;
        float av = 0.0f;
        auto add = [&](const float *r) {
            const float mkw = __ldcg(r + G * D + g), mew = __ldcg(r + G * D + 2 * G + g);
            const float fk = (mkw == -INFINITY) ? 0.0f : ex2(mkw - s.mk);
            const float fe = (mew == -INFINITY) ? 0.0f : ex2(mew - s.me);
            s.lk += __ldcg(r + G * D + G + g) * fk;
            s.le += __ldcg(r + G * D + 3 * G + g) * fe;
            if (!is_stat) av += __ldcg(r + e) * fk;
        };
        if (split) {
            for (int j = jf; j <= jl; j++) {
                if (!(sm.rlo()[j] < sm.rlo()[j + 1])) continue;
                add(a.partial + ((int64_t)j * 2 + ((pfx < sm.rlo()[j]) ? 0 : 1)) * LY::REC);
            }
        } else if (flag & 2u) {
            add(a.hrec + (int64_t)c * LY::REC);
        }
        for (int i = 0; i < ncl; i++) {
            const size_t idx = cb + clist[i];
            const float z = __ldcg(a.cz + idx * G + g);
            if (cand_fate(a, sm, local, b, clist[i])) {
                const float w = ex2(z - s.mk);
                s.lk += w;
                if (!is_stat) av += w * row_elt<M>(a.cv + idx * a.row_bytes, e - g * D);
            } else {
                s.le += ex2(z - s.me);
            }
        }
        if (!is_stat) {
            a.out[(int64_t)c * G * D + e] = s.lk > 0.0f ? av / s.lk : 0.0f;
        } else {
            if (a.lse) a.lse[(int64_t)c * G + g] = s.lk > 0.0f ? (s.mk + __log2f(s.lk)) * LN2 : -INFINITY;
            if (a.dropped) a.dropped[(int64_t)c * G + g] = dm_of(s);
        }
    }
    __syncthreads();
}

// Warp-level merge of head c (same sources and result as combine_head):
// lanes load every record's per-row statistics and every candidate's logits
// in one round, lanes 0..G-1 merge them per query row, then every lane
// accumulates EPL output elements with the records' loads issued together.
// Returns false (nothing written) when the head has more than RCAP records
// or CCAP candidates; the block-wide merge handles it then.
// VW consecutive floats from p (one 16-byte load when VW is 4), zeros when !ok.
template <int VW>
__device__ __forceinline__ void load_group(float (&v)[VW], const float *p, bool ok) {
    if constexpr (VW == 4) {
        const float4 x = ok ? __ldcg(reinterpret_cast<const float4 *>(p)) : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
        v[0] = x.x;
        v[1] = x.y;
        v[2] = x.z;
        v[3] = x.w;
    } else {
#pragma unroll
        for (int q = 0; q < VW; q++) v[q] = ok ? __ldcg(p + q) : 0.0f;
    }
}
template <int VW>
__device__ __forceinline__ void store_group(float *p, const float (&v)[VW]) {
    if constexpr (VW == 4) {
        *reinterpret_cast<float4 *>(p) = make_float4(v[0], v[1], v[2], v[3]);
    } else {
#pragma unroll
        for (int q = 0; q < VW; q++) p[q] = v[q];
    }
}
// Elements d .. d + VW - 1 of a V row in the pool dtype, as floats.
template <class M, int VW>
__device__ __forceinline__ void row_group(float (&r)[VW], const unsigned char *row, int d) {
    if constexpr (VW == 4 && M::ROW_BYTES / M::DIM == 2) {
        const uint2 x = __ldcg(reinterpret_cast<const uint2 *>(row) + d / 4);
        r[0] = __uint_as_float(x.x << 16);
        r[1] = __uint_as_float(x.x & 0xFFFF0000u);
        r[2] = __uint_as_float(x.y << 16);
        r[3] = __uint_as_float(x.y & 0xFFFF0000u);
    } else if constexpr (VW == 4) {
        const float4 x = __ldcg(reinterpret_cast<const float4 *>(row) + d / 4);
        r[0] = x.x;
        r[1] = x.y;
        r[2] = x.z;
        r[3] = x.w;
    } else {
#pragma unroll
        for (int q = 0; q < VW; q++) r[q] = row_elt<M>(row, d + q);
    }
}

template <class M, int D, int G>
__device__ bool combine_warp(const StepArgs &a, const Sm &sm, const Ctx &cx, WarpScr &w, int c, int64_t pfx,
                             int jf, int jl, uint32_t flag, bool cands, bool local) {
    using LY = StepLayout<M, D, G>;
    constexpr int GD = G * D;
    constexpr int VW = GD % 128 == 0 ? 4 : 1;
    constexpr int NU = (GD + 32 * VW - 1) / (32 * VW);
    const int lane = threadIdx.x & 31;
    const int b = c / a.LH;
    const int cl = c - b * a.LH;
    // ---- sources ----
    int nrec = 0;
    if (lane == 0) {
        if (jf != jl) {
            for (int j = jf; j <= jl; j++) {
                const int64_t lo = sm.rlo()[j];
                if (!(lo < sm.rlo()[j + 1])) continue;
                if (nrec < RCAP) w.recp[nrec] = a.partial + ((int64_t)j * 2 + ((pfx < lo) ? 0 : 1)) * LY::REC;
                nrec++;
            }
        } else if (flag & 2u) {
            w.recp[0] = a.hrec + (int64_t)c * LY::REC;
            nrec = 1;
        }
    }
    nrec = __shfl_sync(0xFFFFFFFFu, nrec, 0);
    if (nrec > RCAP) return false;
    int ncl = 0;
    const size_t cb = (size_t)b * WIN_CAP;
    if (cands) {
        const int nown = sm.misc()[MS_NOWN];
        if (nown <= OWN_CAP) {
            // this CTA's list of its own heads' candidates (shared memory)
            const int kk = c - (int)((int64_t)blockIdx.x * a.C / gridDim.x);
            for (int base = 0; base < nown; base += 32) {
                const int i = base + lane;
                const int32_t e = i < nown ? sm.own()[i] : -1;
                const bool mine = i < nown && (e >> 16) == kk;
                const uint32_t ball = __ballot_sync(0xFFFFFFFFu, mine);
                const int k = ncl + __popc(ball & ((1u << lane) - 1u));
                if (mine && k < CCAP) w.cidx[k] = e & 0xFFFF;
                ncl += __popc(ball);
            }
        } else {
            const int nb = (int)sm.nc()[b];
            for (int base = 0; base < nb; base += 32) {
                const int i = base + lane;
                bool mine = false;
                if (i < nb) {
                    const uint64_t K = __ldcg(a.ckey + cb + i);
                    mine = (a.ibits >= 32 ? 0 : (int)((uint32_t)K >> a.ibits)) == cl;
                }
                const uint32_t ball = __ballot_sync(0xFFFFFFFFu, mine);
                const int k = ncl + __popc(ball & ((1u << lane) - 1u));
                if (mine && k < CCAP) w.cidx[k] = i;
                ncl += __popc(ball);
            }
        }
        if (ncl > CCAP) return false;
    }
    __syncwarp();
    // ---- one round of loads: record statistics, candidate logits and fates ----
    for (int t = lane; t < nrec * G; t += 32) {
        const float *r = w.recp[t / G] + GD + (t % G);
        w.st[0][t] = __ldcg(r);
        w.st[1][t] = __ldcg(r + G);
        w.st[2][t] = __ldcg(r + 2 * G);
        w.st[3][t] = __ldcg(r + 3 * G);
    }
    for (int t = lane; t < ncl * G; t += 32) w.cz[t] = __ldcg(a.cz + (cb + w.cidx[t / G]) * G + (t % G));
    for (int i = lane; i < ncl; i += 32) w.cfate[i] = cand_fate(a, sm, local, b, w.cidx[i]);
    // the first two records' output values, in the same round: each lane
    // holds NU groups of VW consecutive elements (e = (lane + 32 u) VW + q;
    // 16-byte loads and stores when the row length allows)
    float v0[NU][VW], v1[NU][VW];
#pragma unroll
    for (int u = 0; u < NU; u++) {
        const int e = (lane + 32 * u) * VW;
        load_group<VW>(v0[u], w.recp[0] + e, nrec > 0 && e < GD);
        load_group<VW>(v1[u], w.recp[1] + e, nrec > 1 && e < GD);
    }
    __syncwarp();
    // ---- per query row: merged maxima, sums, lse and dropped mass ----
    if (lane < G) {
        const int g = lane;
        Merged s;
        s.mk = -INFINITY;
        s.me = -INFINITY;
        for (int k = 0; k < nrec; k++) {
            s.mk = fmaxf(s.mk, w.st[0][k * G + g]);
            s.me = fmaxf(s.me, w.st[2][k * G + g]);
        }
        for (int i = 0; i < ncl; i++) {
            const float z = w.cz[i * G + g];
            if (w.cfate[i]) s.mk = fmaxf(s.mk, z); else s.me = fmaxf(s.me, z);
        }
        s.lk = 0.0f;
        s.le = 0.0f;
        for (int k = 0; k < nrec; k++) {
            const float mkw = w.st[0][k * G + g], mew = w.st[2][k * G + g];
            const float fk = (mkw == -INFINITY) ? 0.0f : ex2(mkw - s.mk);
            const float fe = (mew == -INFINITY) ? 0.0f : ex2(mew - s.me);
            w.fk[k * G + g] = fk;
            s.lk += w.st[1][k * G + g] * fk;
            s.le += w.st[3][k * G + g] * fe;
        }
        for (int i = 0; i < ncl; i++) {
            const float z = w.cz[i * G + g];
            if (w.cfate[i]) {
                const float f = ex2(z - s.mk);
                w.cz[i * G + g] = f;
                s.lk += f;
            } else {
                w.cz[i * G + g] = 0.0f;
                s.le += ex2(z - s.me);
            }
        }
        w.mk[g] = s.mk;
        w.lk[g] = s.lk;
        if (a.lse) a.lse[(int64_t)c * G + g] = s.lk > 0.0f ? (s.mk + __log2f(s.lk)) * LN2 : -INFINITY;
        if (a.dropped) a.dropped[(int64_t)c * G + g] = dm_of(s);
    }
    __syncwarp();
    // ---- outputs: NU groups of VW elements per lane, two records' loads in flight at a time ----
    float av[NU][VW];
#pragma unroll
    for (int u = 0; u < NU; u++) {
        const int e = (lane + 32 * u) * VW;
        const int g = (e < GD ? e : 0) / D;  // (a group never straddles two query rows)
#pragma unroll
        for (int q = 0; q < VW; q++)
            av[u][q] = (nrec > 0 ? v0[u][q] * w.fk[g] : 0.0f) + (nrec > 1 ? v1[u][q] * w.fk[G + g] : 0.0f);
    }
    for (int k = 2; k < nrec; k++) {
#pragma unroll
        for (int u = 0; u < NU; u++) {
            const int e = (lane + 32 * u) * VW;
            load_group<VW>(v0[u], w.recp[k] + e, e < GD);
        }
#pragma unroll
        for (int u = 0; u < NU; u++) {
            const int e = (lane + 32 * u) * VW;
            const float f = w.fk[k * G + (e < GD ? e : 0) / D];
#pragma unroll
            for (int q = 0; q < VW; q++) av[u][q] += v0[u][q] * f;
        }
    }
    for (int i = 0; i < ncl; i++) {
        if (!w.cfate[i]) continue;
        const unsigned char *row = a.cv + (cb + w.cidx[i]) * a.row_bytes;
#pragma unroll
        for (int u = 0; u < NU; u++) {
            const int e = (lane + 32 * u) * VW;
            if (e < GD) {
                float r[VW];
                row_group<M, VW>(r, row, e % D);
                const float f = w.cz[i * G + e / D];
#pragma unroll
                for (int q = 0; q < VW; q++) av[u][q] += f * r[q];
            }
        }
    }
#pragma unroll
    for (int u = 0; u < NU; u++) {
        const int e = (lane + 32 * u) * VW;
        if (e < GD) {
            const float lk = w.lk[e / D];
            float o[VW];
#pragma unroll
            for (int q = 0; q < VW; q++) o[q] = lk > 0.0f ? av[u][q] / lk : 0.0f;
            store_group<VW>(a.out + (int64_t)c * GD + e, o);
        }
    }
    __syncwarp();
    return true;
}

// Hole-fill compaction of head c (n entries, nn kept): the j-th non-kept
// slot below nn takes the j-th kept slot at or above nn.  This call moves the
// ranks [moves * part / parts, moves * (part + 1) / parts), so several CTAs
// can share a head; with push, pages past ceil(nn/16) go to the free stack at
// this head's plan offset (only once every part of the head has moved).
// Pairs are resolved CMP_PAIRS at a time; each warp then moves CPW rows with
// all their loads issued before the stores.
template <int ROWB>
__device__ void compact_head(const StepArgs &a, const Sm &sm, const Ctx &cx, int c, int n, int nn, int32_t off,
                             int part, int parts, bool push) {
    constexpr int E = (2 * ROWB / 16 + 31) / 32;  // 16-byte pieces per lane of a row's K and V
    constexpr int CPW = 8 / E;                    // rows a warp moves at a time
    static_assert(2 * ROWB / 16 <= 64, "row bytes");
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int mp = a.max_pages;
    int32_t *tbl = reinterpret_cast<int32_t *>(sm.big() + T_TBL);
    int32_t *src_pfx = tbl + mp;
    int32_t *hole_pfx = src_pfx + mp + 1;
    uint16_t *msk = reinterpret_cast<uint16_t *>(hole_pfx + mp + 1);
    int2 *pairs = reinterpret_cast<int2 *>(sm.big() + T_PAIRS);
    const int W = (n + PAGE - 1) / PAGE, Wn = (nn + PAGE - 1) / PAGE;
    const int64_t cm = (int64_t)c * mp;
    // table and keep words, LDW per thread per round with their loads issued
    // together; per word its sources (kept slots at or above nn) and holes
    // (non-kept slots below nn)
    constexpr int LDW = 8;
    for (int w0 = 0; w0 < W; w0 += NTH * LDW) {
        int32_t tv[LDW];
        uint32_t mv[LDW];
#pragma unroll
        for (int k = 0; k < LDW; k++) {
            const int w = w0 + k * NTH + tid;
            tv[k] = 0;
            mv[k] = 0u;
            if (w < W) {
                tv[k] = __ldcg(a.block_table + cm + w);
                mv[k] = (uint32_t)__ldcg(a.keep_mask + cm + w);
            }
        }
#pragma unroll
        for (int k = 0; k < LDW; k++) {
            const int w = w0 + k * NTH + tid;
            if (w < W) {
                const uint32_t m = mv[k] & below_bits(w, n);
                tbl[w] = tv[k];
                msk[w] = (uint16_t)m;
                const uint32_t below = below_bits(w, nn);
                src_pfx[w] = __popc(m & ~below);
                hole_pfx[w] = __popc(~m & below & 0xFFFFu);
            }
        }
    }
    __syncthreads();
    scan_words2(src_pfx, hole_pfx, W, sm.scan());
    const int moves = min(hole_pfx[W], src_pfx[W]);
    const int ra = (int)((int64_t)moves * part / parts), rb = (int)((int64_t)moves * (part + 1) / parts);
    constexpr int chunks = ROWB / 16;
    // last word w in [0, W) with pfx[w] <= r (pfx[0] = 0 <= r)
    auto word_of = [&](const int32_t *pfx, int r) {
        int lo = 0, hi = W - 1;
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (pfx[mid] <= r) lo = mid; else hi = mid - 1;
        }
        return lo;
    };
    for (int r0 = ra; r0 < rb; r0 += CMP_PAIRS) {
        const int r1 = min(rb, r0 + CMP_PAIRS);
        // the rank-th hole and the rank-th source for every rank of the
        // round: each thread expands whole words of the words holding them
        {
            const int h0 = word_of(hole_pfx, r0), h1 = word_of(hole_pfx, r1 - 1);
            for (int w = h0 + tid; w <= h1; w += NTH) {
                uint32_t hb = ~(uint32_t)msk[w] & below_bits(w, nn) & 0xFFFFu;
                int rank = hole_pfx[w];
                const int64_t pbase = (int64_t)tbl[w] * PAGE;
                while (hb) {
                    const int bit = __ffs(hb) - 1;
                    hb &= hb - 1;
                    if (rank >= r0 && rank < r1) pairs[rank - r0].x = (int)(pbase + bit);
                    rank++;
                }
            }
            const int s0 = word_of(src_pfx, r0), s1 = word_of(src_pfx, r1 - 1);
            for (int w = s0 + tid; w <= s1; w += NTH) {
                uint32_t sb = (uint32_t)msk[w] & ~below_bits(w, nn);
                int rank = src_pfx[w];
                const int64_t pbase = (int64_t)tbl[w] * PAGE;
                while (sb) {
                    const int bit = __ffs(sb) - 1;
                    sb &= sb - 1;
                    if (rank >= r0 && rank < r1) pairs[rank - r0].y = (int)(pbase + bit);
                    rank++;
                }
            }
        }
        __syncthreads();
        const int np_ = r1 - r0;
        for (int p0 = warp * CPW; p0 < np_; p0 += NWARP * CPW) {
            uint4 v[CPW][E];
            int32_t pos = 0;
            float lbv = 0.0f;
#pragma unroll
            for (int j = 0; j < CPW; j++) {
#pragma unroll
                for (int e = 0; e < E; e++) v[j][e] = make_uint4(0, 0, 0, 0);
                if (p0 + j < np_) {
                    const int64_t src = pairs[p0 + j].y;
                    const uint4 *ks = reinterpret_cast<const uint4 *>((const unsigned char *)a.k_pool + src * ROWB);
                    const uint4 *vs = reinterpret_cast<const uint4 *>((const unsigned char *)a.v_pool + src * ROWB);
#pragma unroll
                    for (int e = 0; e < E; e++) {
                        const int i = lane + 32 * e;
                        if (i < 2 * chunks) v[j][e] = i < chunks ? __ldcg(ks + i) : __ldcg(vs + i - chunks);
                    }
                }
            }
            if (lane < CPW && p0 + lane < np_) {
                const int64_t src = pairs[p0 + lane].y;
                pos = __ldcg(a.pos_pool + src);
                lbv = __ldcg(a.lb_pool + src);
            }
#pragma unroll
            for (int j = 0; j < CPW; j++) {
                if (p0 + j < np_) {
                    const int64_t dst = pairs[p0 + j].x;
                    uint4 *kd = reinterpret_cast<uint4 *>((unsigned char *)a.k_pool + dst * ROWB);
                    uint4 *vd = reinterpret_cast<uint4 *>((unsigned char *)a.v_pool + dst * ROWB);
#pragma unroll
                    for (int e = 0; e < E; e++) {
                        const int i = lane + 32 * e;
                        if (i < 2 * chunks) {
                            if (i < chunks) kd[i] = v[j][e]; else vd[i - chunks] = v[j][e];
                        }
                    }
                }
            }
            if (lane < CPW && p0 + lane < np_) {
                const int64_t dst = pairs[p0 + lane].x;
                a.pos_pool[dst] = pos;
                a.lb_pool[dst] = lbv;
            }
        }
        __syncthreads();
    }
    if (push) {
        for (int pi = Wn + tid; pi < W; pi += NTH) {
            a.free_stack[cx.top0 + off + (pi - Wn)] = tbl[pi];
            a.block_table[cm + pi] = -1;
        }
    }
    __syncthreads();
}

// Warp-level hole-fill compaction of head c (same result as compact_head)
// for heads with at most HCAP evicted entries; returns false otherwise and
// the block-wide compaction runs.  Keep words and block-table entries are
// read WPL per lane per round (all loads issued together); holes (non-kept
// slots below nn) and sources (kept slots at or above nn) are listed in
// ascending order with warp scans, already as physical rows, and freed pages
// are pushed from the same registers; rows then move four pairs at a time
// with every load issued before the stores.
__device__ bool compact_warp(const StepArgs &a, const Ctx &cx, WarpScr &w, int c, int n, int nn, int32_t off) {
    if (n - nn > HCAP) return false;
    constexpr int WPL = 8;
    const int lane = threadIdx.x & 31;
    const int64_t cm = (int64_t)c * a.max_pages;
    const int W = (n + PAGE - 1) / PAGE, Wn = (nn + PAGE - 1) / PAGE;
    int nh = 0, ns = 0;
    for (int w0 = 0; w0 < W; w0 += 32 * WPL) {
        uint32_t m[WPL];
        int32_t pg[WPL];
#pragma unroll
        for (int u = 0; u < WPL; u++) {
            const int wd = w0 + 32 * u + lane;
            m[u] = wd < W ? ((uint32_t)__ldcg(a.keep_mask + cm + wd) & below_bits(wd, n)) : 0u;
            pg[u] = wd < W ? __ldcg(a.block_table + cm + wd) : 0;
        }
#pragma unroll
        for (int u = 0; u < WPL; u++) {
            if (w0 + 32 * u >= W) break;
            const int wd = w0 + 32 * u + lane;
            const uint32_t below = below_bits(wd, nn);
            uint32_t hb = ~m[u] & below & 0xFFFFu, sb = m[u] & ~below;
            const int hc = __popc(hb), sc = __popc(sb);
            int hx = hc, sx = sc;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(0xFFFFFFFFu, hx, o), z = __shfl_up_sync(0xFFFFFFFFu, sx, o);
                if (lane >= o) {
                    hx += y;
                    sx += z;
                }
            }
            const int htot = __shfl_sync(0xFFFFFFFFu, hx, 31), stot = __shfl_sync(0xFFFFFFFFu, sx, 31);
            hx = nh + hx - hc;
            sx = ns + sx - sc;
            while (hb) {
                const int bit = __ffs(hb) - 1;
                hb &= hb - 1;
                if (hx < HCAP) w.holes[hx] = pg[u] * PAGE + bit;
                hx++;
            }
            while (sb) {
                const int bit = __ffs(sb) - 1;
                sb &= sb - 1;
                if (sx < HCAP) w.srcs[sx] = pg[u] * PAGE + bit;
                sx++;
            }
            // pages past ceil(nn/16): pushed at this head's offset in the stack
            // (the moves below use the rows listed above, not the table)
            if (wd >= Wn && wd < W) {
                a.free_stack[cx.top0 + off + (wd - Wn)] = pg[u];
                a.block_table[cm + wd] = -1;
            }
            nh += htot;
            ns += stot;
        }
    }
    __syncwarp();
    const int moves = min(min(nh, ns), HCAP);
    const int chunks = a.row_bytes / 16;
    for (int p0 = 0; p0 < moves; p0 += 4) {
        uint4 v[4][2];
        int32_t pos = 0;
        float lbv = 0.0f;
#pragma unroll
        for (int q = 0; q < 4; q++) {
            const int p = p0 + q;
            const int64_t src = p < moves ? w.srcs[p] : 0;
#pragma unroll
            for (int h = 0; h < 2; h++) {
                const int i = lane + 32 * h;
                v[q][h] = make_uint4(0, 0, 0, 0);
                if (p < moves && i < 2 * chunks) {
                    const uint4 *base = reinterpret_cast<const uint4 *>(
                        (const unsigned char *)(i < chunks ? a.k_pool : a.v_pool) + src * a.row_bytes);
                    v[q][h] = __ldcg(base + (i < chunks ? i : i - chunks));
                }
            }
            if (lane == q && p < moves) {
                pos = __ldcg(a.pos_pool + src);
                lbv = __ldcg(a.lb_pool + src);
            }
        }
#pragma unroll
        for (int q = 0; q < 4; q++) {
            const int p = p0 + q;
            if (p >= moves) break;
            const int64_t dst = w.holes[p];
#pragma unroll
            for (int h = 0; h < 2; h++) {
                const int i = lane + 32 * h;
                if (i < 2 * chunks) {
                    uint4 *base = reinterpret_cast<uint4 *>((unsigned char *)(i < chunks ? a.k_pool : a.v_pool) +
                                                            dst * a.row_bytes);
                    base[i < chunks ? i : i - chunks] = v[q][h];
                }
            }
            if (lane == q) {
                a.pos_pool[dst] = pos;
                a.lb_pool[dst] = lbv;
            }
        }
    }
    __syncwarp();
    return true;
}

// Bounded wait until every CTA has finished its compactions (pushes).
__device__ bool wait_pushes(const StepArgs &a, const Ctx &cx) {
    const uint32_t target = gridDim.x;
    if (ld_acquire_gpu(arrive_of(a, cx)) >= target) return true;
    const uint64_t t0 = globaltimer_ns(), lim = cross_wait_limit_ns(a.status);
    const uint32_t every = lim < 100000ull ? 0u : 255u;
    uint32_t spins = 0;
    while (ld_acquire_gpu(arrive_of(a, cx)) < target) {
        if ((++spins & every) == 0 && globaltimer_ns() - t0 > lim) {
            record_timeout(a.status, 0x200);
            return false;
        }
    }
    return true;
}

// Append of the new token to head c (one warp): slot k (the post-compaction
// length) takes K, V, position t and log-retention; a page is popped when k
// is a multiple of 16 (the pop-th pop of this call, ascending head order).
// A head whose table is full takes no pop rank (the tail's scan counts pops
// of heads with k < max_pages*16 only); a head that cannot append (full
// table, empty stack, a timed-out wait) is skipped with its length unchanged.
__device__ void append_head(const StepArgs &a, const Sm &sm, const Ctx &cx, int c, int k, int pop, uint32_t pushes) {
    const int lane = threadIdx.x & 31;
    const int chunks = a.row_bytes / 16;
    const int i0 = lane, i1 = lane + 32;
    uint4 v0 = make_uint4(0, 0, 0, 0), v1 = v0;
    const uint4 *kn = reinterpret_cast<const uint4 *>((const unsigned char *)a.k_new + (int64_t)c * a.row_bytes);
    const uint4 *vn = reinterpret_cast<const uint4 *>((const unsigned char *)a.v_new + (int64_t)c * a.row_bytes);
    if (i0 < 2 * chunks) v0 = i0 < chunks ? __ldg(kn + i0) : __ldg(vn + i0 - chunks);
    if (i1 < 2 * chunks) v1 = i1 < chunks ? __ldg(kn + i1) : __ldg(vn + i1 - chunks);
    int64_t row = -1;
    if (lane == 0) {
        const int pidx = k / PAGE;
        if (pidx >= a.max_pages) {
            set_status(a.status, RKV_DEV_TABLE_OVERFLOW);
        } else if (k % PAGE == 0) {
            const int idx = cx.top0 + (int)pushes - 1 - pop;
            if (idx < 0) {
                set_status(a.status, RKV_DEV_POOL_EXHAUSTED);
            } else if (idx < cx.top0 || wait_pushes(a, cx)) {
                const int32_t page = __ldcg(a.free_stack + idx);
                a.block_table[(int64_t)c * a.max_pages + pidx] = page;
                row = (int64_t)page * PAGE;
            }
        } else {
            row = (int64_t)__ldcg(a.block_table + (int64_t)c * a.max_pages + pidx) * PAGE + (k % PAGE);
        }
        if (row >= 0) {
            a.pos_pool[row] = sm.t()[c / a.LH];
            a.lb_pool[row] = __ldg(a.lb_new + c);
            a.len[c] = k + 1;  // a skipped head keeps its length
        }
    }
    row = __shfl_sync(0xFFFFFFFFu, row, 0);
    if (row >= 0) {
        uint4 *kd = reinterpret_cast<uint4 *>((unsigned char *)a.k_pool + row * a.row_bytes);
        uint4 *vd = reinterpret_cast<uint4 *>((unsigned char *)a.v_pool + row * a.row_bytes);
        if (i0 < 2 * chunks) {
            if (i0 < chunks) kd[i0] = v0; else vd[i0 - chunks] = v0;
        }
        if (i1 < 2 * chunks) {
            if (i1 < chunks) kd[i1] = v1; else vd[i1 - chunks] = v1;
        }
    }
}

template <class M, int D, int G>
__device__ bool tail(const StepArgs &a, const Sm &sm, Ctx &cx, bool spec, bool local) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nct = gridDim.x;
    const int C = a.C;
    const int hc0 = (int)((int64_t)blockIdx.x * C / nct), hc1 = (int)((int64_t)(blockIdx.x + 1) * C / nct);
    int32_t *st_npre = reinterpret_cast<int32_t *>(sm.big() + T_STASH);
    int32_t *st_nnew = st_npre + NTH, *st_pfx = st_nnew + NTH, *st_plan = st_pfx + NTH, *st_pop = st_plan + NTH;
    // exact-select histograms are no longer read by anyone: clear them
    if (cx.passes > 0) {
        const size_t nh = (size_t)cx.passes * a.B * NBINS;
        for (size_t i = (size_t)blockIdx.x * NTH + tid; i < nh; i += (size_t)nct * NTH) a.ghist[i] = 0u;
    }
    // per head: pre-step pages, freed pages, pops -- prefixes over all heads.
    // The same pass queues this CTA's tail tasks: merges (heads split across
    // CTAs or holding candidates) and compactions are independent tasks (kept
    // candidates' keep bits were set by the resolve step) that warps take from
    // a queue in shared memory; heads too large for a warp are done
    // block-wide afterwards, one at a time.
    int32_t *st_heavy = st_pop + NTH;
    int32_t *tasks = reinterpret_cast<int32_t *>(sm.big() + T_CL);  // [2 * NTH]
    if (tid == 0) {
        sm.misc()[MS_QN] = 0;  // ordered before the queue's atomics by the scan's barriers
        sm.misc()[MS_QH] = 0;
    }
    uint32_t carry[3] = {0u, 0u, 0u}, total[3] = {0u, 0u, 0u};
    int base0 = 0;
    if (C > NTH) {
        // many heads: each thread sums a contiguous chunk (its loads in flight
        // together), one block scan gives the prefixes at this CTA's first
        // head and the totals; the scan below then covers this CTA's heads only
        const int CS = (C + NTH - 1) / NTH;
        const int c0 = min(C, tid * CS), c1 = min(C, c0 + CS);
        uint32_t sum[3] = {0u, 0u, 0u}, pre[3] = {0u, 0u, 0u};
#pragma unroll 4
        for (int c = c0; c < c1; c++) {
            const int32_t np = __ldcg(a.npre + c);
            int32_t nn = cx.evict ? (int32_t)__ldcg(head_kept_of(a, cx) + c) : np;
            if (local) nn += (int32_t)reinterpret_cast<const uint32_t *>(sm.big() + T_WARP + RES_CAP * 8)[c];
            const uint32_t pg = (uint32_t)((np + PAGE - 1) / PAGE);
            const uint32_t v[3] = {pg, cx.evict ? pg - (uint32_t)((nn + PAGE - 1) / PAGE) : 0u,
                                   (nn % PAGE == 0 && nn / PAGE < a.max_pages) ? 1u : 0u};
#pragma unroll
            for (int q = 0; q < 3; q++) {
                sum[q] += v[q];
                if (c < hc0) pre[q] += v[q];
            }
        }
        uint32_t ex[3];
        block_scan_n<3>(sum, ex, total, sm.scan());
        uint32_t *at_hc0 = sm.scan() + 3 * 36;
        if (c0 <= hc0 && hc0 < c1) {
#pragma unroll
            for (int q = 0; q < 3; q++) at_hc0[q] = ex[q] + pre[q];
        }
        __syncthreads();
        if (hc0 < C) {
#pragma unroll
            for (int q = 0; q < 3; q++) carry[q] = at_hc0[q];
        }
        base0 = hc0;
    }
    for (int base = base0; base < (C > NTH ? hc1 : C); base += NTH) {
        const int c = base + tid;
        const bool mine = c >= hc0 && c < hc1;
        int32_t np = 0, nn = 0;
        uint32_t flag = 0u;
        uint32_t v[3] = {0u, 0u, 0u};
        if (c < (C > NTH ? hc1 : C)) {
            np = __ldcg(a.npre + c);
            nn = cx.evict ? (int32_t)__ldcg(head_kept_of(a, cx) + c) : np;
            if (mine) flag = __ldcg(head_flag_of(a, cx) + c);
            if (local) nn += (int32_t)reinterpret_cast<const uint32_t *>(sm.big() + T_WARP + RES_CAP * 8)[c];
            v[0] = (uint32_t)((np + PAGE - 1) / PAGE);
            v[1] = cx.evict ? v[0] - (uint32_t)((nn + PAGE - 1) / PAGE) : 0u;
            v[2] = (nn % PAGE == 0 && nn / PAGE < a.max_pages) ? 1u : 0u;
        }
        uint32_t ex[3], tot[3];
        block_scan_n<3>(v, ex, tot, sm.scan());
        if (mine) {
            const int k = c - hc0;
            const int64_t pfx = carry[0] + ex[0];
            st_npre[k] = np;
            st_nnew[k] = nn;
            st_pfx[k] = (int32_t)pfx;
            st_plan[k] = (int32_t)(carry[1] + ex[1]);
            st_pop[k] = (int32_t)(carry[2] + ex[2]);
            st_heavy[k] = 0;
            const int pages = (int)v[0];
            const bool merge = pages > 0 && (owner_rlo(sm.rlo(), nct, pfx) != owner_rlo(sm.rlo(), nct, pfx + pages - 1) ||
                                             (flag & 2u) || (spec && (flag & 1u)));
            if (merge) tasks[atomicAdd(&sm.misc()[MS_QN], 1)] = (k << 2) | 1;
            if (cx.evict && nn < np) tasks[atomicAdd(&sm.misc()[MS_QN], 1)] = (k << 2) | 2;
        }
#pragma unroll
        for (int s = 0; s < 3; s++) carry[s] += tot[s];
    }
    const uint32_t pushes = C > NTH ? total[1] : carry[1], pops = C > NTH ? total[2] : carry[2];
    __syncthreads();
    if (cx.evict) {
        for (int k = tid; k < hc1 - hc0; k += NTH) {
            a.kept[hc0 + k] = st_nnew[k];
            a.plan[hc0 + k] = st_plan[k];
        }
    }
    if (cx.exact && blockIdx.x == 0 && tid < a.B && !(sm.fl()[tid] & SF_TRIVIAL)) {
        // thresholds of the exact selection: largest kept key + 1 (every CTA's
        // final pass is complete), and the window for the next call
        const uint64_t kap = __ldcg(kmax_of(a, cx, tid)) + 1ull;
        a.kappa[tid] = kap;
        window_next(a.win + (size_t)tid * 4, kap, (int)sm.wres()[tid], sm.nc()[tid], sm.h1()[tid]);
    }
    if (blockIdx.x == nct - 1 && tid == 0) {
        if (cx.evict) {
            a.plan[C] = (int32_t)pushes;
            a.plan[C + 1] = cx.top0;
        }
        const int nt = cx.top0 + (int)pushes - (int)pops;
        *a.free_top = nt < 0 ? 0 : nt;
    }
    WarpScr &wsc = *reinterpret_cast<WarpScr *>(sm.big() + T_WARP + warp * WARP_SCR);
    const int ntask = sm.misc()[MS_QN];
    for (;;) {
        int t = 0;
        if (lane == 0) t = atomicAdd(&sm.misc()[MS_QH], 1);
        t = __shfl_sync(0xFFFFFFFFu, t, 0);
        if (t >= ntask) break;
        const int task = tasks[t], k = task >> 2, c = hc0 + k;
        const int np = st_npre[k], nn = st_nnew[k];
        const bool comp = (task & 2) != 0;
        if (task & 1) {
            const int pages = (np + PAGE - 1) / PAGE;
            const int64_t pfx = st_pfx[k];
            const int jf = owner_rlo(sm.rlo(), nct, pfx), jl = owner_rlo(sm.rlo(), nct, pfx + pages - 1);
            const uint32_t flag = __ldcg(head_flag_of(a, cx) + c);
            if (!combine_warp<M, D, G>(a, sm, cx, wsc, c, pfx, jf, jl, flag, spec && (flag & 1u), local) && lane == 0)
                atomicOr(st_heavy + k, 1);
        }
        if (comp && !compact_warp(a, cx, wsc, c, np, nn, st_plan[k]) && lane == 0) atomicOr(st_heavy + k, 2);
    }
    __syncthreads();
    // A large eviction (an exact selection that frees many pages, e.g. the
    // prefill eviction) spreads the moves of the heads too large for a warp
    // over every CTA, parts per head; their owners push the freed pages after
    // a grid barrier.  The decision is the same in every CTA.
    const bool spread = cx.exact && cx.evict && pushes >= (uint32_t)nct * 4u;
    for (int k = 0; k < hc1 - hc0; k++) {
        if (!(st_heavy[k] & 1)) continue;
        const int c = hc0 + k;
        const int pages = (st_npre[k] + PAGE - 1) / PAGE;
        const int64_t pfx = st_pfx[k];
        const int jf = owner_rlo(sm.rlo(), nct, pfx), jl = owner_rlo(sm.rlo(), nct, pfx + pages - 1);
        const uint32_t flag = __ldcg(head_flag_of(a, cx) + c);
        combine_head<M, D, G>(a, sm, cx, c, pfx, jf, jl, flag, spec && (flag & 1u), local);
    }
    // heavy compactions: this CTA's own heads, or (spread) its share of every
    // head's parts (about two per CTA: each part costs a few microseconds of
    // loads and scans before its copies, and fewer parts balance worse)
    const int parts = spread ? min(64, max(1, (2 * nct + C - 1) / C)) : 1;
    const int njobs = spread ? (int)(((int64_t)C * parts - blockIdx.x + nct - 1) / nct) : hc1 - hc0;
    for (int j = 0; j < njobs; j++) {
        int c, part = 0, np, nn;
        int32_t off = 0;
        if (spread) {
            const int64_t id = blockIdx.x + (int64_t)j * nct;
            c = (int)(id / parts);
            part = (int)(id % parts);
            np = __ldcg(a.npre + c);
            nn = (int)__ldcg(head_kept_of(a, cx) + c);
            if (!(nn < np && np - nn > HCAP)) continue;
        } else {
            if (!(st_heavy[j] & 2)) continue;
            c = hc0 + j;
            np = st_npre[j];
            nn = st_nnew[j];
            off = st_plan[j];
            if (!(cx.evict && nn < np)) continue;
        }
        compact_head<M::PAGE_BYTES / PAGE>(a, sm, cx, c, np, nn, off, part, parts, !spread);
    }
    if (spread) {
        if (!grid_barrier(a.bar, ++cx.epoch, a.status, &sm.misc()[MS_BAR])) return false;
        for (int k = 0; k < hc1 - hc0; k++) {
            if (!(st_heavy[k] & 2)) continue;
            const int64_t cm = (int64_t)(hc0 + k) * a.max_pages;
            const int W = (st_npre[k] + PAGE - 1) / PAGE, Wn = (st_nnew[k] + PAGE - 1) / PAGE;
            for (int pi = Wn + tid; pi < W; pi += NTH) {
                a.free_stack[cx.top0 + st_plan[k] + (pi - Wn)] = __ldcg(a.block_table + cm + pi);
                a.block_table[cm + pi] = -1;
            }
        }
    }
    __syncthreads();
    if (tid == 0) {
        __threadfence();
        atomicAdd(arrive_of(a, cx), 1u);
    }
    for (int k = warp; k < hc1 - hc0; k += NWARP) append_head(a, sm, cx, hc0 + k, st_nnew[k], st_pop[k], pushes);
    return true;
}

// ---------------------------------------------------------------- kernel ----
template <class M, int D, int G>
__global__ void __launch_bounds__(NTH, 1)
    step_kernel(StepArgs a, const __grid_constant__ CUtensorMap tmk, const __grid_constant__ CUtensorMap tmv) {
    using LY = StepLayout<M, D, G>;
    extern __shared__ __align__(128) unsigned char smem_raw[];
    unsigned char *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    Sm sm;
    sm.base = smem;

    Ctx cx;
    prologue<M, D, G>(a, sm, cx, &tmk, &tmv);
    bool spec = false, local = false;
    if (cx.evict && !sm.misc()[MS_RADIX]) {
        if (head_per_warp(cx)) attn_pass_hpw<M, D, G, true>(a, sm, cx, &tmk, &tmv);
        else attn_pass<M, D, G, true>(a, sm, cx, &tmk, &tmv);
        if (!grid_barrier(a.bar, ++cx.epoch, a.status, &sm.misc()[MS_BAR])) return;
        const int res = resolve(a, sm, cx);
        if (res != RES_MISS) {
            if (res == RES_MODE_GRID) {
                if (!grid_barrier(a.bar, ++cx.epoch, a.status, &sm.misc()[MS_BAR])) return;
                own_list_grid(a, sm);
            }
            spec = true;
            local = res == RES_MODE_LOCAL;
            if (blockIdx.x == 0 && threadIdx.x == 0) atomicAdd(a.status + 2, 1);
        } else {
            // a window missed: drop the speculative counts, select exactly
            for (size_t i = (size_t)blockIdx.x * NTH + threadIdx.x; i < 2 * (size_t)a.C; i += (size_t)gridDim.x * NTH)
                head_kept_of(a, cx)[i] = 0u;  // head_kept and head_flag are adjacent
        }
    }
    if (!spec) {
        if (cx.evict && blockIdx.x == 0 && threadIdx.x == 0) atomicAdd(a.status + 3, 1);
        if (cx.evict && !exact_select(a, sm, cx)) return;
        if (head_per_warp(cx)) attn_pass_hpw<M, D, G, false>(a, sm, cx, &tmk, &tmv);
        else attn_pass<M, D, G, false>(a, sm, cx, &tmk, &tmv);
        if (!grid_barrier(a.bar, ++cx.epoch, a.status, &sm.misc()[MS_BAR])) return;
    }
    if (!tail<M, D, G>(a, sm, cx, spec, local)) return;
    // exit ticket: the last CTA resets the barrier counter and flips the half
    // of the per-call counters the next call uses
    __syncthreads();
    if (threadIdx.x == 0) {
        __threadfence();
        if (atomicAdd(a.leave, 1u) == gridDim.x - 1) {
            *a.bar = 0u;
            *a.leave = 0u;
            *a.parity = cx.par ^ 1u;
            __threadfence();
        }
    }
}

template <class M, int D, int G>
cudaError_t launch_one(const StepArgs &a, int grid, cudaStream_t s, const CUtensorMap &tk, const CUtensorMap &tv) {
    using LY = StepLayout<M, D, G>;
    auto *k = step_kernel<M, D, G>;
    const size_t smem = LY::smem(a.max_pages);
    if (smem > 227 * 1024) return cudaErrorNotSupported;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(NTH);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, k, a, tk, tv);
}

template <int DT, int D, int G>
struct Pick;
template <int D, int G>
struct Pick<RKV_BF16, D, G> {
    using M = MmaMath<D, G, true>;
};
template <int D, int G>
struct Pick<RKV_F32, D, G> {
    using M = CoreMath<float, D, G, true>;
};

#define RKV_STEP_CASES(X)                                                                                  \
    X(RKV_BF16, 128, 1) X(RKV_BF16, 128, 2) X(RKV_BF16, 128, 4) X(RKV_BF16, 128, 7) X(RKV_BF16, 128, 8)   \
    X(RKV_BF16, 64, 1) X(RKV_BF16, 64, 2) X(RKV_BF16, 64, 4) X(RKV_F32, 64, 1) X(RKV_F32, 64, 2)          \
    X(RKV_F32, 64, 4) X(RKV_F32, 128, 1) X(RKV_F32, 128, 2) X(RKV_F32, 128, 4)

}  // namespace

bool step_supported(int dtype, int D, int G) {
#define X(DT, DD, GG) \
    if (dtype == DT && D == DD && G == GG) return true;
    RKV_STEP_CASES(X)
#undef X
    return false;
}

size_t step_smem_bytes(int dtype, int D, int G, int max_pages) {
#define X(DT, DD, GG) \
    if (dtype == DT && D == DD && G == GG) return StepLayout<typename Pick<DT, DD, GG>::M, DD, GG>::smem(max_pages);
    RKV_STEP_CASES(X)
#undef X
    return 0;
}

cudaError_t launch_step(const StepArgs &a, int dtype, int D, int G, int grid, cudaStream_t s,
                        const CUtensorMap &tk, const CUtensorMap &tv) {
#define X(DT, DD, GG) \
    if (dtype == DT && D == DD && G == GG) return launch_one<typename Pick<DT, DD, GG>::M, DD, GG>(a, grid, s, tk, tv);
    RKV_STEP_CASES(X)
#undef X
    return cudaErrorNotSupported;
}

}  // namespace rkv
