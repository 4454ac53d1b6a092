// attn.cu -- split-K paged grouped-query decode attention over the kept
// entries, with the dropped mass fused into the same pass (sm_100a).
//
// Trust the Mass (ContourKV), Problem definition: after selection the
// softmax is renormalised over the kept set (forced weights).  Methodology 3
// and main contributions: the dropped mass is the dense softmax weight held
// by the evicted keys, over every entry present before the eviction.
//
// Design (HBM-bound; see the roofline notes in the design document):
// * Persistent grid, one CTA per SM.  The pages of all heads (pre-compaction
//   lengths, 16 rows each) are flattened in head order and split evenly
//   across CTAs, so ragged per-head lengths cost no imbalance.
// * Warp specialisation: one producer warp streams each page's K (and V when
//   the page holds a kept row) into a multi-stage shared-memory ring with
//   cp.async.bulk (TMA bulk copies, 16-byte aligned, mbarrier transaction
//   counts), plus each head's queries; eight consumer warps take pages
//   round-robin.
// * Consumer math on CUDA cores in fp32: RL lanes share a row, each owning
//   16-byte chunks (128-bit shared loads, conflict-free), q held in
//   registers pre-scaled by scale*log2(e); packed f32x2 FMAs; a butterfly
//   over the RL lanes finishes each dot product.  Online softmax in base 2
//   with separate running maxima for kept and evicted rows; PV only for kept
//   rows.
// * Head boundaries: warps merge through shared memory; a head split across
//   CTAs writes partial (max, sum, acc) records and the last CTA to arrive
//   (atomic counter, no waiting) merges them -- the cross-split combine.
#include "common.cuh"
#include "internal.h"

namespace rkv {

namespace {

constexpr int NCW = 8;                 // consumer warps
constexpr int ATTN_THREADS = (NCW + 1) * 32;
constexpr int QR = 4;                  // query ring slots
constexpr float LN2 = 0.69314718055994530942f;

template <typename T, int D, int G, bool WITH_V>
struct Cfg {
    static constexpr int ROW_BYTES = D * (int)sizeof(T);
    static constexpr int CHUNKS = ROW_BYTES / 16;
    static constexpr int RL0 = (G <= 4) ? 8 : 16;
    static constexpr int RL = RL0 < CHUNKS ? RL0 : CHUNKS;   // lanes per row
    static constexpr int CPL = CHUNKS / RL;                   // 16-byte chunks per lane
    static constexpr int EPC = 16 / (int)sizeof(T);           // elements per chunk
    static constexpr int DL = CPL * EPC;                      // dims per lane
    static constexpr int RPP = 32 / RL;                       // rows per pass
    static constexpr int NPASSES = PAGE / RPP;
    static constexpr int PAGE_BYTES = PAGE * ROW_BYTES;
    static constexpr int STAGE_BYTES = PAGE_BYTES * (WITH_V ? 2 : 1);
    static constexpr int NST0 = 98304 / STAGE_BYTES;
    static constexpr int NST = NST0 < 4 ? 4 : (NST0 > 16 ? 16 : NST0);
    static constexpr int QBYTES = G * D * 4;
    static constexpr int REC = G * (D + 4);                   // partial record floats
    static constexpr int WSLOT = G * D + 4 * G;               // per-warp merge slot floats
    // shared-memory layout (bytes)
    static constexpr int OFF_STAGE = 0;
    static constexpr int OFF_Q = OFF_STAGE + NST * STAGE_BYTES;
    static constexpr int OFF_MERGE = OFF_Q + QR * QBYTES;
    static constexpr int OFF_META = OFF_MERGE + 2 * NCW * WSLOT * 4;
    static constexpr int OFF_BAR = (OFF_META + NST * 4 + 15) / 16 * 16;
    static constexpr int OFF_MISC = OFF_BAR + (2 * NST + 2 * QR) * 8;
    static constexpr int SMEM = OFF_MISC + 128;
    static_assert(CHUNKS % RL == 0 && 32 % RL == 0, "lane mapping");
    static_assert(ROW_BYTES % 16 == 0, "rows must be 16-byte multiples");
    static_assert(QBYTES % 16 == 0, "query block must be a 16-byte multiple");
    static_assert(SMEM <= 227 * 1024, "shared memory");
};

// Walks the heads this CTA owns, in order.  A head c with pages = ceil(len/16)
// occupies flattened pages [pfx, pfx + pages).  The CTA owns every head whose
// pages intersect [x0, x1), every empty head with x0 <= pfx < x1, and (last
// CTA only) the trailing empty heads.  Lengths are fetched 32 at a time.
struct Walker {
    const int32_t *len;
    int C;
    int64_t x1;
    bool last;
    int c;
    int64_t pfx;
    int cbuf;
    int32_t lbuf;

    __device__ void init(const int32_t *len_, int C_, int64_t x1_, bool last_, int c0, int64_t pfx0) {
        len = len_; C = C_; x1 = x1_; last = last_; c = c0; pfx = pfx0; cbuf = -64; lbuf = 0;
    }
    // Returns false when done; else the next head and its first page / pages.
    __device__ bool next(int *hc, int64_t *hpfx, int *hpages, int *hlen) {
        if (c >= C) return false;
        if (c < cbuf || c >= cbuf + 32) {
            cbuf = c;
            const int lane = threadIdx.x & 31;
            lbuf = (cbuf + lane < C) ? __ldcg(len + cbuf + lane) : 0;
        }
        int32_t n = __shfl_sync(0xFFFFFFFFu, lbuf, c - cbuf);
        if (n < 0) n = 0;
        const int pages = (n + PAGE - 1) / PAGE;
        if (pfx >= x1 && !last) return false;
        *hc = c; *hpfx = pfx; *hpages = pages; *hlen = n;
        pfx += pages;
        c += 1;
        return true;
    }
};

__device__ __forceinline__ int64_t range_lo(int j, int64_t TP, int n) { return ((int64_t)j * TP) / n; }

__device__ __forceinline__ int owner_of(int64_t x, int64_t TP, int n) {
    int j = (int)((x * n) / TP);
    if (j >= n) j = n - 1;
    while (j + 1 < n && range_lo(j + 1, TP, n) <= x) j++;
    while (j > 0 && range_lo(j, TP, n) > x) j--;
    return j;
}

// Combine per-source (m_k, l_k, m_e, l_e, acc) states; m in base-2 units.
struct Merged {
    float mk, lk, me, le;
};

__device__ __forceinline__ float dm_of(const Merged &s) {
    if (s.le <= 0.0f) return 0.0f;
    if (s.lk <= 0.0f) return 1.0f;
    const float mm = fmaxf(s.mk, s.me);
    const float a = s.lk * ex2(s.mk - mm), b = s.le * ex2(s.me - mm);
    return b / (a + b);
}

template <typename T, int D, int G, bool WITH_V>
__global__ void __launch_bounds__(ATTN_THREADS, 1) attn_kernel(AttnArgs a) {
    using CF = Cfg<T, D, G, WITH_V>;
    extern __shared__ __align__(128) unsigned char smem[];
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + CF::OFF_BAR);
    uint64_t *empty = full + CF::NST;
    uint64_t *qfull = empty + CF::NST;
    uint64_t *qempty = qfull + QR;
    uint32_t *meta = reinterpret_cast<uint32_t *>(smem + CF::OFF_META);
    float *qring = reinterpret_cast<float *>(smem + CF::OFF_Q);
    float *merge = reinterpret_cast<float *>(smem + CF::OFF_MERGE);
    int *misc = reinterpret_cast<int *>(smem + CF::OFF_MISC);
    int64_t *misc64 = reinterpret_cast<int64_t *>(smem + CF::OFF_MISC + 64);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int nct = gridDim.x;

    // ---- prologue: total pages, this CTA's page range and first head ----
    uint32_t *scan = reinterpret_cast<uint32_t *>(merge);  // reused before the merge slots are live
    const int CS = (a.C + ATTN_THREADS - 1) / ATTN_THREADS;
    const int h0 = min(a.C, tid * CS), h1 = min(a.C, h0 + CS);
    uint32_t my_pages = 0;
    for (int c = h0; c < h1; c++) my_pages += (uint32_t)((max(__ldcg(a.len + c), 0) + PAGE - 1) / PAGE);
    if (tid == 0) misc[0] = a.C;
    if (tid < 2 * CF::NST + 2 * QR) {
        // full/empty: one arrival (producer / consuming warp); qfull: producer; qempty: every consumer warp
        mbar_init(full + tid, tid >= 2 * CF::NST + QR ? NCW : 1);
    }
    uint32_t TPu;
    const uint32_t my_pfx = block_exclusive_scan(my_pages, scan + 64, &TPu);
    const int64_t TP = TPu;
    const int64_t x0 = range_lo(blockIdx.x, TP, nct), x1 = range_lo(blockIdx.x + 1, TP, nct);
    const bool last = blockIdx.x == nct - 1;
    // first head c with pfx_c + max(pages_c, 1) > x0 (an empty head at x0 belongs here)
    int cand = a.C;
    int64_t cand_pfx = TP;
    {
        int64_t p = my_pfx;
        for (int c = h0; c < h1; c++) {
            const int64_t pg = (max(__ldcg(a.len + c), 0) + PAGE - 1) / PAGE;
            if (p + (pg > 0 ? pg : 1) > x0) { cand = c; cand_pfx = p; break; }
            p += pg;
        }
    }
    atomicMin(&misc[0], cand);
    fence_mbar_init();
    __syncthreads();
    if (cand < a.C && cand == misc[0]) misc64[0] = cand_pfx;
    __syncthreads();
    const int c_start = misc[0];
    const int64_t pfx_start = c_start < a.C ? misc64[0] : TP;

    if (warp == NCW) {
        // =============================== producer ===============================
        Walker w;
        w.init(a.len, a.C, x1, last, c_start, pfx_start);
        const uint64_t pol_kv = policy_evict_first();
        const uint64_t pol_q = policy_evict_last();
        int nq = 0;
        int c, pages, n;
        int64_t pfx;
        while (w.next(&c, &pfx, &pages, &n)) {
            if (pages == 0) continue;
            const int64_t pa = max(pfx, x0), pb = min(pfx + pages, x1);
            if (lane == 0) {
                const int slot = nq % QR;
                mbar_wait(&qempty[slot], ((nq / QR) & 1) ^ 1, a.status);
                mbar_arrive_expect_tx(&qfull[slot], CF::QBYTES);
                bulk_g2s(qring + slot * G * D, a.q + (int64_t)c * G * D, CF::QBYTES, &qfull[slot], pol_q);
            }
            nq++;
            for (int64_t base = pa; base < pb; base += 32) {
                const int64_t i = base + lane;
                int32_t phys = 0;
                uint32_t m = 0;
                if (i < pb) {
                    const int64_t pidx = i - pfx;
                    phys = __ldg(a.block_table + (int64_t)c * a.max_pages + pidx);
                    const int nv = min(PAGE, n - (int)pidx * PAGE);
                    const uint32_t valid = nv >= PAGE ? 0xFFFFu : ((1u << nv) - 1u);
                    const uint32_t kp = a.keep_mask ? (uint32_t)__ldg(a.keep_mask + (int64_t)c * a.max_pages + pidx)
                                                    : 0xFFFFu;
                    m = (kp & valid) | (valid << 16);
                }
                const int cnt = (int)min((int64_t)32, pb - base);
                for (int j = 0; j < cnt; j++) {
                    const int32_t pj = __shfl_sync(0xFFFFFFFFu, phys, j);
                    const uint32_t mj = __shfl_sync(0xFFFFFFFFu, m, j);
                    if (lane == 0) {
                        const int64_t li = base + j - x0;
                        const int st = (int)(li % CF::NST);
                        mbar_wait(&empty[st], (uint32_t)((li / CF::NST) & 1) ^ 1u, a.status);
                        meta[st] = mj;
                        const bool load_v = WITH_V && (mj & 0xFFFFu);
                        mbar_arrive_expect_tx(&full[st], CF::PAGE_BYTES * (load_v ? 2 : 1));
                        unsigned char *sk = smem + CF::OFF_STAGE + st * CF::STAGE_BYTES;
                        bulk_g2s(sk, (const unsigned char *)a.k_pool + (int64_t)pj * CF::PAGE_BYTES, CF::PAGE_BYTES,
                                 &full[st], pol_kv);
                        if (load_v)
                            bulk_g2s(sk + CF::PAGE_BYTES, (const unsigned char *)a.v_pool + (int64_t)pj * CF::PAGE_BYTES,
                                     CF::PAGE_BYTES, &full[st], pol_kv);
                    }
                    __syncwarp();
                }
            }
        }
        return;
    }

    // ================================ consumers ================================
    constexpr int RL = CF::RL, DL = CF::DL, CPL = CF::CPL, EPC = CF::EPC, RPP = CF::RPP, NPASSES = CF::NPASSES;
    const int rg = lane / RL, tl = lane % RL;
    Walker w;
    w.init(a.len, a.C, x1, last, c_start, pfx_start);
    int nq = 0;
    int c, pages, n;
    int64_t pfx;
    const int64_t TPl = TP;

    while (w.next(&c, &pfx, &pages, &n)) {
        if (pages == 0) {
            // a head with no entries: o = 0, lse = -inf, dropped = 0
            if (warp == 0) {
                for (int e = lane; e < G * D; e += 32)
                    if (a.out) a.out[(int64_t)c * G * D + e] = 0.0f;
                if (lane < G) {
                    if (a.lse) a.lse[(int64_t)c * G + lane] = -INFINITY;
                    if (a.dropped) a.dropped[(int64_t)c * G + lane] = 0.0f;
                }
            }
            continue;
        }
        const int64_t pa = max(pfx, x0), pb = min(pfx + pages, x1);
        const bool whole = (pfx >= x0) && (pfx + pages <= x1);

        // ---- this head's queries, pre-scaled to base-2 logits ----
        float2 q2[G][DL / 2];
        {
            const int slot = nq % QR;
            mbar_wait(&qfull[slot], (nq / QR) & 1, a.status);
            const float *qs = qring + slot * G * D;
#pragma unroll
            for (int g = 0; g < G; g++)
#pragma unroll
                for (int j = 0; j < CPL; j++)
#pragma unroll
                    for (int e = 0; e < EPC; e += 2) {
                        const int d = (tl + RL * j) * EPC + e;
                        q2[g][(j * EPC + e) / 2] = make_float2(qs[g * D + d] * a.qscale, qs[g * D + d + 1] * a.qscale);
                    }
            __syncwarp();
            if (lane == 0) mbar_arrive(&qempty[slot]);
        }
        float mk[G], lk[G], me[G], le[G];
        float2 acc[G][WITH_V ? DL / 2 : 1];
#pragma unroll
        for (int g = 0; g < G; g++) {
            mk[g] = -INFINITY; lk[g] = 0.0f; me[g] = -INFINITY; le[g] = 0.0f;
#pragma unroll
            for (int i = 0; i < (WITH_V ? DL / 2 : 1); i++) acc[g][i] = make_float2(0.0f, 0.0f);
        }

        // ---- pages of this head handled by this warp ----
        const int64_t la = pa - x0, lb = pb - x0;
        int64_t li = la + (((int64_t)warp - la) % NCW + NCW) % NCW;
        for (; li < lb; li += NCW) {
            const int st = (int)(li % CF::NST);
            mbar_wait(&full[st], (uint32_t)((li / CF::NST) & 1), a.status);
            const uint32_t mt = meta[st];
            const uint32_t keepm = mt & 0xFFFFu, validm = mt >> 16, evm = validm & ~keepm;
            const unsigned char *sk = smem + CF::OFF_STAGE + st * CF::STAGE_BYTES;

            // logits of this lane's rows (all-reduced over the RL lanes of a row)
            float y[NPASSES][G];
#pragma unroll
            for (int ps = 0; ps < NPASSES; ps++) {
                const int row = ps * RPP + rg;
                const uint4 *kr = reinterpret_cast<const uint4 *>(sk + row * CF::ROW_BYTES);
                float2 part[G];
#pragma unroll
                for (int g = 0; g < G; g++) part[g] = make_float2(0.0f, 0.0f);
#pragma unroll
                for (int j = 0; j < CPL; j++) {
                    const uint4 wv = kr[tl + RL * j];
                    float2 kp[EPC / 2];
                    if constexpr (sizeof(T) == 2) {
                        kp[0] = bf16x2_to_f2(wv.x); kp[1] = bf16x2_to_f2(wv.y);
                        kp[2] = bf16x2_to_f2(wv.z); kp[3] = bf16x2_to_f2(wv.w);
                    } else {
                        kp[0] = make_float2(__uint_as_float(wv.x), __uint_as_float(wv.y));
                        kp[1] = make_float2(__uint_as_float(wv.z), __uint_as_float(wv.w));
                    }
#pragma unroll
                    for (int e = 0; e < EPC / 2; e++)
#pragma unroll
                        for (int g = 0; g < G; g++) part[g] = ffma2(q2[g][j * EPC / 2 + e], kp[e], part[g]);
                }
#pragma unroll
                for (int g = 0; g < G; g++) {
                    float s = part[g].x + part[g].y;
#pragma unroll
                    for (int o = 1; o < RL; o <<= 1) s += __shfl_xor_sync(0xFFFFFFFFu, s, o);
                    y[ps][g] = s;
                }
            }

            // dense stats of evicted rows, then the online softmax over kept rows
#pragma unroll
            for (int g = 0; g < G; g++) {
                float pk = -INFINITY, pe = -INFINITY;
#pragma unroll
                for (int ps = 0; ps < NPASSES; ps++) {
                    const int row = ps * RPP + rg;
                    if ((keepm >> row) & 1u) pk = fmaxf(pk, y[ps][g]);
                    if ((evm >> row) & 1u) pe = fmaxf(pe, y[ps][g]);
                }
#pragma unroll
                for (int o = RL; o < 32; o <<= 1) {
                    pk = fmaxf(pk, __shfl_xor_sync(0xFFFFFFFFu, pk, o));
                    pe = fmaxf(pe, __shfl_xor_sync(0xFFFFFFFFu, pe, o));
                }
                if (evm) {
                    const float mn = fmaxf(me[g], pe);
                    float sum = 0.0f;
#pragma unroll
                    for (int ps = 0; ps < NPASSES; ps++) {
                        const int row = ps * RPP + rg;
                        if ((evm >> row) & 1u) sum += ex2(y[ps][g] - mn);
                    }
                    le[g] = le[g] * ex2(me[g] - mn) + (tl == 0 ? sum : 0.0f);  // me = -inf -> 0
                    me[g] = mn;
                }
                if (keepm) {
                    const float mn = fmaxf(mk[g], pk);
                    const float alpha = ex2(mk[g] - mn);  // mk = -inf -> 0
                    if (alpha != 1.0f) {
                        lk[g] *= alpha;
                        if constexpr (WITH_V) {
#pragma unroll
                            for (int i = 0; i < DL / 2; i++) { acc[g][i].x *= alpha; acc[g][i].y *= alpha; }
                        }
                    }
                    mk[g] = mn;
                    float sum = 0.0f;
#pragma unroll
                    for (int ps = 0; ps < NPASSES; ps++) {
                        const int row = ps * RPP + rg;
                        const float p = ((keepm >> row) & 1u) ? ex2(y[ps][g] - mn) : 0.0f;
                        y[ps][g] = p;   // y now holds the kept weights
                        sum += p;
                    }
                    lk[g] += (tl == 0) ? sum : 0.0f;
                }
            }

            // PV over kept rows
            if constexpr (WITH_V) {
                if (keepm) {
                    const unsigned char *sv = sk + CF::PAGE_BYTES;
#pragma unroll
                    for (int ps = 0; ps < NPASSES; ps++) {
                        const int row = ps * RPP + rg;
                        const uint4 *vr = reinterpret_cast<const uint4 *>(sv + row * CF::ROW_BYTES);
#pragma unroll
                        for (int j = 0; j < CPL; j++) {
                            const uint4 wv = vr[tl + RL * j];
                            float2 vp[EPC / 2];
                            if constexpr (sizeof(T) == 2) {
                                vp[0] = bf16x2_to_f2(wv.x); vp[1] = bf16x2_to_f2(wv.y);
                                vp[2] = bf16x2_to_f2(wv.z); vp[3] = bf16x2_to_f2(wv.w);
                            } else {
                                vp[0] = make_float2(__uint_as_float(wv.x), __uint_as_float(wv.y));
                                vp[1] = make_float2(__uint_as_float(wv.z), __uint_as_float(wv.w));
                            }
#pragma unroll
                            for (int g = 0; g < G; g++) {
                                const float2 pp = make_float2(y[ps][g], y[ps][g]);
#pragma unroll
                                for (int e = 0; e < EPC / 2; e++)
                                    acc[g][j * EPC / 2 + e] = ffma2(pp, vp[e], acc[g][j * EPC / 2 + e]);
                            }
                        }
                    }
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[st]);
        }

        // ---- warp state -> shared merge slot ----
        const int par = nq & 1;
        float *ws_slot = merge + (par * NCW + warp) * CF::WSLOT;
#pragma unroll
        for (int g = 0; g < G; g++) {
#pragma unroll
            for (int o = RL; o < 32; o <<= 1) {
                lk[g] += __shfl_xor_sync(0xFFFFFFFFu, lk[g], o);
                le[g] += __shfl_xor_sync(0xFFFFFFFFu, le[g], o);
            }
            // lk/le were accumulated by lane tl == 0 of each row group only
            if constexpr (WITH_V) {
#pragma unroll
                for (int i = 0; i < DL / 2; i++) {
#pragma unroll
                    for (int o = RL; o < 32; o <<= 1) {
                        acc[g][i].x += __shfl_xor_sync(0xFFFFFFFFu, acc[g][i].x, o);
                        acc[g][i].y += __shfl_xor_sync(0xFFFFFFFFu, acc[g][i].y, o);
                    }
                }
                if (rg == 0) {
#pragma unroll
                    for (int j = 0; j < CPL; j++)
#pragma unroll
                        for (int e = 0; e < EPC; e += 2) {
                            const int d = (tl + RL * j) * EPC + e;
                            ws_slot[g * D + d] = acc[g][(j * EPC + e) / 2].x;
                            ws_slot[g * D + d + 1] = acc[g][(j * EPC + e) / 2].y;
                        }
                }
            }
            if (lane == 0) {
                ws_slot[G * D + g] = mk[g];
                ws_slot[G * D + G + g] = lk[g];
                ws_slot[G * D + 2 * G + g] = me[g];
                ws_slot[G * D + 3 * G + g] = le[g];
            }
        }
        nq++;
        named_bar_sync(1, NCW * 32);

        // ---- merge the warps (consumer threads 0 .. NCW*32-1) ----
        const int ctid = tid;  // consumers are warps 0..NCW-1
        const float *mb = merge + par * NCW * CF::WSLOT;
        float *rec = nullptr;
        int slot_rec = 0;
        if (!whole) {
            slot_rec = (pfx < x0) ? 0 : 1;
            rec = a.partial + ((int64_t)blockIdx.x * 2 + slot_rec) * CF::REC;
        }
        for (int e = ctid; e < G * D + G; e += NCW * 32) {
            const bool is_stat = e >= G * D;
            const int g = is_stat ? e - G * D : e / D;
            Merged s;
            s.mk = -INFINITY; s.me = -INFINITY;
#pragma unroll
            for (int wi = 0; wi < NCW; wi++) {
                s.mk = fmaxf(s.mk, mb[wi * CF::WSLOT + G * D + g]);
                s.me = fmaxf(s.me, mb[wi * CF::WSLOT + G * D + 2 * G + g]);
            }
            s.lk = 0.0f; s.le = 0.0f;
            float av = 0.0f;
#pragma unroll
            for (int wi = 0; wi < NCW; wi++) {
                const float *src = mb + wi * CF::WSLOT;
                const float mkw = src[G * D + g], mew = src[G * D + 2 * G + g];
                const float fk = (mkw == -INFINITY) ? 0.0f : ex2(mkw - s.mk);
                const float fe = (mew == -INFINITY) ? 0.0f : ex2(mew - s.me);
                s.lk += src[G * D + G + g] * fk;
                s.le += src[G * D + 3 * G + g] * fe;
                if (WITH_V && !is_stat) av += src[e] * fk;
            }
            if (whole) {
                if (!is_stat) {
                    if (WITH_V) a.out[(int64_t)c * G * D + e] = s.lk > 0.0f ? av / s.lk : 0.0f;
                } else {
                    if (a.lse) a.lse[(int64_t)c * G + g] = s.lk > 0.0f ? (s.mk + __log2f(s.lk)) * LN2 : -INFINITY;
                    if (a.dropped) a.dropped[(int64_t)c * G + g] = dm_of(s);
                }
            } else {
                if (!is_stat) {
                    if (WITH_V) rec[e] = av;
                } else {
                    rec[G * D + g] = s.mk;
                    rec[G * D + G + g] = s.lk;
                    rec[G * D + 2 * G + g] = s.me;
                    rec[G * D + 3 * G + g] = s.le;
                }
            }
        }
        if (!whole) {
            // cross-CTA combine: the last of the CTAs covering this head merges
            __threadfence();
            named_bar_sync(1, NCW * 32);
            const int jf = owner_of(pfx, TPl, nct), jl = owner_of(pfx + pages - 1, TPl, nct);
            if (ctid == 0) {
                int ncover = 0;
                for (int j = jf; j <= jl; j++) ncover += range_lo(j, TPl, nct) < range_lo(j + 1, TPl, nct) ? 1 : 0;
                const uint32_t prev = atomicAdd(a.head_cnt + c, 1u);
                misc[4] = (prev + 1 == (uint32_t)ncover) ? 1 : 0;
            }
            named_bar_sync(1, NCW * 32);
            if (misc[4]) {
                __threadfence();
                for (int e = ctid; e < G * D + G; e += NCW * 32) {
                    const bool is_stat = e >= G * D;
                    const int g = is_stat ? e - G * D : e / D;
                    Merged s;
                    s.mk = -INFINITY; s.me = -INFINITY; s.lk = 0.0f; s.le = 0.0f;
                    for (int j = jf; j <= jl; j++) {
                        if (!(range_lo(j, TPl, nct) < range_lo(j + 1, TPl, nct))) continue;
                        const float *r = a.partial + ((int64_t)j * 2 + ((pfx < range_lo(j, TPl, nct)) ? 0 : 1)) * CF::REC;
                        s.mk = fmaxf(s.mk, __ldcg(r + G * D + g));
                        s.me = fmaxf(s.me, __ldcg(r + G * D + 2 * G + g));
                    }
                    float av = 0.0f;
                    for (int j = jf; j <= jl; j++) {
                        if (!(range_lo(j, TPl, nct) < range_lo(j + 1, TPl, nct))) continue;
                        const float *r = a.partial + ((int64_t)j * 2 + ((pfx < range_lo(j, TPl, nct)) ? 0 : 1)) * CF::REC;
                        const float mkw = __ldcg(r + G * D + g), mew = __ldcg(r + G * D + 2 * G + g);
                        const float fk = (mkw == -INFINITY) ? 0.0f : ex2(mkw - s.mk);
                        const float fe = (mew == -INFINITY) ? 0.0f : ex2(mew - s.me);
                        s.lk += __ldcg(r + G * D + G + g) * fk;
                        s.le += __ldcg(r + G * D + 3 * G + g) * fe;
                        if (WITH_V && !is_stat) av += __ldcg(r + e) * fk;
                    }
                    if (!is_stat) {
                        if (WITH_V) a.out[(int64_t)c * G * D + e] = s.lk > 0.0f ? av / s.lk : 0.0f;
                    } else {
                        if (a.lse) a.lse[(int64_t)c * G + g] = s.lk > 0.0f ? (s.mk + __log2f(s.lk)) * LN2 : -INFINITY;
                        if (a.dropped) a.dropped[(int64_t)c * G + g] = dm_of(s);
                    }
                }
                if (ctid == 0) a.head_cnt[c] = 0u;
            }
        }
    }
}

template <typename T, int D, int G, bool WITH_V>
cudaError_t launch_one(const AttnArgs &a, int sm_count, cudaStream_t s) {
    using CF = Cfg<T, D, G, WITH_V>;
    auto *k = attn_kernel<T, D, G, WITH_V>;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, CF::SMEM);
    if (e != cudaSuccess) return e;
    int grid = sm_count < MAX_ATTN_CTAS ? sm_count : MAX_ATTN_CTAS;
    k<<<grid, ATTN_THREADS, CF::SMEM, s>>>(a);
    return cudaGetLastError();
}

template <typename T, int D, int G>
cudaError_t launch_dg(const AttnArgs &a, int sm_count, cudaStream_t s) {
    return a.out ? launch_one<T, D, G, true>(a, sm_count, s) : launch_one<T, D, G, false>(a, sm_count, s);
}

#define RKV_ATTN_CASES(X)                                                                              \
    X(uint16_t, RKV_BF16, 128, 1) X(uint16_t, RKV_BF16, 128, 2) X(uint16_t, RKV_BF16, 128, 4)         \
    X(uint16_t, RKV_BF16, 128, 7) X(uint16_t, RKV_BF16, 128, 8) X(uint16_t, RKV_BF16, 64, 1)          \
    X(uint16_t, RKV_BF16, 64, 2) X(uint16_t, RKV_BF16, 64, 4) X(float, RKV_F32, 64, 1)                \
    X(float, RKV_F32, 64, 2) X(float, RKV_F32, 64, 4) X(float, RKV_F32, 128, 1) X(float, RKV_F32, 128, 2) \
    X(float, RKV_F32, 128, 4)

}  // namespace

bool attn_supported(int dtype, int D, int G) {
#define X(T, DT, DD, GG) \
    if (dtype == DT && D == DD && G == GG) return true;
    RKV_ATTN_CASES(X)
#undef X
    return false;
}

size_t attn_partial_rec_floats(int D, int G) { return (size_t)G * (D + 4); }

cudaError_t launch_attn(const AttnArgs &a, int dtype, int D, int G, int sm_count, cudaStream_t s) {
#define X(T, DT, DD, GG) \
    if (dtype == DT && D == DD && G == GG) return launch_dg<T, DD, GG>(a, sm_count, s);
    RKV_ATTN_CASES(X)
#undef X
    return cudaErrorNotSupported;
}

}  // namespace rkv
