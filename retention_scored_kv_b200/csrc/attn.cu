// attn.cu -- split-K paged grouped-query decode attention over the kept
// entries, with the dropped mass fused into the same pass (sm_100a).
//
// Trust the Mass (ContourKV), Problem definition: after selection the
// softmax is renormalised over the kept set (forced weights).  Methodology 3
// and main contributions: the dropped mass is the dense softmax weight held
// by the evicted keys, over every entry present before the eviction.
//
// Design (HBM-bound: ~512 bytes of K/V per kept entry against 4*G*D flops):
// * Persistent grid, one CTA per SM.  The pages of all heads (pre-compaction
//   lengths, 16 rows each) are flattened in head order and split evenly
//   across CTAs, so ragged per-head lengths cost no imbalance.
// * Warp specialisation: one producer warp streams each page's K (and V when
//   the page holds a kept row) into a multi-stage shared-memory ring through
//   the TMA engine (mbarrier transaction counts), plus each head's queries;
//   eight consumer warps take pages round-robin.
// * Math policies.  bf16 pools (MmaMath): pages arrive as 64-column tensor
//   boxes in the 128-byte-swizzled layout; QK^T and PV run on the tensor
//   cores as m16n8k16 bf16 MMAs with fp32 accumulation -- the G query rows of
//   a KV head padded to 16, queries and softmax weights split into bf16
//   high + low parts so the products keep ~fp32 accuracy; ldmatrix feeds the
//   fragments without bank conflicts.  fp32 pools (CoreMath): CUDA-core FMAs,
//   RL lanes per row, packed f32x2 FMAs and a butterfly per dot product.
// * Online softmax in base 2 with separate running maxima for kept rows and
//   for evicted rows (the latter only for the dropped mass); PV only for kept
//   rows, and V is not fetched for pages without a kept row.
// * Head boundaries: warps merge through shared memory; a head split across
//   CTAs writes partial (max, sum, acc) records and the last CTA to arrive
//   (atomic counter, no waiting) merges them -- the cross-split combine.
#include <cuda.h>

#include "attn_core.cuh"
#include "common.cuh"
#include "internal.h"

namespace rkv {

namespace {

using namespace core;
// ------------------------------------------------------------- skeleton ----
template <class M, int D, int G, bool WITH_V>
struct Layout {
    static constexpr int STAGE_BYTES = M::PAGE_BYTES * (WITH_V ? 2 : 1);
    static constexpr int BUDGET = 131072;                     // stage-ring bytes per CTA
    static constexpr int NSW0 = BUDGET / (NCW * STAGE_BYTES);
    static constexpr int NSW = NSW0 < 1 ? 1 : (NSW0 > 8 ? 8 : NSW0);   // stages per consumer warp
    static constexpr int NST = NCW * NSW;
    static constexpr int QBYTES = G * D * 4;
    static constexpr int REC = G * (D + 4);                   // partial record floats
    static constexpr int WSLOT = G * D + 4 * G;               // per-warp merge slot floats
    static constexpr int OFF_STAGE = 0;
    static constexpr int OFF_Q = OFF_STAGE + NST * STAGE_BYTES;
    static constexpr int OFF_MERGE = OFF_Q + QR * QBYTES;
    static constexpr int OFF_META = OFF_MERGE + 2 * NCW * WSLOT * 4;
    static constexpr int OFF_BAR = (OFF_META + NST * 4 + 15) / 16 * 16;
    static constexpr int NBAR = 2 * NST + 2 * QR;
    static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
    static constexpr int SMEM = OFF_MISC + 128 + M::STAGE_ALIGN;  // + slack to align the stages
    static_assert(QBYTES % 16 == 0, "query block must be a 16-byte multiple");
    static_assert(STAGE_BYTES % M::STAGE_ALIGN == 0, "stage alignment");
    static_assert(SMEM <= 227 * 1024, "shared memory");
    static_assert(NBAR <= ATTN_THREADS, "barrier init");
};

// Pages are dealt to consumer warps round-robin (page li -> warp li % NCW);
// each consumer warp owns a private ring of NSW stages, filled in order by
// the producer warp serving it (warp w is served by producer w % NPW), so
// every mbarrier has exactly one producer and one consumer and a phase is
// never waited on before the previous phase of the same stage completed.
template <class M, int D, int G, bool WITH_V>
__global__ void __launch_bounds__(ATTN_THREADS, 1)
    attn_kernel(AttnArgs a, const __grid_constant__ CUtensorMap tmk, const __grid_constant__ CUtensorMap tmv) {
    using LY = Layout<M, D, G, WITH_V>;
    extern __shared__ __align__(128) unsigned char smem_raw[];
    unsigned char *smem = smem_raw + ((M::STAGE_ALIGN - (smem_u32(smem_raw) & (M::STAGE_ALIGN - 1))) &
                                      (M::STAGE_ALIGN - 1));
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + LY::OFF_BAR);  // [NCW][NSW]
    uint64_t *empty = full + LY::NST;                                   // [NCW][NSW]
    uint64_t *qfull = empty + LY::NST;
    uint64_t *qempty = qfull + QR;
    uint32_t *meta = reinterpret_cast<uint32_t *>(smem + LY::OFF_META);
    float *qring = reinterpret_cast<float *>(smem + LY::OFF_Q);
    float *merge = reinterpret_cast<float *>(smem + LY::OFF_MERGE);
    int *misc = reinterpret_cast<int *>(smem + LY::OFF_MISC);
    int64_t *misc64 = reinterpret_cast<int64_t *>(smem + LY::OFF_MISC + 64);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int nct = gridDim.x;

    // ---- prologue: total pages, this CTA's page range and first head ----
    uint32_t *scan = reinterpret_cast<uint32_t *>(merge);  // reused before the merge slots are live
    const int CS = (a.C + ATTN_THREADS - 1) / ATTN_THREADS;
    const int h0 = min(a.C, tid * CS), h1 = min(a.C, h0 + CS);
    uint32_t my_pages = 0;
    for (int c = h0; c < h1; c++)
        my_pages += (uint32_t)((clamp_len(__ldcg(a.len + c), a.max_pages, a.status) + PAGE - 1) / PAGE);
    if (tid == 0) misc[0] = a.C;
    if (tid < LY::NBAR) {
        // full: producer; empty: the owning consumer warp; qfull: producer 0; qempty: every consumer warp
        mbar_init(full + tid, tid >= 2 * LY::NST + QR ? NCW : 1);
    }
    if (M::USES_TMAP && tid == 0) {
        prefetch_tensormap(&tmk);
        prefetch_tensormap(&tmv);
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
            const int64_t pg = (clamp_len(__ldcg(a.len + c), a.max_pages, nullptr) + PAGE - 1) / PAGE;
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

    if (warp >= NCW) {
        // =============================== producers ===============================
        if constexpr (REG_SPLIT) setmaxnreg_dec<PRODUCER_REGS>();
        const int pw = warp - NCW;
        Walker w;
        w.init(a.len, a.C, a.max_pages, x1, last, c_start, pfx_start);
        const uint64_t pol_kv = policy_evict_first();
        const uint64_t pol_q = policy_evict_last();
        int nq = 0;
        int c, pages, n;
        int64_t pfx;
        while (w.next(&c, &pfx, &pages, &n)) {
            if (pages == 0) continue;
            const int64_t pa = max(pfx, x0), pb = min(pfx + pages, x1);
            if (pw == 0 && lane == 0) {
                const int slot = nq % QR;
                mbar_wait(&qempty[slot], ((nq / QR) & 1) ^ 1, a.status);
                mbar_arrive_expect_tx(&qfull[slot], LY::QBYTES);
                bulk_g2s(qring + slot * G * D, a.q + (int64_t)c * G * D, LY::QBYTES, &qfull[slot], pol_q);
            }
            nq++;
            for (int64_t base = pa; base < pb; base += 32) {
                const int64_t i = base + lane;
                int32_t phys = 0;
                uint32_t m = 0;
                const bool mine = i < pb && ((int)((i - x0) % NCW)) % NPW == pw;
                if (mine) {
                    const int64_t pidx = i - pfx;
                    phys = __ldg(a.block_table + (int64_t)c * a.max_pages + pidx);
                    const int nv = min(PAGE, n - (int)pidx * PAGE);
                    const uint32_t valid = nv >= PAGE ? 0xFFFFu : ((1u << nv) - 1u);
                    const uint32_t kp = a.keep_mask ? (uint32_t)__ldg(a.keep_mask + (int64_t)c * a.max_pages + pidx)
                                                    : 0xFFFFu;
                    m = (kp & valid) | (valid << 16);
                }
                uint32_t todo = __ballot_sync(0xFFFFFFFFu, mine);
                while (todo) {
                    const int j = __ffs(todo) - 1;
                    todo &= todo - 1;
                    const int32_t pj = __shfl_sync(0xFFFFFFFFu, phys, j);
                    const uint32_t mj = __shfl_sync(0xFFFFFFFFu, m, j);
                    if (lane == 0) {
                        const int64_t li = base + j - x0;
                        const int cw = (int)(li % NCW);
                        const int64_t nw = li / NCW;
                        const int sg = cw * LY::NSW + (int)(nw % LY::NSW);
                        mbar_wait(&empty[sg], (uint32_t)((nw / LY::NSW) & 1) ^ 1u, a.status);
                        meta[sg] = mj;
                        const bool load_v = WITH_V && (mj & 0xFFFFu);
                        mbar_arrive_expect_tx(&full[sg], M::PAGE_BYTES * (load_v ? 2 : 1));
                        M::issue(smem + LY::OFF_STAGE + sg * LY::STAGE_BYTES, load_v, pj, &full[sg], a.k_pool,
                                 a.v_pool, &tmk, &tmv, pol_kv);
                    }
                    __syncwarp();
                }
            }
        }
        return;
    }

    // ================================ consumers ================================
    if constexpr (REG_SPLIT) setmaxnreg_inc<CONSUMER_REGS>();
    Walker w;
    w.init(a.len, a.C, a.max_pages, x1, last, c_start, pfx_start);
    int nq = 0;
    int c, pages, n;
    int64_t pfx;
    const int64_t TPl = TP;
    typename M::State st;

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
        {
            const int slot = nq % QR;
            mbar_wait(&qfull[slot], (nq / QR) & 1, a.status);
            M::load_q(st, qring + slot * G * D, a.qscale, lane);
            __syncwarp();
            if (lane == 0) mbar_arrive(&qempty[slot]);
        }
        // ---- pages of this head handled by this warp ----
        const int64_t la = pa - x0, lb = pb - x0;
        for (int64_t li = la + (((int64_t)warp - la) % NCW + NCW) % NCW; li < lb; li += NCW) {
            const int64_t nw = li / NCW;
            const int sg = warp * LY::NSW + (int)(nw % LY::NSW);
            mbar_wait(&full[sg], (uint32_t)((nw / LY::NSW) & 1), a.status);
            const uint32_t mt = meta[sg];
            const uint32_t keepm = mt & 0xFFFFu, evm = (mt >> 16) & ~keepm;
            const unsigned char *sk = smem + LY::OFF_STAGE + sg * LY::STAGE_BYTES;
            M::page(st, sk, sk + M::PAGE_BYTES, keepm, evm, lane);
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[sg]);
        }
        const int par = nq & 1;
        M::flush(st, merge + (par * NCW + warp) * LY::WSLOT, lane);
        nq++;
        named_bar_sync(1, NCW * 32);

        // ---- merge the warps (consumer threads 0 .. NCW*32-1) ----
        const float *mb = merge + par * NCW * LY::WSLOT;
        float *rec = nullptr;
        if (!whole) rec = a.partial + ((int64_t)blockIdx.x * 2 + ((pfx < x0) ? 0 : 1)) * LY::REC;
        for (int e = tid; e < G * D + G; e += NCW * 32) {
            const bool is_stat = e >= G * D;
            const int g = is_stat ? e - G * D : e / D;
            Merged s;
            s.mk = -INFINITY; s.me = -INFINITY;
#pragma unroll
            for (int wi = 0; wi < NCW; wi++) {
                s.mk = fmaxf(s.mk, mb[wi * LY::WSLOT + G * D + g]);
                s.me = fmaxf(s.me, mb[wi * LY::WSLOT + G * D + 2 * G + g]);
            }
            s.lk = 0.0f; s.le = 0.0f;
            float av = 0.0f;
#pragma unroll
            for (int wi = 0; wi < NCW; wi++) {
                const float *src = mb + wi * LY::WSLOT;
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
            if (tid == 0) {
                int ncover = 0;
                for (int j = jf; j <= jl; j++) ncover += range_lo(j, TPl, nct) < range_lo(j + 1, TPl, nct) ? 1 : 0;
                const uint32_t prev = atomicAdd(a.head_cnt + c, 1u);
                misc[4] = (prev + 1 == (uint32_t)ncover) ? 1 : 0;
            }
            named_bar_sync(1, NCW * 32);
            if (misc[4]) {
                __threadfence();
                for (int e = tid; e < G * D + G; e += NCW * 32) {
                    const bool is_stat = e >= G * D;
                    const int g = is_stat ? e - G * D : e / D;
                    Merged s;
                    s.mk = -INFINITY; s.me = -INFINITY; s.lk = 0.0f; s.le = 0.0f;
                    for (int j = jf; j <= jl; j++) {
                        if (!(range_lo(j, TPl, nct) < range_lo(j + 1, TPl, nct))) continue;
                        const float *r = a.partial + ((int64_t)j * 2 + ((pfx < range_lo(j, TPl, nct)) ? 0 : 1)) * LY::REC;
                        s.mk = fmaxf(s.mk, __ldcg(r + G * D + g));
                        s.me = fmaxf(s.me, __ldcg(r + G * D + 2 * G + g));
                    }
                    float av = 0.0f;
                    for (int j = jf; j <= jl; j++) {
                        if (!(range_lo(j, TPl, nct) < range_lo(j + 1, TPl, nct))) continue;
                        const float *r = a.partial + ((int64_t)j * 2 + ((pfx < range_lo(j, TPl, nct)) ? 0 : 1)) * LY::REC;
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
                if (tid == 0) a.head_cnt[c] = 0u;
            }
        }
    }
}

template <class M, int D, int G, bool WITH_V>
cudaError_t launch_one(const AttnArgs &a, int sm_count, cudaStream_t s, const CUtensorMap &tk, const CUtensorMap &tv) {
    using LY = Layout<M, D, G, WITH_V>;
    auto *k = attn_kernel<M, D, G, WITH_V>;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, LY::SMEM);
    if (e != cudaSuccess) return e;
    const int grid = sm_count < MAX_ATTN_CTAS ? sm_count : MAX_ATTN_CTAS;
    k<<<grid, ATTN_THREADS, LY::SMEM, s>>>(a, tk, tv);
    return cudaGetLastError();
}

template <int DT, int D, int G>
cudaError_t launch_dg(const AttnArgs &a, int sm_count, cudaStream_t s, const CUtensorMap &tk, const CUtensorMap &tv) {
    if constexpr (DT == RKV_BF16) {
        return a.out ? launch_one<MmaMath<D, G, true>, D, G, true>(a, sm_count, s, tk, tv)
                     : launch_one<MmaMath<D, G, false>, D, G, false>(a, sm_count, s, tk, tv);
    } else {
        return a.out ? launch_one<CoreMath<float, D, G, true>, D, G, true>(a, sm_count, s, tk, tv)
                     : launch_one<CoreMath<float, D, G, false>, D, G, false>(a, sm_count, s, tk, tv);
    }
}

#define RKV_ATTN_CASES(X)                                                                                  \
    X(RKV_BF16, 128, 1) X(RKV_BF16, 128, 2) X(RKV_BF16, 128, 4) X(RKV_BF16, 128, 7) X(RKV_BF16, 128, 8)   \
    X(RKV_BF16, 64, 1) X(RKV_BF16, 64, 2) X(RKV_BF16, 64, 4) X(RKV_F32, 64, 1) X(RKV_F32, 64, 2)          \
    X(RKV_F32, 64, 4) X(RKV_F32, 128, 1) X(RKV_F32, 128, 2) X(RKV_F32, 128, 4)

}  // namespace

bool attn_supported(int dtype, int D, int G) {
#define X(DT, DD, GG) \
    if (dtype == DT && D == DD && G == GG) return true;
    RKV_ATTN_CASES(X)
#undef X
    return false;
}

bool attn_uses_tensor_maps(int dtype) { return dtype == RKV_BF16; }

size_t attn_partial_rec_floats(int D, int G) { return (size_t)G * (D + 4); }

cudaError_t launch_attn(const AttnArgs &a, int dtype, int D, int G, int sm_count, cudaStream_t s,
                        const CUtensorMap &tk, const CUtensorMap &tv) {
#define X(DT, DD, GG) \
    if (dtype == DT && D == DD && G == GG) return launch_dg<DT, DD, GG>(a, sm_count, s, tk, tv);
    RKV_ATTN_CASES(X)
#undef X
    return cudaErrorNotSupported;
}

}  // namespace rkv
