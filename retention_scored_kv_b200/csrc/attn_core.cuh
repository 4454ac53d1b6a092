// attn_core.cuh -- pieces of the paged decode attention shared by the
// standalone attention kernel and the fused decode-step kernel: warp roles
// and register split, the two math policies (tensor-core bf16 pages and
// CUDA-core fp32 pages), the head walker and the split-state merge helpers.
#pragma once
#include <cuda.h>

#include "common.cuh"

namespace rkv {
namespace core {


constexpr int NCW = 8;                 // consumer warps
constexpr int NPW = 4;                 // producer warps (one issuing lane each)
constexpr int ATTN_THREADS = (NCW + NPW) * 32;
// Register split between warpgroups (consumers: warps 0..NCW-1, producers:
// the last NPW warps).  The block launches with LAUNCH_REGS per thread; the
// producer warpgroup gives registers back to the consumer warpgroups:
// NPW*32*PRODUCER_REGS + NCW*32*CONSUMER_REGS <= ATTN_THREADS*LAUNCH_REGS.
constexpr int LAUNCH_REGS = 168;
constexpr int PRODUCER_REGS = 56;
constexpr int CONSUMER_REGS = 224;
constexpr bool REG_SPLIT = (NCW % 4 == 0) && (NPW % 4 == 0);
static_assert(!REG_SPLIT || NPW * 32 * PRODUCER_REGS + NCW * 32 * CONSUMER_REGS <= ATTN_THREADS * LAUNCH_REGS,
              "register split exceeds the launch allocation");

template <int N>
__device__ __forceinline__ void setmaxnreg_inc() {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N));
}
template <int N>
__device__ __forceinline__ void setmaxnreg_dec() {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N));
}
constexpr int QR = 4;                  // query ring slots
constexpr float LN2 = 0.69314718055994530942f;

// ------------------------------------------------------------ CUDA cores ----
template <typename T, int D, int G, bool WITH_V>
struct CoreMath {
    static constexpr int DIM = D;
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
    static constexpr int STAGE_ALIGN = 128;
    static constexpr bool USES_TMAP = false;
    static_assert(CHUNKS % RL == 0 && 32 % RL == 0, "lane mapping");

    struct State {
        float2 q2[G][DL / 2];
        float mk[G], lk[G], me[G], le[G];
        float2 acc[G][WITH_V ? DL / 2 : 1];
    };

    __device__ static void load_q(State &s, const float *qs, float qscale, int lane) {
        const int tl = lane % RL;
#pragma unroll
        for (int g = 0; g < G; g++)
#pragma unroll
            for (int j = 0; j < CPL; j++)
#pragma unroll
                for (int e = 0; e < EPC; e += 2) {
                    const int d = (tl + RL * j) * EPC + e;
                    s.q2[g][(j * EPC + e) / 2] = make_float2(qs[g * D + d] * qscale, qs[g * D + d + 1] * qscale);
                }
#pragma unroll
        for (int g = 0; g < G; g++) {
            s.mk[g] = -INFINITY; s.lk[g] = 0.0f; s.me[g] = -INFINITY; s.le[g] = 0.0f;
#pragma unroll
            for (int i = 0; i < (WITH_V ? DL / 2 : 1); i++) s.acc[g][i] = make_float2(0.0f, 0.0f);
        }
    }

    __device__ static void widen(const uint4 &w, float2 *out) {
        if constexpr (sizeof(T) == 2) {
            out[0] = bf16x2_to_f2(w.x); out[1] = bf16x2_to_f2(w.y);
            out[2] = bf16x2_to_f2(w.z); out[3] = bf16x2_to_f2(w.w);
        } else {
            out[0] = make_float2(__uint_as_float(w.x), __uint_as_float(w.y));
            out[1] = make_float2(__uint_as_float(w.z), __uint_as_float(w.w));
        }
    }

    // keepm / evm: rows accumulated as kept / as evicted.  With CAND, rows in
    // candm (neither kept nor evicted yet) have their G logits stored at
    // zdst[k*G + g], k = rank of the row among candm's bits, for k < zcap.
    template <bool CAND = false>
    __device__ static void page(State &s, const unsigned char *sk, const unsigned char *sv, uint32_t keepm,
                                uint32_t evm, int lane, uint32_t candm = 0u, float *zdst = nullptr, int zcap = 0) {
        const int rg = lane / RL, tl = lane % RL;
        float y[NPASSES][G];
#pragma unroll
        for (int ps = 0; ps < NPASSES; ps++) {
            const int row = ps * RPP + rg;
            const uint4 *kr = reinterpret_cast<const uint4 *>(sk + row * ROW_BYTES);
            float2 part[G];
#pragma unroll
            for (int g = 0; g < G; g++) part[g] = make_float2(0.0f, 0.0f);
#pragma unroll
            for (int j = 0; j < CPL; j++) {
                float2 kp[EPC / 2];
                widen(kr[tl + RL * j], kp);
#pragma unroll
                for (int e = 0; e < EPC / 2; e++)
#pragma unroll
                    for (int g = 0; g < G; g++) part[g] = ffma2(s.q2[g][j * EPC / 2 + e], kp[e], part[g]);
            }
#pragma unroll
            for (int g = 0; g < G; g++) {
                float v = part[g].x + part[g].y;
#pragma unroll
                for (int o = 1; o < RL; o <<= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
                y[ps][g] = v;
            }
        }
        if constexpr (CAND) {
            if (candm && tl == 0) {
#pragma unroll
                for (int ps = 0; ps < NPASSES; ps++) {
                    const int row = ps * RPP + rg;
                    const int k = __popc(candm & ((1u << row) - 1u));
                    if (((candm >> row) & 1u) && k < zcap) {
#pragma unroll
                        for (int g = 0; g < G; g++) zdst[k * G + g] = y[ps][g];
                    }
                }
            }
        }
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
                const float mn = fmaxf(s.me[g], pe);
                float sum = 0.0f;
#pragma unroll
                for (int ps = 0; ps < NPASSES; ps++)
                    if ((evm >> (ps * RPP + rg)) & 1u) sum += ex2(y[ps][g] - mn);
                s.le[g] = s.le[g] * ex2(s.me[g] - mn) + (tl == 0 ? sum : 0.0f);  // me = -inf -> 0
                s.me[g] = mn;
            }
            if (keepm) {
                const float mn = fmaxf(s.mk[g], pk);
                const float alpha = ex2(s.mk[g] - mn);  // mk = -inf -> 0
                if (alpha != 1.0f) {
                    s.lk[g] *= alpha;
                    if constexpr (WITH_V) {
#pragma unroll
                        for (int i = 0; i < DL / 2; i++) { s.acc[g][i].x *= alpha; s.acc[g][i].y *= alpha; }
                    }
                }
                s.mk[g] = mn;
                float sum = 0.0f;
#pragma unroll
                for (int ps = 0; ps < NPASSES; ps++) {
                    const float p = ((keepm >> (ps * RPP + rg)) & 1u) ? ex2(y[ps][g] - mn) : 0.0f;
                    y[ps][g] = p;
                    sum += p;
                }
                s.lk[g] += (tl == 0) ? sum : 0.0f;
            }
        }
        if constexpr (WITH_V) {
            if (keepm) {
#pragma unroll
                for (int ps = 0; ps < NPASSES; ps++) {
                    const uint4 *vr = reinterpret_cast<const uint4 *>(sv + (ps * RPP + rg) * ROW_BYTES);
#pragma unroll
                    for (int j = 0; j < CPL; j++) {
                        float2 vp[EPC / 2];
                        widen(vr[tl + RL * j], vp);
#pragma unroll
                        for (int g = 0; g < G; g++) {
                            const float2 pp = make_float2(y[ps][g], y[ps][g]);
#pragma unroll
                            for (int e = 0; e < EPC / 2; e++)
                                s.acc[g][j * EPC / 2 + e] = ffma2(pp, vp[e], s.acc[g][j * EPC / 2 + e]);
                        }
                    }
                }
            }
        }
    }

    // Warp state -> merge slot [G*D acc][mk G][lk G][me G][le G].
    __device__ static void flush(State &s, float *slot, int lane) {
        const int rg = lane / RL, tl = lane % RL;
#pragma unroll
        for (int g = 0; g < G; g++) {
#pragma unroll
            for (int o = RL; o < 32; o <<= 1) {
                s.lk[g] += __shfl_xor_sync(0xFFFFFFFFu, s.lk[g], o);
                s.le[g] += __shfl_xor_sync(0xFFFFFFFFu, s.le[g], o);
            }
            if constexpr (WITH_V) {
#pragma unroll
                for (int i = 0; i < DL / 2; i++) {
#pragma unroll
                    for (int o = RL; o < 32; o <<= 1) {
                        s.acc[g][i].x += __shfl_xor_sync(0xFFFFFFFFu, s.acc[g][i].x, o);
                        s.acc[g][i].y += __shfl_xor_sync(0xFFFFFFFFu, s.acc[g][i].y, o);
                    }
                }
                if (rg == 0) {
#pragma unroll
                    for (int j = 0; j < CPL; j++)
#pragma unroll
                        for (int e = 0; e < EPC; e += 2) {
                            const int d = (tl + RL * j) * EPC + e;
                            slot[g * D + d] = s.acc[g][(j * EPC + e) / 2].x;
                            slot[g * D + d + 1] = s.acc[g][(j * EPC + e) / 2].y;
                        }
                }
            }
            if (lane == 0) {
                slot[G * D + g] = s.mk[g];
                slot[G * D + G + g] = s.lk[g];
                slot[G * D + 2 * G + g] = s.me[g];
                slot[G * D + 3 * G + g] = s.le[g];
            }
        }
    }

    // Row j of a staged page (row-major) to dst, 16-byte chunks over the lanes.
    __device__ static void copy_row(const unsigned char *sv, int j, void *dst, int lane) {
        const uint4 *src = reinterpret_cast<const uint4 *>(sv + j * ROW_BYTES);
        for (int i = lane; i < CHUNKS; i += 32) reinterpret_cast<uint4 *>(dst)[i] = src[i];
    }

    // Producer: the page's K (and V) rows are contiguous -- one bulk copy each.
    __device__ static void issue(unsigned char *sk, bool load_v, int32_t phys, uint64_t *bar, const void *k_pool,
                                 const void *v_pool, const CUtensorMap *, const CUtensorMap *, uint64_t pol) {
        bulk_g2s(sk, (const unsigned char *)k_pool + (int64_t)phys * PAGE_BYTES, PAGE_BYTES, bar, pol);
        if (load_v)
            bulk_g2s(sk + PAGE_BYTES, (const unsigned char *)v_pool + (int64_t)phys * PAGE_BYTES, PAGE_BYTES, bar,
                     pol);
    }
};

// ----------------------------------------------------------- tensor cores ----
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}
__device__ __forceinline__ float bf16_lo_f(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi_f(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// Split (x0, x1) into bf16x2 high parts and bf16x2 residuals.
__device__ __forceinline__ void split_bf16(float x0, float x1, uint32_t &hi, uint32_t &lo) {
    hi = pack_bf16(x0, x1);
    lo = pack_bf16(x0 - bf16_lo_f(hi), x1 - bf16_hi_f(hi));
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t (&r)[4]) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t (&r)[4]) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}

// D += A * B for m16n8k16 bf16 -> fp32 with all four accumulators: rows 0-7
// of A in a0/a2 (outputs c0/c1), rows 8-15 in a1/a3 (outputs c2/c3).
__device__ __forceinline__ void mma_rows16(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                           uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

template <int D, int G, bool WITH_V>
struct MmaMath {
    static_assert(G >= 1 && G <= 8, "query rows of one KV head must fit 8 MMA rows");
    static_assert(D == 64 || D == 128, "head dim");
    static constexpr int DIM = D;
    static constexpr int ROW_BYTES = D * 2;
    static constexpr int PAGE_BYTES = PAGE * ROW_BYTES;
    static constexpr int NBOX = D / 64;          // 128-byte lines per row (64 columns each)
    static constexpr int KSTEPS = D / 16;
    static constexpr int NT = D / 8;             // PV n-tiles of 8 columns
    static constexpr int STAGE_ALIGN = 1024;     // 128-byte swizzle atoms
    static constexpr bool USES_TMAP = true;

    struct State {
        uint32_t qh[KSTEPS][2], ql[KSTEPS][2];   // A fragments a0, a2 of query row g = lane/4
        float mk, lk, me, le;                     // stats of row g (lk, le: this lane's partial)
        float o[WITH_V ? NT : 1][2];              // PV accumulators c0, c1 of row g
    };

    // A page lands as NBOX planes (64-column halves) of 16 rows x 128 bytes
    // (line L = half*16 + row), the 16-byte chunks of each line XOR-swizzled by
    // L mod 8 -- eight consecutive rows of one half hit eight distinct bank
    // groups, so every 8x8 ldmatrix is conflict-free.
    __device__ static uint32_t swz(int r, int h, int c) {
        const int L = h * PAGE + r;
        return (uint32_t)(L * 128 + ((c ^ (L & 7)) << 4));
    }

    __device__ static void load_q(State &s, const float *qs, float qscale, int lane) {
        const int g = lane >> 2, t = lane & 3;
#pragma unroll
        for (int ks = 0; ks < KSTEPS; ks++) {
#pragma unroll
            for (int h = 0; h < 2; h++) {
                const int d = ks * 16 + h * 8 + 2 * t;
                float x0 = 0.0f, x1 = 0.0f;
                if (g < G) {
                    x0 = qs[g * D + d] * qscale;
                    x1 = qs[g * D + d + 1] * qscale;
                }
                split_bf16(x0, x1, s.qh[ks][h], s.ql[ks][h]);
            }
        }
        s.mk = -INFINITY; s.lk = 0.0f; s.me = -INFINITY; s.le = 0.0f;
#pragma unroll
        for (int i = 0; i < (WITH_V ? NT : 1); i++) s.o[i][0] = s.o[i][1] = 0.0f;
    }

    // keepm / evm / CAND, candm, zdst, zcap: as in CoreMath::page.
    template <bool CAND = false>
    __device__ static void page(State &s, const unsigned char *sk, const unsigned char *sv, uint32_t keepm,
                                uint32_t evm, int lane, uint32_t candm = 0u, float *zdst = nullptr, int zcap = 0) {
        const int t = lane & 3, mi = lane >> 3, r8 = lane & 7;
        // ---- S = Q K^T for the 16 rows of the page (two n-tiles of 8 rows) ----
        // the high query parts fill MMA rows 0-7 and the low parts rows 8-15,
        // so one MMA carries both; two accumulation chains (the 8-row halves
        // of the page), high and low parts summed at the end
        float s0[4] = {0.0f, 0.0f, 0.0f, 0.0f}, s1[4] = {0.0f, 0.0f, 0.0f, 0.0f};
        const uint32_t kbase = smem_u32(sk);
#pragma unroll
        for (int ks = 0; ks < KSTEPS; ks++) {
            const int r = (mi >> 1) * 8 + r8, ch = (ks & 3) * 2 + (mi & 1);
            uint32_t b[4];
            ldsm_x4(kbase + swz(r, ks >> 2, ch), b);
            mma_rows16(s0, s.qh[ks][0], s.ql[ks][0], s.qh[ks][1], s.ql[ks][1], b[0], b[1]);
            mma_rows16(s1, s.qh[ks][0], s.ql[ks][0], s.qh[ks][1], s.ql[ks][1], b[2], b[3]);
        }
        // this lane holds row g = lane/4 at page rows j = 2t, 2t+1, 2t+8, 2t+9
        const float y[4] = {s0[0] + s0[2], s0[1] + s0[3], s1[0] + s1[2], s1[1] + s1[3]};
        const int jr[4] = {2 * t, 2 * t + 1, 2 * t + 8, 2 * t + 9};
        if constexpr (CAND) {
            if (candm && (lane >> 2) < G) {
#pragma unroll
                for (int i = 0; i < 4; i++) {
                    const int k = __popc(candm & ((1u << jr[i]) - 1u));
                    if (((candm >> jr[i]) & 1u) && k < zcap) zdst[k * G + (lane >> 2)] = y[i];
                }
            }
        }
        float pk = -INFINITY, pe = -INFINITY;
#pragma unroll
        for (int i = 0; i < 4; i++) {
            if ((keepm >> jr[i]) & 1u) pk = fmaxf(pk, y[i]);
            if ((evm >> jr[i]) & 1u) pe = fmaxf(pe, y[i]);
        }
#pragma unroll
        for (int o = 1; o < 4; o <<= 1) {
            pk = fmaxf(pk, __shfl_xor_sync(0xFFFFFFFFu, pk, o));
            pe = fmaxf(pe, __shfl_xor_sync(0xFFFFFFFFu, pe, o));
        }
        if (evm) {
            const float mn = fmaxf(s.me, pe);
            float sum = 0.0f;
#pragma unroll
            for (int i = 0; i < 4; i++)
                if ((evm >> jr[i]) & 1u) sum += ex2(y[i] - mn);
            s.le = s.le * ex2(s.me - mn) + sum;  // me = -inf -> 0
            s.me = mn;
        }
        if (!keepm) return;
        const float mn = fmaxf(s.mk, pk);
        const float alpha = ex2(s.mk - mn);  // mk = -inf -> 0
        s.mk = mn;
        float p[4];
#pragma unroll
        for (int i = 0; i < 4; i++) p[i] = ((keepm >> jr[i]) & 1u) ? ex2(y[i] - mn) : 0.0f;
        s.lk = s.lk * alpha + (p[0] + p[1]) + (p[2] + p[3]);
        if constexpr (WITH_V) {
            if (__any_sync(0xFFFFFFFFu, alpha != 1.0f)) {
#pragma unroll
                for (int i = 0; i < NT; i++) { s.o[i][0] *= alpha; s.o[i][1] *= alpha; }
            }
            uint32_t ph0, pl0, ph2, pl2;
            split_bf16(p[0], p[1], ph0, pl0);
            split_bf16(p[2], p[3], ph2, pl2);
            const uint32_t vbase = smem_u32(sv);
#pragma unroll
            for (int np = 0; np < NT / 2; np++) {
                const int r = (mi & 1) * 8 + r8, ch = (np & 3) * 2 + (mi >> 1);
                uint32_t b[4];
                ldsm_x4_t(vbase + swz(r, np >> 2, ch), b);
                // high weights in MMA rows 0-7, low weights in rows 8-15
                float d0[4] = {s.o[2 * np][0], s.o[2 * np][1], 0.0f, 0.0f};
                float d1[4] = {s.o[2 * np + 1][0], s.o[2 * np + 1][1], 0.0f, 0.0f};
                mma_rows16(d0, ph0, pl0, ph2, pl2, b[0], b[1]);
                mma_rows16(d1, ph0, pl0, ph2, pl2, b[2], b[3]);
                s.o[2 * np][0] = d0[0] + d0[2];
                s.o[2 * np][1] = d0[1] + d0[3];
                s.o[2 * np + 1][0] = d1[0] + d1[2];
                s.o[2 * np + 1][1] = d1[1] + d1[3];
            }
        }
    }

    __device__ static void flush(State &s, float *slot, int lane) {
        const int g = lane >> 2, t = lane & 3;
#pragma unroll
        for (int o = 1; o < 4; o <<= 1) {
            s.lk += __shfl_xor_sync(0xFFFFFFFFu, s.lk, o);
            s.le += __shfl_xor_sync(0xFFFFFFFFu, s.le, o);
        }
        if (g < G) {
            if constexpr (WITH_V) {
                // (column pairs 2t, 2t + 1: one 8-byte store each; slots are 8-byte aligned)
#pragma unroll
                for (int i = 0; i < NT; i++)
                    *reinterpret_cast<float2 *>(slot + g * D + i * 8 + 2 * t) = make_float2(s.o[i][0], s.o[i][1]);
            }
            if (t == 0) {
                slot[G * D + g] = s.mk;
                slot[G * D + G + g] = s.lk;
                slot[G * D + 2 * G + g] = s.me;
                slot[G * D + 3 * G + g] = s.le;
            }
        }
    }

    // Row j of a staged page to dst as D row-major bf16: lane h*8 + c copies
    // chunk c of half h out of the swizzled planes.
    __device__ static void copy_row(const unsigned char *sv, int j, void *dst, int lane) {
        if (lane < NBOX * 8) {
            const int h = lane >> 3, c = lane & 7;
            reinterpret_cast<uint4 *>(dst)[h * 8 + c] = *reinterpret_cast<const uint4 *>(sv + swz(j, h, c));
        }
    }

    // Producer: one 3-D tensor box (64 columns x 16 rows x NBOX halves) per
    // page of K (and of V), 128-byte swizzled.
    __device__ static void issue(unsigned char *sk, bool load_v, int32_t phys, uint64_t *bar, const void *,
                                 const void *, const CUtensorMap *tk, const CUtensorMap *tv, uint64_t pol) {
        tma_load_3d(sk, tk, 0, phys * PAGE, 0, bar, pol);
        if (load_v) tma_load_3d(sk + PAGE_BYTES, tv, 0, phys * PAGE, 0, bar, pol);
    }
};

// Walks the heads this CTA owns, in order.  A head c with pages = ceil(len/16)
// occupies flattened pages [pfx, pfx + pages).  The CTA owns every head whose
// pages intersect [x0, x1), every empty head with x0 <= pfx < x1, and (last
// CTA only) the trailing empty heads.  Lengths are fetched 32 at a time and
// clamped to [0, max_pages*16] (the kernels' prologues record a length past
// that as bad input).
struct Walker {
    const int32_t *len;
    int C, maxlen;
    int64_t x1;
    bool last;
    int c;
    int64_t pfx;
    int cbuf;
    int32_t lbuf;

    __device__ void init(const int32_t *len_, int C_, int max_pages, int64_t x1_, bool last_, int c0,
                         int64_t pfx0) {
        len = len_; C = C_; maxlen = max_pages * PAGE; x1 = x1_; last = last_; c = c0; pfx = pfx0;
        cbuf = -64; lbuf = 0;
    }
    __device__ bool next(int *hc, int64_t *hpfx, int *hpages, int *hlen) {
        if (c >= C) return false;
        if (c < cbuf || c >= cbuf + 32) {
            cbuf = c;
            const int lane = threadIdx.x & 31;
            lbuf = (cbuf + lane < C) ? __ldcg(len + cbuf + lane) : 0;
        }
        int32_t n = __shfl_sync(0xFFFFFFFFu, lbuf, c - cbuf);
        n = n < 0 ? 0 : (n > maxlen ? maxlen : n);
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

}  // namespace core
}  // namespace rkv
