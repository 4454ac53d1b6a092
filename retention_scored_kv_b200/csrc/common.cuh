// common.cuh -- device helpers shared by the librkv kernels (sm_100a).
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "../../include/rkv.h"

namespace rkv {

constexpr int PAGE = 16;           // rows per page (fixed; keep masks are uint16)
constexpr int NPASS = 6;           // radix digits of the 64-bit key: 11,11,10 | 11,11,10
constexpr int NBINS = 2048;        // bins of the widest digit
constexpr int MAX_ATTN_CTAS = 512; // upper bound of the persistent attention grid
constexpr int WIN_CAP = 1024;      // threshold-window candidates per sequence
// A window that resolved its call is halved above WIN_HI candidates and
// doubled below WIN_LO.
constexpr uint32_t WIN_LO = 16, WIN_HI = 128;
constexpr uint32_t KEY_INVALID = 0xFFFFFFFFu;  // hi word no valid score maps to (NaN space)

// ---------------------------------------------------------------- keys ----
// Order-preserving map of a binary32 score to uint32 such that a HIGHER score
// gives a SMALLER key (negative scores: the bit pattern itself, since larger
// magnitude = lower score; positive scores: complement of the pattern below
// 0x80000000).  +0 maps to 0x7FFFFFFF; -inf to 0xFF800000.  Callers
// canonicalise -0 to +0 and reject NaN first.
__device__ __forceinline__ uint32_t score_key_desc(float s) {
    uint32_t u = __float_as_uint(s);
    return (u & 0x80000000u) ? u : (~u & 0x7FFFFFFFu);
}

// Digit p of the 64-bit key (hi:lo); widths 11,11,10 per 32-bit half.
__device__ __forceinline__ uint32_t key_digit(uint32_t hi, uint32_t lo, int p) {
    uint32_t w = p < 3 ? hi : lo;
    int q = p < 3 ? p : p - 3;
    return q == 0 ? (w >> 21) : (q == 1 ? ((w >> 10) & 0x7FFu) : (w & 0x3FFu));
}
__host__ __device__ __forceinline__ int digit_bits(int p) { return (p % 3 == 2) ? 10 : 11; }
__host__ __device__ __forceinline__ int digit_shift(int p) {
    // bit position of digit p's least significant bit within the 64-bit key
    return (p < 3 ? 32 : 0) + (p % 3 == 0 ? 21 : (p % 3 == 1 ? 10 : 0));
}

// ------------------------------------------------------------ status ----
__device__ __forceinline__ void set_status(int32_t *status, int32_t bits) {
    if ((__ldcg(status) & bits) != bits) atomicOr(status, bits);
}

// A head length as the kernels use it: a negative length counts as 0, and a
// length past the head's block-table row (max_pages * 16 slots) is cut to it
// and recorded as RKV_DEV_BAD_INPUT (status may be NULL at sites that re-read
// a length already checked), so no read leaves the head's row of the table.
__device__ __forceinline__ int32_t clamp_len(int32_t n, int max_pages, int32_t *status) {
    const int32_t cap = max_pages * PAGE;
    if (n > cap) {
        if (status) set_status(status, RKV_DEV_BAD_INPUT);
        return cap;
    }
    return n < 0 ? 0 : n;
}

// A bounded wait that gave up: RKV_DEV_TIMEOUT in status[0] and, if no
// earlier wait gave up, its site code in status[1].
__device__ __forceinline__ void record_timeout(int32_t *status, int32_t site) {
    set_status(status, RKV_DEV_TIMEOUT);
    atomicCAS(status + 1, 0, site);
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Limit of a wait on other CTAs (grid barriers, the append's wait for the
// compactions): status[4] microseconds when set, else 2 s.
__device__ __forceinline__ uint64_t cross_wait_limit_ns(const int32_t *status) {
    const int32_t us = __ldcg(status + 4);
    return us > 0 ? (uint64_t)us * 1000ull : 2000000000ull;
}

__device__ __forceinline__ uint32_t ld_acquire_gpu(const uint32_t *p) {
    uint32_t v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// Grid-wide barrier for a cooperative (co-resident) grid.  `count` is a
// monotonically increasing arrival counter, zero when the launch starts; barrier
// number `epoch` (1, 2, ...) completes when count reaches epoch*gridDim.x.
// The wait is bounded (2 s of globaltimer, or the workspace's wait limit);
// on timeout RKV_DEV_TIMEOUT is recorded and false returned, so the caller
// can leave the kernel.
__device__ __forceinline__ bool grid_barrier(uint32_t *count, uint32_t epoch, int32_t *status,
                                             int *smem_flag, int32_t site = 0x100) {
    __syncthreads();
    if (threadIdx.x == 0) {
        __threadfence();
        atomicAdd(count, 1u);
        const uint32_t target = epoch * gridDim.x;
        int ok = 1;
        if (ld_acquire_gpu(count) < target) {
            const uint64_t t0 = globaltimer_ns(), lim = cross_wait_limit_ns(status);
            const uint32_t every = lim < 100000ull ? 0u : 255u;  // a short limit is checked on every spin
            uint32_t spins = 0;
            while (ld_acquire_gpu(count) < target) {
                if ((++spins & every) == 0 && globaltimer_ns() - t0 > lim) {
                    record_timeout(status, site + (int32_t)epoch);
                    ok = 0;
                    break;
                }
            }
        }
        __threadfence();
        *smem_flag = ok;
    }
    __syncthreads();
    return *smem_flag != 0;
}

// Threshold window kept across calls, per sequence: w[0] bit 0 valid and
// bits 8.. log2(floor) + 1 (0: no floor), [w[1], w[2]) the score-key (high
// word) range whose keys are ranked individually next call, w[3] its half
// width (a power of two).  Centred on this call's threshold score key and
// resized by how this call went: wres 1 resolved in the window (wn
// candidates: shrink above WIN_HI, but never below the floor; grow below
// WIN_LO), 2 missed (grow 4x; the floor becomes twice the half width that
// missed), 3 too many candidates (shrink 4x, drop the floor), 0 no window was
// used.  The floor also follows the threshold's own movement: after every
// call but an overflowing one it is at least DRIFT_MARGIN times the distance
// between this call's threshold score key and the previous window's centre
// (rounded up to a power of two; capped where the key density this call saw
// would put more than WIN_CAP/2 keys inside), and the half width is raised to
// the floor, so the window does not shrink into the step-to-step drift of the
// threshold.  A sequence's
// first window is sized from the density of keys around its threshold when
// the exact selection measured it (h1: keys in the threshold's 1024-wide
// bucket of score keys, 0 if unknown) so that about WIN_INIT keys fall
// inside, else 2^14.  Nothing changes when nothing or everything was kept
// (kappa 0 or ~0).
constexpr uint32_t DRIFT_MARGIN = 4, WIN_INIT = 256;
__device__ __forceinline__ void window_next(uint32_t *w, uint64_t kappa, int wres, uint32_t wn, uint32_t h1 = 0u) {
    if (kappa == 0ull || kappa == ~0ull) return;
    const uint32_t center = (uint32_t)((kappa - 1ull) >> 32);
    const bool had = (w[0] & 1u) != 0u;
    uint32_t hw = w[3];
    if (hw == 0u) {
        hw = 1u << 14;
        if (h1) {
            hw = 1u;
            while (hw < (1u << 20) && (uint64_t)hw * h1 < (uint64_t)WIN_INIT * 512u) hw <<= 1;
        }
    }
    const uint32_t fe = w[0] >> 8;
    uint32_t floor = fe ? 1u << (fe - 1u) : 0u;
    if (had && wres != 3) {
        const uint32_t old = w[1] > 0u ? w[1] + w[3] : w[2] - w[3];
        const uint64_t d = center > old ? center - old : old - center;
        // no higher than the half width at which about WIN_CAP/2 keys would
        // fall inside, at the density this call's window saw (wn keys when it
        // resolved the call)
        uint64_t lim = 1u << 26;
        if (wres == 1 && wn > 0u) {
            const uint64_t dl = (uint64_t)w[3] * (WIN_CAP / 2) / wn;
            if (dl < lim) lim = dl;
        }
        uint32_t fd = 1u;
        while ((uint64_t)fd * 2u <= lim && (uint64_t)fd < DRIFT_MARGIN * d) fd <<= 1;
        if (fd > floor) floor = fd;
        if (hw < floor) hw = floor;
    }
    if (wres == 1) {
        if (wn > WIN_HI) {
            if (hw > 1u && (hw >> 1) >= floor) hw >>= 1;
        } else if (wn < WIN_LO && hw < (1u << 28)) {
            hw <<= 1;
        }
    } else if (wres == 2) {
        floor = hw < (1u << 27) ? hw << 1 : (1u << 28);
        hw = hw < (1u << 26) ? hw << 2 : (1u << 28);
    } else if (wres == 3) {
        floor = 0u;
        hw = hw > 4u ? hw >> 2 : 1u;
    }
    w[1] = center > hw ? center - hw : 0u;
    w[2] = center < 0xFFFFFFFFu - hw ? center + hw : 0xFFFFFFFFu;
    w[3] = hw;
    w[0] = 1u | (floor ? (uint32_t)__ffs(floor) << 8 : 0u);
}

// ------------------------------------------------ mbarrier / bulk copy ----
__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
    asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.shared::cta.b64 st, [%0];\n\t}" ::"r"(smem_u32(bar))
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n\t}" ::"r"(
                     smem_u32(bar)),
                 "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\tselp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Bounded wait on an mbarrier phase.  Every producer of the phase is in the
// same CTA and always arrives, so the bound is a guard, not a protocol:
// after ~2 s the wait records RKV_DEV_TIMEOUT and returns false.  A timeout
// recorded elsewhere (another CTA's wait on the grid) does not end this
// wait: the phase still completes, and leaving early could let the CTA exit
// while bulk copies are still landing in its shared memory.
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity, int32_t *status, int32_t site = 1) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    uint32_t spins = 0;
    while (!mbar_try_wait(bar, parity)) {
        if ((++spins & 255u) == 0 && globaltimer_ns() - t0 > 2000000000ull) {
            record_timeout(status, site);
            return false;
        }
    }
    return true;
}

// One bulk asynchronous global->shared copy through the TMA engine
// (cp.async.bulk, no tensor map): both addresses 16-byte aligned, size a
// multiple of 16; completion is signalled as transaction bytes on `bar`.
__device__ __forceinline__ void bulk_g2s(void *smem_dst, const void *gmem_src, uint32_t bytes, uint64_t *bar,
                                         uint64_t policy) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;" ::"r"(
            smem_u32(smem_dst)),
        "l"(gmem_src), "r"(bytes), "r"(smem_u32(bar)), "l"(policy)
        : "memory");
}

// One 2-D tiled TMA load (cp.async.bulk.tensor) of the box at element
// coordinates (x, y) of `tmap` into shared memory; x * element size must be
// a multiple of 16 bytes.  Completion is counted as transaction bytes on `bar`.
__device__ __forceinline__ void tma_load_2d(void *smem_dst, const CUtensorMap *tmap, int x, int y, uint64_t *bar,
                                            uint64_t policy) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1, {%2, %3}], [%4], %5;" ::"r"(smem_u32(smem_dst)),
        "l"(reinterpret_cast<uint64_t>(tmap)), "r"(x), "r"(y), "r"(smem_u32(bar)), "l"(policy)
        : "memory");
}

// 3-D tiled TMA load of the box at element coordinates (x, y, z).
__device__ __forceinline__ void tma_load_3d(void *smem_dst, const CUtensorMap *tmap, int x, int y, int z,
                                            uint64_t *bar, uint64_t policy) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1, {%2, %3, %4}], [%5], %6;" ::"r"(smem_u32(smem_dst)),
        "l"(reinterpret_cast<uint64_t>(tmap)), "r"(x), "r"(y), "r"(z), "r"(smem_u32(bar)), "l"(policy)
        : "memory");
}

__device__ __forceinline__ void prefetch_tensormap(const CUtensorMap *tmap) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(tmap)) : "memory");
}

__device__ __forceinline__ uint64_t policy_evict_first() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
    return p;
}
__device__ __forceinline__ uint64_t policy_evict_last() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
    return p;
}

__device__ __forceinline__ void named_bar_sync(int id, int nthreads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// ------------------------------------------------------------- math ----
// Base-2 exponential on the SFU (ex2.approx: relative error ~2^-22).
__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Packed fp32 pair multiply-add (sm_100: fma.rn.f32x2), d = a*b + c per lane.
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) {
    uint64_t A, B, Cc, Dd;
    asm("mov.b64 %0, {%1,%2};" : "=l"(A) : "f"(a.x), "f"(a.y));
    asm("mov.b64 %0, {%1,%2};" : "=l"(B) : "f"(b.x), "f"(b.y));
    asm("mov.b64 %0, {%1,%2};" : "=l"(Cc) : "f"(c.x), "f"(c.y));
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(Dd) : "l"(A), "l"(B), "l"(Cc));
    float2 d;
    asm("mov.b64 {%0,%1}, %2;" : "=f"(d.x), "=f"(d.y) : "l"(Dd));
    return d;
}

// bf16x2 word -> two floats (exact widening: a bf16 is the top half of an fp32).
__device__ __forceinline__ float2 bf16x2_to_f2(uint32_t w) {
    return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
}

// ------------------------------------------------------------- scans ----
// Block-wide exclusive scan of one uint32 per thread (blockDim.x <= 1024,
// multiple of 32).  `scratch` holds >= 33 words.  Returns the exclusive
// prefix; *total receives the block sum.
__device__ __forceinline__ uint32_t block_exclusive_scan(uint32_t v, uint32_t *scratch, uint32_t *total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
    uint32_t x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        uint32_t y = __shfl_up_sync(0xFFFFFFFFu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) scratch[warp] = x;
    __syncthreads();
    if (warp == 0) {
        uint32_t w = lane < nw ? scratch[lane] : 0u;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            uint32_t y = __shfl_up_sync(0xFFFFFFFFu, w, o);
            if (lane >= o) w += y;
        }
        if (lane < nw) scratch[lane] = w;
        if (lane == 31) scratch[32] = w;
    }
    __syncthreads();
    uint32_t base = warp > 0 ? scratch[warp - 1] : 0u;
    *total = scratch[32];
    __syncthreads();
    return base + x - v;
}

}  // namespace rkv
