// compact.cu -- physical compaction of the kept entries and token append
// (sm_100a).
//
// Trust the Mass (ContourKV), Methodology 2: the budget is enforced
// physically -- evicted rows are really removed and pages returned, rather
// than masked.  Make Each Token Count (DBTrimKV), Methodology 4: each head
// keeps its own length in a paged layout.
//
// Compaction: one CTA per head.  Keep-mask words give per-word hole counts
// (non-kept slots below n_new) and source counts (kept slots at or above
// n_new); block-wide exclusive scans turn them into ranks, and the j-th hole
// takes the j-th source (binary search over the source prefix, then select
// the bit inside the word).  Warps move whole rows (K, V: 16-byte chunks per
// lane; position and log-retention).  Freed pages go to the free stack at
// offsets given by the per-head prefix the selection kernel computed, so the
// result does not depend on scheduling order.
//
// Append: heads are split across CTAs; each CTA counts the page-needing heads
// before its slice (len % 16 == 0), scans its own slice, pops pages from the
// top of the stack in ascending head order, and warps copy the new rows.  The
// last CTA to finish (atomic ticket, no waiting) bumps every length and the
// stack top, so no CTA ever reads a length another CTA already changed.
#include "common.cuh"
#include "internal.h"

namespace rkv {

namespace {

constexpr int CMP_THREADS = 256;
constexpr int APP_THREADS = 256;

__device__ __forceinline__ int64_t slot_row(const int32_t *table, int64_t c, int max_pages, int k) {
    return (int64_t)__ldg(table + c * max_pages + k / PAGE) * PAGE + (k % PAGE);
}

// Warp-cooperative move of one row (K and V of row_bytes each, position,
// log-retention) from physical row src to physical row dst.
__device__ __forceinline__ void move_row(const CompactArgs &a, int64_t dst, int64_t src, int lane) {
    const int chunks = a.row_bytes / 16;
    uint4 *kd = reinterpret_cast<uint4 *>((unsigned char *)a.k_pool + dst * a.row_bytes);
    const uint4 *ks = reinterpret_cast<const uint4 *>((const unsigned char *)a.k_pool + src * a.row_bytes);
    uint4 *vd = reinterpret_cast<uint4 *>((unsigned char *)a.v_pool + dst * a.row_bytes);
    const uint4 *vs = reinterpret_cast<const uint4 *>((const unsigned char *)a.v_pool + src * a.row_bytes);
    for (int i = lane; i < 2 * chunks; i += 32) {
        if (i < chunks) kd[i] = ks[i];
        else vd[i - chunks] = vs[i - chunks];
    }
    if (lane == 0) {
        a.pos_pool[dst] = a.pos_pool[src];
        a.lb_pool[dst] = a.lb_pool[src];
    }
}

__device__ __forceinline__ uint32_t below_bits(int w, int nn) {
    const int lo = w * PAGE;
    if (lo + PAGE <= nn) return 0xFFFFu;
    if (lo >= nn) return 0u;
    return (1u << (nn - lo)) - 1u;
}

__global__ void __launch_bounds__(CMP_THREADS) compact_kernel(CompactArgs a) {
    extern __shared__ __align__(16) int32_t cs[];
    __shared__ uint32_t scan[40];
    const int64_t c = blockIdx.x;
    const int n = __ldg(a.n_pre + c), nn = __ldg(a.kept + c);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nwarp = blockDim.x >> 5;
    if (c == 0 && tid == 0) *a.free_top = __ldg(a.plan + a.C + 1) + __ldg(a.plan + a.C);
    if (tid == 0) a.len[c] = nn;
    if (nn >= n) return;  // nothing evicted in this head

    const int W = (n + PAGE - 1) / PAGE, Wn = (nn + PAGE - 1) / PAGE;
    int32_t *src_pfx = cs;            // [W]
    int32_t *hole_pfx = cs + W + 1;   // [W]
    const uint16_t *mask = a.keep_mask + c * a.max_pages;
    uint32_t carry_s = 0, carry_h = 0;
    for (int base = 0; base < W; base += blockDim.x) {
        const int w = base + tid;
        uint32_t sc = 0, hc = 0;
        if (w < W) {
            const uint32_t valid = below_bits(w, n);
            const uint32_t m = (uint32_t)__ldg(mask + w) & valid;
            const uint32_t below = below_bits(w, nn);
            sc = __popc(m & ~below & valid);
            hc = __popc(~m & below & 0xFFFFu);
        }
        uint32_t ts, th;
        const uint32_t es = block_exclusive_scan(sc, scan, &ts);
        const uint32_t eh = block_exclusive_scan(hc, scan, &th);
        if (w < W) {
            src_pfx[w] = (int32_t)(carry_s + es);
            hole_pfx[w] = (int32_t)(carry_h + eh);
        }
        carry_s += ts;
        carry_h += th;
    }
    __syncthreads();

    // hole j <- source j
    for (int w = warp; w < Wn; w += nwarp) {
        const uint32_t m = (uint32_t)__ldg(mask + w) & below_bits(w, n);
        uint32_t hb = ~m & below_bits(w, nn) & 0xFFFFu;
        int rank = hole_pfx[w];
        while (hb) {
            const int bit = __ffs(hb) - 1;
            hb &= hb - 1;
            // word holding the rank-th source: largest w' with src_pfx[w'] <= rank
            int lo = 0, hi = W - 1;
            while (lo < hi) {
                const int mid = (lo + hi + 1) >> 1;
                if (src_pfx[mid] <= rank) lo = mid; else hi = mid - 1;
            }
            const uint32_t sm = (uint32_t)__ldg(mask + lo) & below_bits(lo, n) & ~below_bits(lo, nn);
            int skip = rank - src_pfx[lo];
            uint32_t sb = sm;
            for (int i = 0; i < skip; i++) sb &= sb - 1;
            const int sbit = __ffs(sb) - 1;
            const int hslot = w * PAGE + bit, sslot = lo * PAGE + sbit;
            move_row(a, slot_row(a.block_table, c, a.max_pages, hslot), slot_row(a.block_table, c, a.max_pages, sslot),
                     lane);
            rank++;
        }
    }
    __syncthreads();
    // freed pages, ascending table index, at this head's offset in the stack
    const int top0 = __ldg(a.plan + a.C + 1), off = __ldg(a.plan + c);
    for (int pi = Wn + tid; pi < W; pi += blockDim.x) {
        int32_t *e = a.block_table + c * a.max_pages + pi;
        a.free_stack[top0 + off + (pi - Wn)] = *e;
        *e = -1;
    }
}

__global__ void __launch_bounds__(APP_THREADS) append_kernel(AppendArgs a) {
    __shared__ uint32_t scan[40];
    __shared__ int64_t rows[APP_THREADS];
    __shared__ int last_flag;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nwarp = blockDim.x >> 5;
    const int c0 = blockIdx.x * blockDim.x;
    const int c = c0 + tid;
    const int top = __ldcg(a.free_top);
    // page-needing heads before this CTA's slice
    uint32_t before = 0;
    for (int cc = tid; cc < c0; cc += blockDim.x) before += (__ldcg(a.len + cc) % PAGE == 0) ? 1u : 0u;
    uint32_t tot_before;
    block_exclusive_scan(before, scan, &tot_before);
    int k = 0;
    uint32_t need = 0;
    if (c < a.C) {
        k = __ldcg(a.len + c);
        need = (k % PAGE == 0) ? 1u : 0u;
    }
    uint32_t tot_local;
    const uint32_t ex = block_exclusive_scan(need, scan, &tot_local);
    int64_t row = -1;
    if (c < a.C) {
        const int pidx = k / PAGE;
        if (pidx >= a.max_pages) {
            set_status(a.status, RKV_DEV_TABLE_OVERFLOW);
        } else if (need) {
            const int idx = top - 1 - (int)(tot_before + ex);
            if (idx < 0) {
                set_status(a.status, RKV_DEV_POOL_EXHAUSTED);
            } else {
                const int32_t page = __ldcg(a.free_stack + idx);
                a.block_table[(int64_t)c * a.max_pages + pidx] = page;
                row = (int64_t)page * PAGE + (k % PAGE);
            }
        } else {
            row = (int64_t)__ldcg(a.block_table + (int64_t)c * a.max_pages + pidx) * PAGE + (k % PAGE);
        }
        if (row >= 0) {
            a.pos_pool[row] = __ldg(a.t + c / a.LH);
            a.lb_pool[row] = __ldg(a.lb_new + c);
        }
    }
    rows[tid] = row;
    __syncthreads();
    const int chunks = a.row_bytes / 16;
    for (int h = warp; h < (int)blockDim.x; h += nwarp) {
        const int64_t r = rows[h];
        const int64_t ch = c0 + h;
        if (r < 0 || ch >= a.C) continue;
        uint4 *kd = reinterpret_cast<uint4 *>((unsigned char *)a.k_pool + r * a.row_bytes);
        uint4 *vd = reinterpret_cast<uint4 *>((unsigned char *)a.v_pool + r * a.row_bytes);
        const uint4 *ks = reinterpret_cast<const uint4 *>((const unsigned char *)a.k_new + ch * a.row_bytes);
        const uint4 *vs = reinterpret_cast<const uint4 *>((const unsigned char *)a.v_new + ch * a.row_bytes);
        for (int i = lane; i < 2 * chunks; i += 32) {
            if (i < chunks) kd[i] = __ldg(ks + i);
            else vd[i - chunks] = __ldg(vs + i - chunks);
        }
    }
    // last CTA to finish: every length +1, stack top lowered by the pops
    __threadfence();
    __syncthreads();
    if (tid == 0) last_flag = (atomicAdd(a.done, 1u) == gridDim.x - 1) ? 1 : 0;
    __syncthreads();
    if (!last_flag) return;
    __threadfence();
    uint32_t pops = 0;
    for (int cc = tid; cc < a.C; cc += blockDim.x) {
        const int32_t n = __ldcg(a.len + cc);
        pops += (n % PAGE == 0) ? 1u : 0u;
        a.len[cc] = n + 1;
    }
    uint32_t tot_pops;
    block_exclusive_scan(pops, scan, &tot_pops);
    if (tid == 0) {
        const int nt = top - (int)tot_pops;
        *a.free_top = nt < 0 ? 0 : nt;
        *a.done = 0u;
    }
}

}  // namespace

cudaError_t launch_compact(const CompactArgs &a, cudaStream_t s) {
    if (a.C == 0) return cudaSuccess;
    const size_t smem = (size_t)(2 * (a.max_pages + 1)) * sizeof(int32_t);
    cudaError_t e = cudaFuncSetAttribute(compact_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    compact_kernel<<<a.C, CMP_THREADS, smem, s>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_append(const AppendArgs &a, cudaStream_t s) {
    if (a.C == 0) return cudaSuccess;
    append_kernel<<<(a.C + APP_THREADS - 1) / APP_THREADS, APP_THREADS, 0, s>>>(a);
    return cudaGetLastError();
}

}  // namespace rkv
