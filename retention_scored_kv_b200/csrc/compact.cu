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
// Append: 32 heads per CTA; each CTA counts the page-needing heads before its
// slice (len % 16 == 0 with room left in the head's table), scans its own
// slice, pops pages from the top of the stack in ascending head order, and
// warps store the new rows (loaded into registers at kernel start).  The last
// CTA to finish (atomic ticket, no waiting) bumps the length of every head
// that appended and lowers the stack top, so no CTA ever reads a length
// another CTA already changed; a head that could not append keeps its length.
#include "common.cuh"
#include "internal.h"

namespace rkv {

namespace {

constexpr int CMP_THREADS = 128;
constexpr int CMP_PAIRS = 1024;   // hole/source pairs resolved per round
constexpr int APP_THREADS = 128;  // 4 warps
constexpr int APP_HEADS = 32;     // heads per append CTA (8 per warp)
constexpr int MAX_ROW_CHUNKS = 32; // 16-byte chunks of one K (or V) row: D*elt <= 512 bytes

// A head of length n pops a page on append: n is a multiple of 16 and the
// new page's table index n/16 is inside the head's table row.
__device__ __forceinline__ bool pops_page(int32_t n, int max_pages) {
    return n >= 0 && n % PAGE == 0 && n / PAGE < max_pages;
}

__device__ __forceinline__ uint32_t below_bits(int w, int nn) {
    const int lo = w * PAGE;
    if (lo + PAGE <= nn) return 0xFFFFu;
    if (lo >= nn) return 0u;
    return (1u << (nn - lo)) - 1u;
}

// Block-wide exclusive scan over W words of a shared array, in place.
__device__ void scan_words(int32_t *v, int W, uint32_t *scratch) {
    uint32_t carry = 0;
    for (int base = 0; base < W; base += blockDim.x) {
        const int w = base + threadIdx.x;
        const uint32_t x = w < W ? (uint32_t)v[w] : 0u;
        uint32_t tot;
        const uint32_t ex = block_exclusive_scan(x, scratch, &tot);
        if (w < W) v[w] = (int32_t)(carry + ex);
        carry += tot;
    }
    if (threadIdx.x == 0) v[W] = (int32_t)carry;
    __syncthreads();
}

// One CTA per head.  The head's keep-mask words and block-table entries are
// staged in shared memory with one round of independent loads; per-word hole
// and source counts are scanned into ranks; pairs (j-th hole, j-th source) are
// resolved in shared memory, then warps move the rows with every lane's
// loads issued before its stores.
__global__ void __launch_bounds__(CMP_THREADS) compact_kernel(CompactArgs a) {
    extern __shared__ __align__(16) int32_t cs[];
    __shared__ uint32_t scan[40];
    __shared__ int2 pairs[CMP_PAIRS];
    const int64_t c = blockIdx.x;
    const int n = __ldg(a.n_pre + c), nn = __ldg(a.kept + c);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nwarp = blockDim.x >> 5;
    if (c == 0 && tid == 0) *a.free_top = __ldg(a.plan + a.C + 1) + __ldg(a.plan + a.C);
    if (nn >= n) return;  // nothing evicted in this head (len unchanged)
    if (tid == 0) a.len[c] = nn;

    const int W = (n + PAGE - 1) / PAGE, Wn = (nn + PAGE - 1) / PAGE;
    const int mp = a.max_pages;
    int32_t *tbl = cs;                  // [W] page ids
    uint16_t *msk = reinterpret_cast<uint16_t *>(cs + mp);   // [W] keep words (valid bits only)
    int32_t *src_pfx = cs + mp + (mp + 1) / 2 + 1;           // [W + 1]
    int32_t *hole_pfx = src_pfx + mp + 1;                    // [W + 1]
    const uint16_t *mask = a.keep_mask + c * mp;
    for (int w = tid; w < W; w += blockDim.x) {
        tbl[w] = a.block_table[c * mp + w];
        msk[w] = (uint16_t)((uint32_t)__ldg(mask + w) & below_bits(w, n));
    }
    __syncthreads();
    for (int w = tid; w < W; w += blockDim.x) {
        const uint32_t m = msk[w], below = below_bits(w, nn);
        src_pfx[w] = __popc(m & ~below);
        hole_pfx[w] = __popc(~m & below & 0xFFFFu);
    }
    __syncthreads();
    scan_words(src_pfx, W, scan);
    scan_words(hole_pfx, W, scan);
    const int moves = hole_pfx[W];
    const int chunks = a.row_bytes / 16;

    for (int r0 = 0; r0 < moves; r0 += CMP_PAIRS) {
        const int r1 = min(moves, r0 + CMP_PAIRS);
        // resolve pairs with rank in [r0, r1): thread per hole word
        for (int w = tid; w < Wn; w += blockDim.x) {
            int rank = hole_pfx[w];
            if (rank >= r1 || hole_pfx[w + 1] <= r0) continue;
            uint32_t hb = ~(uint32_t)msk[w] & below_bits(w, nn) & 0xFFFFu;
            while (hb) {
                const int bit = __ffs(hb) - 1;
                hb &= hb - 1;
                if (rank >= r0 && rank < r1) {
                    int lo = 0, hi = W - 1;  // word of the rank-th source: last w' with src_pfx[w'] <= rank
                    while (lo < hi) {
                        const int mid = (lo + hi + 1) >> 1;
                        if (src_pfx[mid] <= rank) lo = mid; else hi = mid - 1;
                    }
                    uint32_t sb = (uint32_t)msk[lo] & ~below_bits(lo, nn);
                    for (int i = rank - src_pfx[lo]; i > 0; i--) sb &= sb - 1;
                    const int hslot = w * PAGE + bit, sslot = lo * PAGE + (__ffs(sb) - 1);
                    pairs[rank - r0] = make_int2((int)((int64_t)tbl[hslot / PAGE] * PAGE + hslot % PAGE),
                                                 (int)((int64_t)tbl[sslot / PAGE] * PAGE + sslot % PAGE));
                }
                rank++;
            }
        }
        __syncthreads();
        // move rows: each warp takes pairs; a row is K chunks then V chunks
        for (int pi = warp; pi < r1 - r0; pi += nwarp) {
            const int64_t dst = pairs[pi].x, src = pairs[pi].y;
            uint4 v0 = make_uint4(0, 0, 0, 0), v1 = v0;
            const int i0 = lane, i1 = lane + 32;
            const uint4 *ks = reinterpret_cast<const uint4 *>((const unsigned char *)a.k_pool + src * a.row_bytes);
            const uint4 *vs = reinterpret_cast<const uint4 *>((const unsigned char *)a.v_pool + src * a.row_bytes);
            if (i0 < 2 * chunks) v0 = i0 < chunks ? ks[i0] : vs[i0 - chunks];
            if (i1 < 2 * chunks) v1 = i1 < chunks ? ks[i1] : vs[i1 - chunks];
            int32_t pos = 0;
            float lbv = 0.0f;
            if (lane == 0) { pos = a.pos_pool[src]; lbv = a.lb_pool[src]; }
            uint4 *kd = reinterpret_cast<uint4 *>((unsigned char *)a.k_pool + dst * a.row_bytes);
            uint4 *vd = reinterpret_cast<uint4 *>((unsigned char *)a.v_pool + dst * a.row_bytes);
            if (i0 < 2 * chunks) { if (i0 < chunks) kd[i0] = v0; else vd[i0 - chunks] = v0; }
            if (i1 < 2 * chunks) { if (i1 < chunks) kd[i1] = v1; else vd[i1 - chunks] = v1; }
            if (lane == 0) { a.pos_pool[dst] = pos; a.lb_pool[dst] = lbv; }
        }
        __syncthreads();
    }
    // freed pages, ascending table index, at this head's offset in the stack
    const int top0 = __ldg(a.plan + a.C + 1), off = __ldg(a.plan + c);
    for (int pi = Wn + tid; pi < W; pi += blockDim.x) {
        a.free_stack[top0 + off + (pi - Wn)] = tbl[pi];
        a.block_table[c * mp + pi] = -1;
    }
}

// APP_HEADS heads per CTA.  Every independent load is issued first: the
// lengths before this slice (pages needed by earlier heads), this slice's
// lengths, the stack top, and the new rows themselves (into registers).
// Pops are ranked by an exclusive scan; the last CTA to finish (atomic
// ticket, no waiting) bumps every length and lowers the stack top.
__global__ void __launch_bounds__(APP_THREADS) append_kernel(AppendArgs a) {
    __shared__ uint32_t scan[40];
    __shared__ int64_t rows[APP_HEADS];
    __shared__ int last_flag;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int c0 = blockIdx.x * APP_HEADS;
    const int chunks = a.row_bytes / 16;                 // <= MAX_ROW_CHUNKS
    constexpr int HPW = APP_HEADS / (APP_THREADS / 32);  // heads per warp
    const int top = __ldcg(a.free_top);
    uint32_t before = 0;
    for (int cc = tid; cc < c0; cc += blockDim.x) before += pops_page(__ldcg(a.len + cc), a.max_pages) ? 1u : 0u;
    int k = 0, tb = 0;
    float lbn = 0.0f;
    const int c = c0 + lane;
    const bool mine = warp == 0 && c < a.C;
    if (mine) {
        k = __ldcg(a.len + c);
        tb = __ldg(a.t + c / a.LH);
        lbn = __ldg(a.lb_new + c);
    }
    // this warp's new rows, chunk i of head h in lane (i % 32), slot i / 32
    uint4 buf[HPW][2];
#pragma unroll
    for (int h = 0; h < HPW; h++) {
        const int64_t ch = c0 + warp * HPW + h;
#pragma unroll
        for (int j = 0; j < 2; j++) {
            const int i = lane + 32 * j;
            buf[h][j] = make_uint4(0, 0, 0, 0);
            if (ch < a.C && i < 2 * chunks) {
                const uint4 *src = reinterpret_cast<const uint4 *>(
                    (const unsigned char *)(i < chunks ? a.k_new : a.v_new) + ch * a.row_bytes);
                buf[h][j] = __ldg(src + (i < chunks ? i : i - chunks));
            }
        }
    }
    uint32_t tot_before;
    block_exclusive_scan(before, scan, &tot_before);
    const uint32_t need = (mine && pops_page(k, a.max_pages)) ? 1u : 0u;
    uint32_t ex = 0;
    {
        // exclusive scan of need over warp 0
        uint32_t x = need;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t y = __shfl_up_sync(0xFFFFFFFFu, x, o);
            if (lane >= o) x += y;
        }
        ex = x - need;
    }
    if (warp == 0) {
        int64_t row = -1;
        if (mine) {
            const int pidx = k / PAGE;
            if (k < 0) {
                set_status(a.status, RKV_DEV_BAD_INPUT);
            } else if (pidx >= a.max_pages) {
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
                a.pos_pool[row] = tb;
                a.lb_pool[row] = lbn;
            }
        }
        rows[lane] = row;
    }
    __syncthreads();
#pragma unroll
    for (int h = 0; h < HPW; h++) {
        const int hl = warp * HPW + h;
        const int64_t r = rows[hl];
        if (r < 0 || c0 + hl >= a.C) continue;
#pragma unroll
        for (int j = 0; j < 2; j++) {
            const int i = lane + 32 * j;
            if (i < 2 * chunks) {
                uint4 *dst = reinterpret_cast<uint4 *>((unsigned char *)(i < chunks ? a.k_pool : a.v_pool) +
                                                       r * a.row_bytes);
                dst[i < chunks ? i : i - chunks] = buf[h][j];
            }
        }
    }
    // last CTA to finish: the length of every head whose append succeeded
    // +1 and the stack top lowered by the pops that found a page.  Success is
    // decided as above: a length in [0, max_pages*16) and, when the head pops,
    // a pop rank (ascending heads) below the stack top.
    __threadfence();
    __syncthreads();
    if (tid == 0) last_flag = (atomicAdd(a.done, 1u) == gridDim.x - 1) ? 1 : 0;
    __syncthreads();
    if (!last_flag) return;
    __threadfence();
    uint32_t rank0 = 0;
    for (int base = 0; base < a.C; base += blockDim.x) {
        const int cc = base + tid;
        const int32_t nl = cc < a.C ? __ldcg(a.len + cc) : -1;
        const bool pops = cc < a.C && pops_page(nl, a.max_pages);
        uint32_t tot;
        const uint32_t ex = block_exclusive_scan(pops ? 1u : 0u, scan, &tot);
        const bool ok = nl >= 0 && nl / PAGE < a.max_pages && (!pops || (int64_t)rank0 + ex < (int64_t)top);
        if (cc < a.C && ok) a.len[cc] = nl + 1;
        rank0 += tot;
    }
    if (tid == 0) {
        const int nt = top - (int)min((int64_t)rank0, (int64_t)(top > 0 ? top : 0));
        *a.free_top = nt < 0 ? 0 : nt;
        *a.done = 0u;
    }
}

}  // namespace

namespace {
__global__ void set_word_kernel(int32_t *p, int32_t v) { *p = v; }
}  // namespace

cudaError_t launch_set_word(int32_t *p, int32_t v, cudaStream_t s) {
    set_word_kernel<<<1, 1, 0, s>>>(p, v);
    return cudaGetLastError();
}

cudaError_t launch_compact(const CompactArgs &a, cudaStream_t s) {
    if (a.C == 0) return cudaSuccess;
    // page ids, keep words, two prefix arrays
    const size_t smem = (size_t)(a.max_pages + (a.max_pages + 1) / 2 + 1 + 2 * (a.max_pages + 1)) * sizeof(int32_t);
    if (smem > 200 * 1024) return cudaErrorNotSupported;
    if (a.row_bytes > 16 * MAX_ROW_CHUNKS) return cudaErrorNotSupported;
    cudaError_t e = cudaFuncSetAttribute(compact_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    compact_kernel<<<a.C, CMP_THREADS, smem, s>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_append(const AppendArgs &a, cudaStream_t s) {
    if (a.C == 0) return cudaSuccess;
    if (a.row_bytes > 16 * MAX_ROW_CHUNKS) return cudaErrorNotSupported;
    append_kernel<<<(a.C + APP_HEADS - 1) / APP_HEADS, APP_THREADS, 0, s>>>(a);
    return cudaGetLastError();
}

}  // namespace rkv
