// evict_err.cu -- eviction error of a selection (sm_100a).
//
// Trust the Mass (ContourKV), Methodology 1: a kept subset A is scored by
// e(A) = ||mu - m_A||, the distance between the dense attention output mu
// and the forced-weight output m_A over A.  mu mixes the kept and the
// evicted outputs by the dropped mass dm: mu = (1 - dm) m_A + dm m_ev, so
// e = dm * ||m_ev - m_A|| needs only the evicted rows' forced-weight output
// m_ev on top of the attention call's out (m_A) and dropped mass.
//
// One CTA per head.  The keep words give the head's evicted slots, gathered
// UB rows at a time (K and V widened to fp32 in shared memory); each warp
// forms logits of (query row, evicted row) pairs with the lanes splitting
// the head dimension; an online softmax in base 2 per query row folds each
// batch into the weighted V sums that the threads hold; the error is the
// distance to out_kept scaled by the dropped mass.  In steady decoding a
// head evicts a few rows per step, so the kernel reads little beyond the
// keep words.
#include "common.cuh"
#include "internal.h"

namespace rkv {

namespace {

constexpr int ET = 256;   // threads per CTA
constexpr int UB = 32;    // evicted rows per batch
constexpr float LOG2E = 1.4426950408889634f;

template <int D, typename T>
__device__ __forceinline__ float load_elt(const void *pool, int64_t row, int d) {
    if constexpr (sizeof(T) == 2) {
        return __uint_as_float((uint32_t)__ldg(reinterpret_cast<const unsigned short *>(pool) + row * D + d) << 16);
    } else {
        return __ldg(reinterpret_cast<const float *>(pool) + row * D + d);
    }
}

template <int D, int G, typename T>
__global__ void __launch_bounds__(ET) evict_err_kernel(EvictErrArgs a) {
    constexpr int EPT = (G * D + ET - 1) / ET;   // output entries per thread
    __shared__ float Ks[UB][D], Vs[UB][D], Qs[G][D];
    __shared__ float Z[G][UB];                  // base-2 logits, then weights
    __shared__ float mx[G], lsum[G], alpha[G], sq[G];
    __shared__ int rows[UB];
    __shared__ uint32_t scan[40];
    const int64_t c = blockIdx.x;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int n = clamp_len(__ldg(a.n_pre + c), a.max_pages, nullptr);
    const int W = (n + PAGE - 1) / PAGE;
    for (int i = tid; i < G * D; i += ET) Qs[i / D][i % D] = __ldg(a.q + c * G * D + i) * (a.scale * LOG2E);
    if (tid < G) {
        mx[tid] = -INFINITY;
        lsum[tid] = 0.0f;
        sq[tid] = 0.0f;
    }
    float acc[EPT];
#pragma unroll
    for (int u = 0; u < EPT; u++) acc[u] = 0.0f;
    for (int w0 = 0; w0 < W; w0 += ET) {
        const int w = w0 + tid;
        uint32_t ev = 0u;
        int32_t pg = 0;
        if (w < W) {
            const int nv = min(PAGE, n - w * PAGE);
            const uint32_t valid = nv >= PAGE ? 0xFFFFu : ((1u << nv) - 1u);
            ev = valid & ~(uint32_t)__ldg(a.keep_mask + c * a.max_pages + w);
            if (ev) pg = __ldg(a.block_table + c * a.max_pages + w);
        }
        uint32_t total;
        const uint32_t before = block_exclusive_scan((uint32_t)__popc(ev), scan, &total);
        for (uint32_t b0 = 0; b0 < total; b0 += UB) {
            uint32_t bits = ev, r = before;
            while (bits) {
                const int j = __ffs(bits) - 1;
                bits &= bits - 1;
                if (r >= b0 && r < b0 + UB) rows[r - b0] = pg * PAGE + j;
                r++;
            }
            const int nb = (int)min((uint32_t)UB, total - b0);
            __syncthreads();
            for (int i = tid; i < nb * D; i += ET) {
                const int64_t row = rows[i / D];
                Ks[i / D][i % D] = load_elt<D, T>(a.k_pool, row, i % D);
                Vs[i / D][i % D] = load_elt<D, T>(a.v_pool, row, i % D);
            }
            __syncthreads();
            // logits: one warp per (query row, evicted row) pair, lanes over D
            for (int pr = warp; pr < G * nb; pr += ET / 32) {
                const int g = pr / nb, rr = pr % nb;
                float dot = 0.0f;
#pragma unroll
                for (int d = lane; d < D; d += 32) dot = fmaf(Qs[g][d], Ks[rr][d], dot);
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) dot += __shfl_xor_sync(0xFFFFFFFFu, dot, o);
                if (lane == 0) Z[g][rr] = dot;
            }
            __syncthreads();
            // online softmax per query row: new max, rescale factor, weights
            if (tid < G) {
                float m = mx[tid];
                for (int rr = 0; rr < nb; rr++) m = fmaxf(m, Z[tid][rr]);
                const float al = ex2(mx[tid] - m);  // mx = -inf -> 0
                float l = 0.0f;
                for (int rr = 0; rr < nb; rr++) {
                    const float p = ex2(Z[tid][rr] - m);
                    Z[tid][rr] = p;
                    l += p;
                }
                lsum[tid] = lsum[tid] * al + l;
                mx[tid] = m;
                alpha[tid] = al;
            }
            __syncthreads();
#pragma unroll
            for (int u = 0; u < EPT; u++) {
                const int e = tid + u * ET;
                if (e < G * D) {
                    const int g = e / D, d = e % D;
                    float s = acc[u] * alpha[g];
                    for (int rr = 0; rr < nb; rr++) s = fmaf(Z[g][rr], Vs[rr][d], s);
                    acc[u] = s;
                }
            }
            __syncthreads();
        }
    }
    // err = dm * ||m_ev - m_A|| per query row
#pragma unroll
    for (int u = 0; u < EPT; u++) {
        const int e = tid + u * ET;
        if (e < G * D) {
            const int g = e / D;
            const float mev = lsum[g] > 0.0f ? acc[u] / lsum[g] : 0.0f;
            const float x = mev - __ldg(a.out_kept + c * G * D + e);
            atomicAdd(&sq[g], x * x);
        }
    }
    __syncthreads();
    if (tid < G) {
        const float dm = __ldg(a.dropped + c * G + tid);
        a.err[c * G + tid] = (dm > 0.0f && lsum[tid] > 0.0f) ? dm * sqrtf(sq[tid]) : 0.0f;
    }
}

template <int D, typename T>
cudaError_t launch_g(const EvictErrArgs &a, int G, cudaStream_t s) {
    switch (G) {
        case 1: evict_err_kernel<D, 1, T><<<a.C, ET, 0, s>>>(a); break;
        case 2: evict_err_kernel<D, 2, T><<<a.C, ET, 0, s>>>(a); break;
        case 4: evict_err_kernel<D, 4, T><<<a.C, ET, 0, s>>>(a); break;
        case 7: evict_err_kernel<D, 7, T><<<a.C, ET, 0, s>>>(a); break;
        case 8: evict_err_kernel<D, 8, T><<<a.C, ET, 0, s>>>(a); break;
        default: return cudaErrorNotSupported;
    }
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_evict_err(const EvictErrArgs &a, int dtype, int D, int G, cudaStream_t s) {
    if (a.C == 0) return cudaSuccess;
    if (D == 128) return dtype == RKV_BF16 ? launch_g<128, uint16_t>(a, G, s) : launch_g<128, float>(a, G, s);
    if (D == 64) return dtype == RKV_BF16 ? launch_g<64, uint16_t>(a, G, s) : launch_g<64, float>(a, G, s);
    return cudaErrorNotSupported;
}

}  // namespace rkv
