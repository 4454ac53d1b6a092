// memory.cu -- latent memory for evicted tokens (sm_100a).
//
// IndexMem (learned KV eviction with latent memory), Methodology B: the
// evicted tokens update a fixed-size state M and a stabilising vector b
// online by outer-product accumulation with decay (fast weights); a learned
// projection and a gate g(q) read it (slow weights); the attention output
// becomes o = o_attn + g(q) * m(q).  This library's form (the page gives
// none): per KV head c, phi(x) = elu(P_l x) + 1,
//   update:  M_c = decay * M_c + sum_{j evicted} phi(k_j) v_j^T,
//            b_c = decay * b_c + sum_{j evicted} phi(k_j);
//   read:    m = phi(q)^T M_c / phi(q)^T b_c  (0 when that is 0),
//            g = sigmoid(w . q + beta),  out += g * m.
//
// Update: one CTA per head.  The head's keep words give its evicted slots;
// they are gathered in batches of UB rows (K and V widened to fp32 in shared
// memory), each batch's features phi(P_l k) are computed against the layer's
// projection staged in shared memory, and every thread accumulates its
// D*D/256 entries of the outer-product sum in registers.  The state is read
// and written once per call (the decay applies to every head).
// Read: one CTA per head; the G queries' features share one pass over M_c.
#include "common.cuh"
#include "internal.h"

namespace rkv {

namespace {

constexpr int MT = 256;   // threads per CTA
constexpr int UB = 32;    // evicted rows per batch

__device__ __forceinline__ float phi_of(float y) { return y > 0.0f ? y + 1.0f : expf(y); }

template <int D, typename T>
__device__ __forceinline__ float load_elt(const void *pool, int64_t row, int d) {
    if constexpr (sizeof(T) == 2) {
        return __uint_as_float((uint32_t)__ldg(reinterpret_cast<const unsigned short *>(pool) + row * D + d) << 16);
    } else {
        return __ldg(reinterpret_cast<const float *>(pool) + row * D + d);
    }
}

template <int D, typename T>
__global__ void __launch_bounds__(MT) memory_update_kernel(MemUpdateArgs a) {
    constexpr int EPT = D * D / MT;        // state entries per thread
    constexpr int TPR = D / EPT;           // threads per state row
    extern __shared__ __align__(16) float msm[];
    float *Pt = msm;                       // [D][D + 1] projection transposed (padded: no bank conflicts)
    float *Ks = Pt + D * (D + 1);          // [UB][D]
    float *Vs = Ks + UB * D;               // [UB][D]
    float *Fs = Vs + UB * D;               // [UB][D] features
    int *rows = reinterpret_cast<int *>(Fs + UB * D);   // [UB] physical rows of the batch
    uint32_t *scan = reinterpret_cast<uint32_t *>(rows + UB);  // [40]
    int *misc = reinterpret_cast<int *>(scan + 40);            // [2]
    const int64_t c = blockIdx.x;
    const int tid = threadIdx.x;
    const int l = (int)((c % a.LH) / a.H);
    const int n = clamp_len(__ldg(a.n_pre + c), a.max_pages, nullptr);
    const int W = (n + PAGE - 1) / PAGE;
    const int si = tid / TPR, sj0 = (tid % TPR) * EPT;  // this thread's state row and first column
    float acc[EPT];
#pragma unroll
    for (int e = 0; e < EPT; e++) acc[e] = 0.0f;
    float accb = 0.0f;
    bool staged = false;
    // walk the keep words MT at a time; evicted slots are gathered UB at a time
    for (int w0 = 0; w0 < W; w0 += MT) {
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
        uint32_t before = block_exclusive_scan((uint32_t)__popc(ev), scan, &total);
        for (uint32_t b0 = 0; b0 < total; b0 += UB) {
            // this batch: evicted slots with rank in [b0, b0 + UB)
            uint32_t bits = ev, r = before;
            while (bits) {
                const int j = __ffs(bits) - 1;
                bits &= bits - 1;
                if (r >= b0 && r < b0 + UB) rows[r - b0] = pg * PAGE + j;
                r++;
            }
            const int nb = (int)min((uint32_t)UB, total - b0);
            if (!staged) {
                for (int i = tid; i < D * D; i += MT) Pt[(i % D) * (D + 1) + i / D] = __ldg(a.proj + (int64_t)l * D * D + i);
                staged = true;
            }
            __syncthreads();
            for (int i = tid; i < nb * D; i += MT) {
                const int64_t row = rows[i / D];
                Ks[i] = load_elt<D, T>(a.k_pool, row, i % D);
                Vs[i] = load_elt<D, T>(a.v_pool, row, i % D);
            }
            __syncthreads();
            // features phi(P_l k) of the batch's rows
            for (int o = tid; o < nb * D; o += MT) {
                const int rr = o / D, fi = o % D;
                const float *k = Ks + rr * D;
                float y = 0.0f;
#pragma unroll 8
                for (int d = 0; d < D; d++) y = fmaf(Pt[d * (D + 1) + fi], k[d], y);
                Fs[o] = phi_of(y);
            }
            __syncthreads();
            for (int rr = 0; rr < nb; rr++) {
                const float f = Fs[rr * D + si];
                const float *v = Vs + rr * D + sj0;
#pragma unroll
                for (int e = 0; e < EPT; e++) acc[e] = fmaf(f, v[e], acc[e]);
                if (tid < D) accb += Fs[rr * D + tid];
            }
            __syncthreads();
        }
    }
    // M_c = decay * M_c + sum, b_c = decay * b_c + sum
    float *M = a.M + c * (int64_t)D * D + (int64_t)si * D + sj0;
#pragma unroll
    for (int e = 0; e < EPT; e += 4) {
        float4 m4 = *reinterpret_cast<float4 *>(M + e);
        m4.x = fmaf(a.decay, m4.x, acc[e]);
        m4.y = fmaf(a.decay, m4.y, acc[e + 1]);
        m4.z = fmaf(a.decay, m4.z, acc[e + 2]);
        m4.w = fmaf(a.decay, m4.w, acc[e + 3]);
        *reinterpret_cast<float4 *>(M + e) = m4;
    }
    if (tid < D) a.b[c * D + tid] = fmaf(a.decay, a.b[c * D + tid], accb);
    (void)misc;
}

// Read: per head, for each of its G query rows, features phi(P_l q), the
// normaliser phi^T b, the gate and phi^T M_c, added to the output row.
template <int D, int G>
__global__ void __launch_bounds__(MT) memory_read_kernel(MemReadArgs a) {
    extern __shared__ __align__(16) float msm[];
    float *Pt = msm;                 // [D][D + 1] projection transposed, padded
    float *Qs = Pt + D * (D + 1);    // [G][D]
    float *Fs = Qs + G * D;          // [G][D]
    float *part = Fs + G * D;        // [2][G][D] half sums of phi^T M
    float *red = part + 2 * G * D;   // [G][2][MT/32] warp partials
    const int64_t c = blockIdx.x;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int l = (int)((c % a.LH) / a.H), h = (int)(c % a.H);
    for (int i = tid; i < D * D; i += MT) Pt[(i % D) * (D + 1) + i / D] = __ldg(a.proj + (int64_t)l * D * D + i);
    for (int i = tid; i < G * D; i += MT) Qs[i] = __ldg(a.q + c * G * D + i);
    __syncthreads();
    for (int o = tid; o < G * D; o += MT) {
        const int g = o / D, fi = o % D;
        const float *x = Qs + g * D;
        float y = 0.0f;
#pragma unroll 8
        for (int d = 0; d < D; d++) y = fmaf(Pt[d * (D + 1) + fi], x[d], y);
        Fs[o] = phi_of(y);
    }
    __syncthreads();
    // phi^T M: thread (half, j) sums rows i of its half for column j
    const float *M = a.M + c * (int64_t)D * D;
    {
        constexpr int HALVES = MT / D;   // 2 for D = 128, 4 for D = 64
        const int j = tid % D, hf = tid / D;
        float s[G];
#pragma unroll
        for (int g = 0; g < G; g++) s[g] = 0.0f;
        for (int i = hf; i < D; i += HALVES) {
            const float m = __ldg(M + (int64_t)i * D + j);
#pragma unroll
            for (int g = 0; g < G; g++) s[g] = fmaf(Fs[g * D + i], m, s[g]);
        }
        // fold the halves pairwise into part[0..1]
        if (HALVES == 2) {
#pragma unroll
            for (int g = 0; g < G; g++) part[(hf * G + g) * D + j] = s[g];
        } else {
#pragma unroll
            for (int g = 0; g < G; g++) part[((hf & 1) * G + g) * D + j] = 0.0f;
            __syncthreads();
#pragma unroll
            for (int g = 0; g < G; g++) atomicAdd(&part[((hf & 1) * G + g) * D + j], s[g]);
        }
    }
    // normaliser phi^T b and gate logit w . q + beta per query row
    for (int g = 0; g < G; g++) {
        float den = 0.0f, z = 0.0f;
        for (int i = tid; i < D; i += MT) {
            den = fmaf(Fs[g * D + i], __ldg(a.b + c * D + i), den);
            z = fmaf(__ldg(a.gate_w + ((int64_t)l * a.Hq + h * G + g) * D + i), Qs[g * D + i], z);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            den += __shfl_xor_sync(0xFFFFFFFFu, den, o);
            z += __shfl_xor_sync(0xFFFFFFFFu, z, o);
        }
        if (lane == 0) {
            red[(g * 2) * (MT / 32) + warp] = den;
            red[(g * 2 + 1) * (MT / 32) + warp] = z;
        }
    }
    __syncthreads();
    for (int o = tid; o < G * D; o += MT) {
        const int g = o / D, j = o % D;
        float den = 0.0f, z = __ldg(a.gate_b + (int64_t)l * a.Hq + h * G + g);
        for (int w = 0; w < MT / 32; w++) {
            den += red[(g * 2) * (MT / 32) + w];
            z += red[(g * 2 + 1) * (MT / 32) + w];
        }
        if (den > 0.0f) {
            const float num = part[(0 * G + g) * D + j] + part[(1 * G + g) * D + j];
            const float gate = 1.0f / (1.0f + expf(-z));
            a.out[c * G * D + o] += gate * (num / den);
        }
    }
}

template <int D, typename T>
cudaError_t launch_update_t(const MemUpdateArgs &a, cudaStream_t s) {
    const size_t smem = (size_t)(D * (D + 1) + 3 * UB * D) * 4 + UB * 4 + 40 * 4 + 16;
    auto *k = memory_update_kernel<D, T>;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    k<<<a.C, MT, smem, s>>>(a);
    return cudaGetLastError();
}

template <int D, int G>
cudaError_t launch_read_t(const MemReadArgs &a, cudaStream_t s) {
    const size_t smem = (size_t)(D * (D + 1) + 2 * G * D + 2 * G * D + G * 2 * (MT / 32)) * 4;
    auto *k = memory_read_kernel<D, G>;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    k<<<a.C, MT, smem, s>>>(a);
    return cudaGetLastError();
}

}  // namespace

bool memory_supported(int D, int G) { return (D == 64 || D == 128) && G >= 1 && G <= 8; }

cudaError_t launch_memory_update(const MemUpdateArgs &a, int dtype, int D, cudaStream_t s) {
    if (a.C == 0) return cudaSuccess;
    if (D == 128) return dtype == RKV_BF16 ? launch_update_t<128, uint16_t>(a, s) : launch_update_t<128, float>(a, s);
    if (D == 64) return dtype == RKV_BF16 ? launch_update_t<64, uint16_t>(a, s) : launch_update_t<64, float>(a, s);
    return cudaErrorNotSupported;
}

cudaError_t launch_memory_read(const MemReadArgs &a, int D, int G, cudaStream_t s) {
    if (a.C == 0) return cudaSuccess;
#define RKV_MEM_G(DD)                                        \
    switch (G) {                                             \
        case 1: return launch_read_t<DD, 1>(a, s);           \
        case 2: return launch_read_t<DD, 2>(a, s);           \
        case 3: return launch_read_t<DD, 3>(a, s);           \
        case 4: return launch_read_t<DD, 4>(a, s);           \
        case 5: return launch_read_t<DD, 5>(a, s);           \
        case 6: return launch_read_t<DD, 6>(a, s);           \
        case 7: return launch_read_t<DD, 7>(a, s);           \
        case 8: return launch_read_t<DD, 8>(a, s);           \
        default: return cudaErrorNotSupported;               \
    }
    if (D == 128) { RKV_MEM_G(128) }
    if (D == 64) { RKV_MEM_G(64) }
#undef RKV_MEM_G
    return cudaErrorNotSupported;
}

}  // namespace rkv
