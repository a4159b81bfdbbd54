// CUDA-core attention forward: exact fp32 FFMA for Q·Kᵀ and P·V, online
// softmax in natural-exp units with expf.  It serves fp32 inputs (whose
// 1e-4 output tolerance rules out TF32 tensor cores) and head dims that the
// tcgen05 kernel does not take (up to 256).
//
// The online-softmax recurrence is the FlashAttention algorithm named on the
// aclnnFlashAttentionScore page ("功能描述": the operator computes
// self-attention with the FlashAttention algorithm); the quantities it
// produces are those of the forward and sink formulas on the
// aclnnFlashAttentionVarLenScoreV5 page.
//
// CTA = 128 threads = 4 warps for 32 query rows (8 rows per warp).  For each
// 32-key tile staged in shared memory, lane j of a warp scores key j against
// one row, the warp reduces the row max and sum with shuffles, and every lane
// accumulates its D/32 output columns.
#include "fa_params.h"

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <math_constants.h>

namespace fa {
namespace {

constexpr int kRows = 32;  // query rows per CTA
constexpr int kKeys = 32;  // keys per tile (one per lane)
constexpr int kWarps = 4;
constexpr int kRowsPerWarp = kRows / kWarps;

__device__ __forceinline__ float to_f(float x) { return x; }
__device__ __forceinline__ float to_f(__half x) { return __half2float(x); }
__device__ __forceinline__ float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T> __device__ __forceinline__ T from_f(float x);
template <> __device__ __forceinline__ float from_f<float>(float x) { return x; }
template <> __device__ __forceinline__ __half from_f<__half>(float x) { return __float2half_rn(x); }
template <> __device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float x) { return __float2bfloat16_rn(x); }

__device__ __forceinline__ float warp_max(float x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
    return x;
}
__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

template <typename T, int DMAX>
__global__ void __launch_bounds__(kWarps * 32) fa_fwd_simt_kernel(const FaParams p) {
    extern __shared__ float smem[];
    constexpr int ld = DMAX + 1;  // odd row pitch: lane-strided reads hit distinct banks
    constexpr int kCols = DMAX / 32;
    float* sQ = smem;
    float* sK = sQ + kRows * ld;
    float* sV = sK + kKeys * ld;

    const int b = blockIdx.z, n = blockIdx.y, i0 = blockIdx.x * kRows;
    const int nk = n / p.group;
    int64_t q_off = 0, kv_off = 0;
    int q_len = p.Sq, kv_len = p.Skv;
    if (p.varlen) {
        q_off = p.cu_q[b];
        q_len = (int)(p.cu_q[b + 1] - q_off);
        kv_off = p.cu_kv[b];
        kv_len = (int)(p.cu_kv[b + 1] - kv_off);
    }
    if (i0 >= q_len) return;

    const T* Q = static_cast<const T*>(p.q) + b * p.q_b + n * p.q_n;
    const T* K = static_cast<const T*>(p.k) + b * p.k_b + nk * p.k_n;
    const T* V = static_cast<const T*>(p.v) + b * p.v_b + nk * p.v_n;
    const int D = p.D, Dv = p.Dv;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    for (int idx = tid; idx < kRows * D; idx += blockDim.x) {
        const int r = idx / D, d = idx % D, i = i0 + r;
        sQ[r * ld + d] = (i < q_len) ? to_f(Q[(q_off + i) * p.q_s + d]) : 0.f;
    }

    float m[kRowsPerWarp], l[kRowsPerWarp], acc[kRowsPerWarp][kCols];
#pragma unroll
    for (int rr = 0; rr < kRowsPerWarp; ++rr) {
        m[rr] = -CUDART_INF_F;
        l[rr] = 0.f;
#pragma unroll
        for (int t = 0; t < kCols; ++t) acc[rr][t] = 0.f;
    }

    float slope = 0.f;
    if (p.pse_type == 2) slope = static_cast<const float*>(p.pse)[b * p.pse_b + n * p.pse_n];
    const T* pse = (p.pse_type == 1) ? static_cast<const T*>(p.pse) + b * p.pse_b + n * p.pse_n : nullptr;
    const uint8_t* mask = p.mask_on ? p.mask + b * p.mask_b + n * p.mask_n : nullptr;

    const int i1 = min(q_len, i0 + kRows) - 1;
    const int j_lo = max(0, i0 - p.pre);
    const int j_hi = min(kv_len - 1, i1 + p.next);
    for (int j0 = (j_lo / kKeys) * kKeys; j0 <= j_hi; j0 += kKeys) {
        __syncthreads();
        for (int idx = tid; idx < kKeys * D; idx += blockDim.x) {
            const int r = idx / D, d = idx % D, j = j0 + r;
            sK[r * ld + d] = (j < kv_len) ? to_f(K[(kv_off + j) * p.k_s + d]) : 0.f;
        }
        for (int idx = tid; idx < kKeys * Dv; idx += blockDim.x) {
            const int r = idx / Dv, d = idx % Dv, j = j0 + r;
            sV[r * ld + d] = (j < kv_len) ? to_f(V[(kv_off + j) * p.v_s + d]) : 0.f;
        }
        __syncthreads();
        const int j = j0 + lane;
#pragma unroll
        for (int rr = 0; rr < kRowsPerWarp; ++rr) {
            const int r = warp * kRowsPerWarp + rr, i = i0 + r;
            float s = 0.f;
            for (int d = 0; d < D; ++d) s = fmaf(sQ[r * ld + d], sK[lane * ld + d], s);
            bool keep = i < q_len && j < kv_len && (j - i >= -p.pre) && (j - i <= p.next);
            if (keep && mask) keep = mask[(int64_t)i * p.mask_i + j] == 0;
            float x = s * p.scale;
            if (keep && pse) x += to_f(pse[(int64_t)i * p.pse_i + j]);
            if (p.pse_type == 2) x -= slope * fabsf((float)(i - j));
            x = keep ? x : -CUDART_INF_F;
            const float m_new = fmaxf(m[rr], warp_max(x));
            if (m_new == -CUDART_INF_F) continue;  // nothing kept yet in this row
            const float alpha = expf(m[rr] - m_new);
            const float pj = keep ? expf(x - m_new) : 0.f;
            l[rr] = l[rr] * alpha + warp_sum(pj);
#pragma unroll
            for (int t = 0; t < kCols; ++t) acc[rr][t] *= alpha;
            for (int jj = 0; jj < kKeys; ++jj) {
                const float pv = __shfl_sync(0xffffffffu, pj, jj);
#pragma unroll
                for (int t = 0; t < kCols; ++t) {
                    const int d = lane + 32 * t;
                    if (d < Dv) acc[rr][t] = fmaf(pv, sV[jj * ld + d], acc[rr][t]);
                }
            }
            m[rr] = m_new;
        }
    }

    T* O = static_cast<T*>(p.o) + b * p.o_b + n * p.o_n;
#pragma unroll
    for (int rr = 0; rr < kRowsPerWarp; ++rr) {
        const int i = i0 + warp * kRowsPerWarp + rr;
        if (i >= q_len) continue;
        float mf = m[rr], lf = l[rr], oscale;
        if (p.has_sink) {
            // sink formula: m = max(sink, max S); denominator gains e^(sink - m)
            const float sk = p.sink[n];
            mf = fmaxf(m[rr], sk);
            const float a = (m[rr] == -CUDART_INF_F) ? 0.f : expf(m[rr] - mf);
            lf = l[rr] * a + expf(sk - mf);
            oscale = a / lf;
        } else {
            oscale = lf > 0.f ? 1.f / lf : 0.f;
        }
        T* orow = O + (q_off + i) * p.o_s;
#pragma unroll
        for (int t = 0; t < kCols; ++t) {
            const int d = lane + 32 * t;
            if (d < Dv) orow[d] = from_f<T>(acc[rr][t] * oscale);
        }
        const int64_t so = b * p.st_b + n * p.st_n + (q_off + i) * p.st_s;
        if (lane < 8) {
            p.smax[so + lane] = mf;
            p.ssum[so + lane] = lf;
        }
    }
}

template <typename T, int DMAX>
cudaError_t launch_t(const FaParams& p, cudaStream_t stream) {
    const size_t smem = size_t(kRows + 2 * kKeys) * (DMAX + 1) * sizeof(float);
    auto kern = fa_fwd_simt_kernel<T, DMAX>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const dim3 grid((p.Sq + kRows - 1) / kRows, p.Nq, p.B);
    if (grid.x == 0) return cudaSuccess;  // every sequence is empty
    kern<<<grid, kWarps * 32, smem, stream>>>(p);
    return cudaGetLastError();
}

template <typename T>
cudaError_t launch_d(const FaParams& p, cudaStream_t stream) {
    const int dmax = p.D > p.Dv ? p.D : p.Dv;
    if (dmax <= 64) return launch_t<T, 64>(p, stream);
    if (dmax <= 128) return launch_t<T, 128>(p, stream);
    return launch_t<T, 256>(p, stream);
}

}  // namespace

cudaError_t launch_simt(const FaParams& p, cudaStream_t stream) {
    switch (p.dtype) {
        case 0: return launch_d<float>(p, stream);
        case 1: return launch_d<__half>(p, stream);
        default: return launch_d<__nv_bfloat16>(p, stream);
    }
}

}  // namespace fa
