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
// CTA = 8 warps, one query row per warp.  Keys go in tiles of kKeys (128, or
// 64 when the head dim exceeds 128) staged in shared memory as fp32; lane l
// scores keys l, l+32, ... (independent FMA chains over the head dim), the
// warp reduces the row max once per tile, keeps its share of the row sum in
// each lane (reduced once at the end), writes P to shared memory and
// accumulates its output columns d = l + 32t over the tile's keys with four
// interleaved partial sums.
#include "fa_params.h"

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <math_constants.h>

namespace fa {
namespace {

constexpr int kWarps = 8;
constexpr int kRows = kWarps;  // query rows per CTA, one per warp

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

template <int DMAX>
struct SimtCfg {
    static constexpr int kKeys = DMAX <= 128 ? 128 : 64;  // keys per tile
    static constexpr int kPerLane = kKeys / 32;
    static constexpr int kCols = DMAX / 32;               // output columns per lane
    static constexpr int ld = DMAX + 1;                   // odd pitch: lane-strided rows hit distinct banks
    static constexpr size_t kSmemBytes = size_t(2 * kKeys * ld + kRows * ld + kRows * kKeys) * sizeof(float);
};

template <typename T, int DMAX>
__global__ void __launch_bounds__(kWarps * 32, 1) fa_fwd_simt_kernel(const FaParams p) {
    using C = SimtCfg<DMAX>;
    constexpr int kKeys = C::kKeys, kPerLane = C::kPerLane, kCols = C::kCols, ld = C::ld;
    extern __shared__ float smem[];
    float* sK = smem;                  // [kKeys][ld]
    float* sV = sK + kKeys * ld;       // [kKeys][ld]
    float* sQ = sV + kKeys * ld;       // [kRows][ld]
    float* sP = sQ + kRows * ld;       // [kRows][kKeys]

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
    // queryRope / keyRope: columns D .. D+Dr-1 of the dot product
    const T* QR = p.Dr ? static_cast<const T*>(p.qr) + b * p.qr_b + n * p.qr_n : nullptr;
    const T* KR = p.Dr ? static_cast<const T*>(p.kr) + b * p.kr_b + nk * p.kr_n : nullptr;
    const int D = p.D, Dv = p.Dv, Dqk = p.D + p.Dr;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int i = i0 + warp;  // this warp's query row
    const bool row_ok = i < q_len;

    // Q rows, zero-padded to DMAX (the dot products run over DMAX)
    for (int idx = tid; idx < kRows * DMAX; idx += blockDim.x) {
        const int r = idx / DMAX, d = idx % DMAX, ii = i0 + r;
        float x = 0.f;
        if (ii < q_len && d < D) x = to_f(Q[(q_off + ii) * p.q_s + d]);
        else if (ii < q_len && d < Dqk) x = to_f(QR[(q_off + ii) * p.qr_s + (d - D)]);
        sQ[r * ld + d] = x;
    }

    float slope = 0.f;
    if (p.pse_type == 2) slope = static_cast<const float*>(p.pse)[b * p.pse_b + n * p.pse_n];
    int pse_cols = 0;
    const T* pse = (p.pse_type == 1 && row_ok) ? pse_row_ptr<T>(p, b, n, q_len, kv_len, i, &pse_cols) : nullptr;
    const uint8_t* mask = p.mask_on ? p.mask + b * p.mask_b + n * p.mask_n : nullptr;

    float m_run = -CUDART_INF_F, l_lane = 0.f;
    float acc[4][kCols];
#pragma unroll
    for (int g = 0; g < 4; ++g)
#pragma unroll
        for (int t = 0; t < kCols; ++t) acc[g][t] = 0.f;

    // keys any row of the CTA keeps under the band
    const int i1 = min(q_len, i0 + kRows) - 1;
    const int j_lo = max(0, i0 - p.pre);
    const int j_hi = min(kv_len - 1, i1 + p.next);
    const float* q = sQ + warp * ld;
    float* pw = sP + warp * kKeys;
    for (int j0 = (j_lo / kKeys) * kKeys; j0 <= j_hi; j0 += kKeys) {
        __syncthreads();
        // K/V tile: batches of kBatch elements per thread, all loads of a batch
        // in flight before their shared-memory stores
        constexpr int kPerThread = kKeys * DMAX / (kWarps * 32);
        constexpr int kBatch = 16;
#pragma unroll 1
        for (int u = 0; u < kPerThread; u += kBatch) {
            float kk[kBatch], vv[kBatch];
#pragma unroll
            for (int e = 0; e < kBatch; ++e) {
                const int idx = tid + (u + e) * (kWarps * 32);
                const int r = idx / DMAX, d = idx % DMAX, j = j0 + r;
                const bool in = j < kv_len;
                kk[e] = (in && d < D) ? to_f(K[(kv_off + j) * p.k_s + d])
                        : (in && d < Dqk) ? to_f(KR[(kv_off + j) * p.kr_s + (d - D)]) : 0.f;
                vv[e] = (in && d < Dv) ? to_f(V[(kv_off + j) * p.v_s + d]) : 0.f;
            }
#pragma unroll
            for (int e = 0; e < kBatch; ++e) {
                const int idx = tid + (u + e) * (kWarps * 32);
                const int r = idx / DMAX, d = idx % DMAX;
                sK[r * ld + d] = kk[e];
                sV[r * ld + d] = vv[e];
            }
        }
        __syncthreads();

        // scores of keys j0 + lane + 32m
        float x[kPerLane];
#pragma unroll
        for (int mm = 0; mm < kPerLane; ++mm) x[mm] = 0.f;
#pragma unroll 8
        for (int d = 0; d < DMAX; ++d) {
            const float qd = q[d];
#pragma unroll
            for (int mm = 0; mm < kPerLane; ++mm) x[mm] = fmaf(qd, sK[(lane + 32 * mm) * ld + d], x[mm]);
        }
        float tile_max = -CUDART_INF_F;
#pragma unroll
        for (int mm = 0; mm < kPerLane; ++mm) {
            const int j = j0 + lane + 32 * mm;
            bool keep = row_ok && j < kv_len && (j - i >= -p.pre) && (j - i <= p.next);
            if (keep && mask) keep = mask[(int64_t)i * p.mask_i + j] == 0;
            float v = x[mm] * p.scale;
            if (keep && pse && j < pse_cols) v += to_f(pse[j]);
            if (p.pse_type == 2) v -= slope * fabsf((float)(i - j - p.alibi_delta));
            x[mm] = keep ? v : -CUDART_INF_F;
            tile_max = fmaxf(tile_max, x[mm]);
        }
        const float m_new = fmaxf(m_run, warp_max(tile_max));
        if (m_new == -CUDART_INF_F) continue;  // nothing kept in this row yet (warp-uniform)
        const float alpha = expf(m_run - m_new);  // 0 when m_run is -inf
        m_run = m_new;
        float psum = 0.f;
#pragma unroll
        for (int mm = 0; mm < kPerLane; ++mm) {
            const float pj = expf(x[mm] - m_new);  // 0 for excluded keys
            psum += pj;
            pw[lane + 32 * mm] = pj;
        }
        l_lane = l_lane * alpha + psum;
        __syncwarp();
#pragma unroll
        for (int g = 0; g < 4; ++g)
#pragma unroll
            for (int t = 0; t < kCols; ++t) acc[g][t] *= alpha;
        // O += P V over the tile: four interleaved partial sums per column
#pragma unroll 2
        for (int jj = 0; jj < kKeys; jj += 4) {
#pragma unroll
            for (int g = 0; g < 4; ++g) {
                const float pj = pw[jj + g];
#pragma unroll
                for (int t = 0; t < kCols; ++t)
                    acc[g][t] = fmaf(pj, sV[(jj + g) * ld + lane + 32 * t], acc[g][t]);
            }
        }
        __syncwarp();
    }

    if (!row_ok) return;
    const float l = warp_sum(l_lane);
    float mf = m_run, lf = l, oscale;
    if (p.has_sink) {
        // sink formula: m = max(sink, max S); denominator gains e^(sink - m)
        const float sk = p.sink[n];
        mf = fmaxf(m_run, sk);
        const float a = (m_run == -CUDART_INF_F) ? 0.f : expf(m_run - mf);
        lf = l * a + expf(sk - mf);
        oscale = a / lf;
    } else {
        oscale = lf > 0.f ? 1.f / lf : 0.f;
    }
    T* orow = static_cast<T*>(p.o) + b * p.o_b + n * p.o_n + (q_off + i) * p.o_s;
#pragma unroll
    for (int t = 0; t < kCols; ++t) {
        const int d = lane + 32 * t;
        if (d < Dv) orow[d] = from_f<T>(((acc[0][t] + acc[1][t]) + (acc[2][t] + acc[3][t])) * oscale);
    }
    const int64_t so = b * p.st_b + n * p.st_n + (q_off + i) * p.st_s;
    if (lane < 8) {
        p.smax[so + lane] = mf;
        p.ssum[so + lane] = lf;
    }
}

template <typename T, int DMAX>
cudaError_t launch_t(const FaParams& p, cudaStream_t stream) {
    const size_t smem = SimtCfg<DMAX>::kSmemBytes;
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
    const int dqk = p.D + p.Dr;
    const int dmax = dqk > p.Dv ? dqk : p.Dv;
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
