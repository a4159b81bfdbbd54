// fa_lse_merge: combines attention results of the same queries over disjoint
// key sets, each given as (out_k, m_k, l_k) with out_k normalised by l_k and
// m_k, l_k the row's max and sum in natural-log units (the statistics the
// forward writes; aclnnFlashAttentionScore / aclnnFlashAttentionVarLenScoreV5,
// softmaxMax / softmaxSum).  With M = max_k m_k (and the sink),
//   l   = sum_k l_k e^(m_k - M) + e^(sink - M)
//   out = sum_k l_k e^(m_k - M) out_k / l
// which is the forward over the union of the key sets: the online-softmax
// update applied to whole partial results.  A partial row with no key
// (l_k = 0) contributes nothing; a row with none at all gets out = 0,
// m = -inf, l = 0 (with a sink: m = sink, l = 1).
#include "fa_params.h"
#include "sm100_ptx.cuh"

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <math_constants.h>

#include <type_traits>

namespace fa {
namespace {

constexpr int kThreads = 256;

__device__ __forceinline__ float to_f(float x) { return x; }
__device__ __forceinline__ float to_f(__half x) { return __half2float(x); }
__device__ __forceinline__ float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }
template <typename T> __device__ __forceinline__ T from_f(float x);
template <> __device__ __forceinline__ float from_f<float>(float x) { return x; }
template <> __device__ __forceinline__ __half from_f<__half>(float x) { return __float2half_rn(x); }
template <> __device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float x) { return __float2bfloat16_rn(x); }

// two packed 16-bit values (low half first) as floats
template <typename T>
__device__ __forceinline__ float2 unpack2(uint32_t w) {
    if constexpr (std::is_same<T, __nv_bfloat16>::value) {
        return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
    } else {
        __half2 h;
        memcpy(&h, &w, sizeof(h));
        return __half22float2(h);
    }
}

// one thread per (row, group of 8 output columns)
template <typename T>
__global__ void __launch_bounds__(kThreads, 4) fa_lse_merge_kernel(const MergeParams mp) {
    const int groups = (mp.Dv + 7) / 8;
    const int64_t idx = static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x;
    const int64_t total = static_cast<int64_t>(mp.B) * mp.N * mp.S * groups;
    if (idx >= total) return;
    const int g = static_cast<int>(idx % groups);
    int64_t r = idx / groups;
    const int s = static_cast<int>(r % mp.S);
    r /= mp.S;
    const int n = static_cast<int>(r % mp.N);
    const int b = static_cast<int>(r / mp.N);

    float m = mp.sink ? mp.sink[n] : -CUDART_INF_F;
    for (int k = 0; k < mp.count; ++k) {
        const int64_t so = b * mp.st_b[k] + n * mp.st_n[k] + s * mp.st_s[k];
        if (mp.ssum[k][so] > 0.f) m = fmaxf(m, mp.smax[k][so]);
    }
    float l = 0.f, acc[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] = 0.f;
    const int d0 = g * 8;
    for (int k = 0; k < mp.count; ++k) {
        const int64_t so = b * mp.st_b[k] + n * mp.st_n[k] + s * mp.st_s[k];
        const float lk = mp.ssum[k][so];
        if (!(lk > 0.f)) continue;
        const float wk = lk * expf(mp.smax[k][so] - m);
        l += wk;
        const T* o = static_cast<const T*>(mp.out[k]) + b * mp.o_b[k] + n * mp.o_n[k] + s * mp.o_s[k] + d0;
        if (sizeof(T) == 2 && d0 + 8 <= mp.Dv && (reinterpret_cast<uintptr_t>(o) & 15u) == 0) {
            const uint4 u = __ldg(reinterpret_cast<const uint4*>(o));  // the 8 columns in one load
            const uint32_t w4[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float2 f = unpack2<T>(w4[e]);
                acc[2 * e] = fmaf(wk, f.x, acc[2 * e]);
                acc[2 * e + 1] = fmaf(wk, f.y, acc[2 * e + 1]);
            }
        } else {
#pragma unroll
            for (int e = 0; e < 8; ++e)
                if (d0 + e < mp.Dv) acc[e] = fmaf(wk, to_f(o[e]), acc[e]);
        }
    }
    if (mp.sink) l += expf(mp.sink[n] - m);
    const float inv = l > 0.f ? 1.f / l : 0.f;
    T* o = static_cast<T*>(mp.res_o) + b * mp.r_o_b + n * mp.r_o_n + s * mp.r_o_s + d0;
    if (sizeof(T) == 2 && d0 + 8 <= mp.Dv && (reinterpret_cast<uintptr_t>(o) & 15u) == 0) {
        uint32_t w4[4];
#pragma unroll
        for (int e = 0; e < 4; ++e)
            w4[e] = std::is_same<T, __nv_bfloat16>::value ? ptx::pack_bf16x2(acc[2 * e] * inv, acc[2 * e + 1] * inv)
                                                          : ptx::pack_f16x2(acc[2 * e] * inv, acc[2 * e + 1] * inv);
        *reinterpret_cast<uint4*>(o) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
    } else {
#pragma unroll
        for (int e = 0; e < 8; ++e)
            if (d0 + e < mp.Dv) o[e] = from_f<T>(acc[e] * inv);
    }
    if (g == 0) {
        const int64_t so = b * mp.r_st_b + n * mp.r_st_n + s * mp.r_st_s;
        const float mo = l > 0.f ? m : -CUDART_INF_F;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            mp.res_max[so + e] = mo;
            mp.res_sum[so + e] = l;
        }
    }
}

template <typename T>
cudaError_t launch_t(const MergeParams& mp, cudaStream_t stream) {
    const int64_t total = static_cast<int64_t>(mp.B) * mp.N * mp.S * ((mp.Dv + 7) / 8);
    if (total == 0) return cudaSuccess;
    fa_lse_merge_kernel<T><<<static_cast<unsigned>((total + kThreads - 1) / kThreads), kThreads, 0, stream>>>(mp);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_lse_merge(const MergeParams& mp, cudaStream_t stream) {
    switch (mp.dtype) {
        case 0: return launch_t<float>(mp, stream);
        case 1: return launch_t<__half>(mp, stream);
        default: return launch_t<__nv_bfloat16>(mp, stream);
    }
}

}  // namespace fa
