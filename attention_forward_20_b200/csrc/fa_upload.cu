// Host-to-device copies of the small per-call tables (cumulative sequence
// offsets, the varlen work table) that stay valid inside a captured CUDA
// graph.  Outside capture a pageable cudaMemcpyAsync does the job: the driver
// stages the source before the call returns.  Under stream capture that copy
// would be recorded with a pointer to host memory that the caller frees or
// reuses before the graph runs, so the bytes travel instead in the launch
// parameters of small copy kernels, which the graph keeps by value.
#include "fa_params.h"

#include <cstring>

namespace fa {
namespace {

constexpr int kChunk = 4000;  // payload bytes per launch (kernel parameters stay below 4 KB)

struct Payload {
    unsigned char bytes[kChunk];
};

__global__ void __launch_bounds__(256) fa_param_copy_kernel(unsigned char* dst, int n, const Payload pl) {
    for (int i = threadIdx.x; i < n; i += blockDim.x) dst[i] = pl.bytes[i];
}

}  // namespace

cudaError_t upload_async(void* dst, const void* src, size_t bytes, cudaStream_t stream) {
    if (bytes == 0) return cudaSuccess;
    cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
    cudaError_t e = cudaStreamIsCapturing(stream, &cap);
    if (e != cudaSuccess) return e;
    if (cap == cudaStreamCaptureStatusNone)
        return cudaMemcpyAsync(dst, src, bytes, cudaMemcpyHostToDevice, stream);
    const unsigned char* s = static_cast<const unsigned char*>(src);
    unsigned char* d = static_cast<unsigned char*>(dst);
    for (size_t off = 0; off < bytes; off += kChunk) {
        const int n = static_cast<int>(bytes - off < kChunk ? bytes - off : kChunk);
        Payload pl;
        std::memcpy(pl.bytes, s + off, n);
        fa_param_copy_kernel<<<1, 256, 0, stream>>>(d + off, n, pl);
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

}  // namespace fa
