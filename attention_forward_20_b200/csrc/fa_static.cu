// fa_fwd_varlen_static: the packed-TND (varlen) forward for callers that
// cannot allocate device memory.
//
// The ordinary varlen call keeps its per-call scratch (the cumulative
// sequence offsets and the list of (sequence, query block) work items) in a
// workspace that the caller allocates.  Code that must not call cudaMalloc --
// for example code that runs while a stream is being captured, or a runtime
// whose device memory is fully handed out up front -- cannot provide one.
// This entry point keeps that scratch in a fixed file-scope device array
// instead, so it allocates nothing: no cudaMalloc / cudaFree, no workspace,
// no host heap (a static host staging buffer holds the table on its way to
// the device).
//
// Limit: at most kStaticMaxSeqs sequences; larger calls are rejected with
// FA_ERR_INNER_NULLPTR before any device work.  With the T <= 1M tokens that
// every call obeys, that bounds the work items (one per 256-row query block of
// each sequence) at 1M/256 + kStaticMaxSeqs = kStaticMaxBlocks.  The device
// array (kScratchBytes, about 130 KB) lives on every GPU that loads the
// library until the process exits.
//
// The array is shared by every call: each call overwrites the ticket counter
// (with zero), the offsets and the table it reads, so nothing has to start at
// zero, but two calls whose work overlaps on the GPU (different streams, or
// different host threads without ordering between them) race on it.
#include "fa_fwd.h"
#include "fa_params.h"

#include <algorithm>
#include <cmath>
#include <cstring>
#include <mutex>

namespace {

constexpr int64_t kStaticMaxSeqs = 2048;
constexpr int64_t kStaticMaxBlocks = (int64_t(1) << 20) / 256 + kStaticMaxSeqs;
constexpr size_t kCuOffset = 256;  // [0, 256): the tcgen05 kernel's ticket counter
constexpr size_t kMaxCuBytes = 2 * (kStaticMaxSeqs + 1) * sizeof(int64_t);
constexpr size_t kScratchBytes = ((kCuOffset + kMaxCuBytes + 255) & ~size_t(255)) + kStaticMaxBlocks * sizeof(int4);
constexpr int kMaxDevices = 64;

// Offset of the work table for a call with nSeq sequences: right after that
// call's offsets, 256-byte aligned (at most kScratchBytes - the table).
size_t table_offset(int64_t nSeq) {
    return (kCuOffset + 2 * (nSeq + 1) * sizeof(int64_t) + 255) & ~size_t(255);
}

// The scratch.  In host code this name is only a stand-in for the symbol, not
// a device address; host code must use the address from cudaGetSymbolAddress.
static __device__ __align__(256) unsigned char g_static_scratch[kScratchBytes];

// Host staging for the offsets and table (static storage, one caller at a time).
static unsigned char g_host_stage[kScratchBytes];
static fa::VarlenEntry g_sort_stage[kStaticMaxBlocks];
static std::mutex g_stage_mutex;

static void* g_scratch_ptr[kMaxDevices];
static std::mutex g_scratch_mutex[kMaxDevices];

// Device address of the scratch on the current device.  A successful lookup
// is kept for the device; a failed one (a transient error, or a first call
// made while a stream is being captured) is not, so the next call tries again.
cudaError_t scratch_address(void** out) {
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_scratch_mutex[dev]);
    if (g_scratch_ptr[dev] == nullptr) {
        void* ptr = nullptr;
        e = cudaGetSymbolAddress(&ptr, g_static_scratch);
        if (e != cudaSuccess) return e;
        g_scratch_ptr[dev] = ptr;
    }
    *out = g_scratch_ptr[dev];
    return cudaSuccess;
}

bool tnd_view(const fa_tensor* t, int64_t* T, int64_t* N, int64_t* D, int64_t* st, int64_t* sn) {
    if (t->ndim != 3 || t->strides[2] != 1) return false;
    for (int i = 0; i < 3; ++i)
        if (t->shape[i] < 1 || t->strides[i] < 0) return false;
    *T = t->shape[0];
    *N = t->shape[1];
    *D = t->shape[2];
    *st = t->strides[0];
    *sn = t->strides[1];
    return true;
}

}  // namespace

extern "C" fa_status fa_fwd_varlen_static(
    const fa_tensor* query, const fa_tensor* key, const fa_tensor* value, const fa_tensor* sink,
    const int64_t* actualSeqQLen, const int64_t* actualSeqKvLen, int64_t nSeq,
    double scaleValue, int64_t preTokens, int64_t nextTokens, int64_t headNum,
    const char* softmaxOutLayout, const fa_tensor* softmaxMax, const fa_tensor* softmaxSum,
    const fa_tensor* attentionOut, void* stream) {
    // ---- the same argument rules as fa_fwd_get_workspace_size with "TND" ----
    if (!query || !key || !value || !softmaxMax || !softmaxSum || !attentionOut || !actualSeqQLen ||
        !actualSeqKvLen)
        return FA_ERR_PARAM_NULLPTR;
    if (!query->data || !key->data || !value->data || !softmaxMax->data || !softmaxSum->data ||
        !attentionOut->data || (sink && !sink->data))
        return FA_ERR_PARAM_NULLPTR;
    const char* sol = softmaxOutLayout ? softmaxOutLayout : "";
    const bool same_as_input = std::strcmp(sol, "same_as_input") == 0;
    if (!same_as_input && sol[0] != '\0') return FA_ERR_PARAM_INVALID;
    const int32_t dt = query->dtype;
    if ((dt != FA_F32 && dt != FA_F16 && dt != FA_BF16) || key->dtype != dt || value->dtype != dt ||
        attentionOut->dtype != dt || softmaxMax->dtype != FA_F32 || softmaxSum->dtype != FA_F32 ||
        (sink && sink->dtype != FA_F32))
        return FA_ERR_PARAM_INVALID;
    if (!std::isfinite(scaleValue) || scaleValue == 0.0 || headNum < 1 || headNum > 256) return FA_ERR_INNER_NULLPTR;
    if (nSeq < 1 || nSeq > kStaticMaxSeqs) return FA_ERR_INNER_NULLPTR;  // scratch limit

    int64_t Tq, Nq, D, qst, qsn, Tk, Nk, Dk, kst, ksn, Tv, Nv, Dv, vst, vsn, To, No, Do, ost, osn;
    if (!tnd_view(query, &Tq, &Nq, &D, &qst, &qsn) || !tnd_view(key, &Tk, &Nk, &Dk, &kst, &ksn) ||
        !tnd_view(value, &Tv, &Nv, &Dv, &vst, &vsn) || !tnd_view(attentionOut, &To, &No, &Do, &ost, &osn))
        return FA_ERR_INNER_NULLPTR;
    if (Nq != headNum || Nk != Nv || Nq % Nk != 0 || Dk != D || Tv != Tk || Dv > D || D > 256 ||
        To != Tq || No != Nq || Do != Dv || Tq > (1 << 20) || Tk > (1 << 20))
        return FA_ERR_INNER_NULLPTR;
    int64_t max_q = 0, max_kv = 0, prev_q = 0, prev_k = 0;
    for (int64_t b = 0; b < nSeq; ++b) {
        if (actualSeqQLen[b] < prev_q || actualSeqKvLen[b] < prev_k) return FA_ERR_INNER_NULLPTR;
        max_q = std::max(max_q, actualSeqQLen[b] - prev_q);
        max_kv = std::max(max_kv, actualSeqKvLen[b] - prev_k);
        prev_q = actualSeqQLen[b];
        prev_k = actualSeqKvLen[b];
    }
    if (prev_q != Tq || prev_k != Tk) return FA_ERR_INNER_NULLPTR;
    for (const fa_tensor* st : {softmaxMax, softmaxSum}) {
        const int64_t a = same_as_input ? Tq : Nq, c = same_as_input ? Nq : Tq;
        if (st->ndim != 3 || st->shape[0] != a || st->shape[1] != c || st->shape[2] != 8 || st->strides[2] != 1 ||
            st->strides[0] < 0 || st->strides[1] < 0)
            return FA_ERR_INNER_NULLPTR;
    }
    if (softmaxMax->strides[0] != softmaxSum->strides[0] || softmaxMax->strides[1] != softmaxSum->strides[1])
        return FA_ERR_INNER_NULLPTR;
    if (sink && (sink->ndim != 1 || sink->shape[0] != Nq || sink->strides[0] != 1)) return FA_ERR_INNER_NULLPTR;
    const int64_t lim = max_q + max_kv + 1;
    const int64_t pre_c = std::min(std::max(preTokens, -lim), lim);
    const int64_t next_c = std::min(std::max(nextTokens, -lim), lim);
    if (pre_c + next_c < 0) return FA_ERR_INNER_NULLPTR;

    // ---- parameter block ------------------------------------------------------
    fa::FaParams p;
    std::memset(&p, 0, sizeof(p));
    p.q = query->data; p.k = key->data; p.v = value->data; p.o = attentionOut->data;
    p.smax = static_cast<float*>(softmaxMax->data);
    p.ssum = static_cast<float*>(softmaxSum->data);
    p.sink = sink ? static_cast<const float*>(sink->data) : nullptr;
    p.q_s = qst; p.q_n = qsn; p.k_s = kst; p.k_n = ksn; p.v_s = vst; p.v_n = vsn; p.o_s = ost; p.o_n = osn;
    if (same_as_input) { p.st_s = softmaxMax->strides[0]; p.st_n = softmaxMax->strides[1]; }
    else { p.st_n = softmaxMax->strides[0]; p.st_s = softmaxMax->strides[1]; }
    p.B = (int32_t)nSeq; p.Nq = (int32_t)Nq; p.Nkv = (int32_t)Nk; p.group = (int32_t)(Nq / Nk);
    p.D = (int32_t)D; p.Dv = (int32_t)Dv; p.Sq = (int32_t)max_q; p.Skv = (int32_t)max_kv;
    p.pre = (int32_t)pre_c; p.next = (int32_t)next_c;
    p.scale = (float)scaleValue;
    p.scale_log2 = (float)(std::fabs(scaleValue) * 1.4426950408889634);
    p.neg_scale = scaleValue < 0 ? 1 : 0;
    p.has_sink = sink ? 1 : 0;
    p.varlen = 1;
    p.dtype = dt;
    p.Tq = (int32_t)Tq; p.Tkv = (int32_t)Tk;
    auto aligned16 = [](const void* ptr) { return (reinterpret_cast<uintptr_t>(ptr) & 15u) == 0; };
    p.o_vec = aligned16(p.o) && p.o_n % 8 == 0 && p.o_s % 8 == 0;
    auto aligned32 = [](const void* ptr) { return (reinterpret_cast<uintptr_t>(ptr) & 31u) == 0; };
    p.o_vec32 = aligned32(p.o) && p.o_n % 16 == 0 && p.o_s % 16 == 0;
    p.st_vec32 = aligned32(p.smax) && aligned32(p.ssum) && p.st_n % 8 == 0 && p.st_s % 8 == 0;
    using fa::tma_dim_ok;
    // the tensor-core kernels: head dims up to 128 on the two-tile kernel,
    // 129..256 on the one-tile (wide) kernel, as for fa_fwd
    const bool sm100 = (dt == FA_F16 || dt == FA_BF16) && D <= 256 && D % 8 == 0 && Dv % 8 == 0 && aligned16(p.q) &&
                       aligned16(p.k) && aligned16(p.v) && tma_dim_ok(qst, Tq) && tma_dim_ok(qsn, Nq) &&
                       tma_dim_ok(kst, Tk) && tma_dim_ok(ksn, Nk) && tma_dim_ok(vst, Tk) && tma_dim_ok(vsn, Nk);

    if (sm100) {
        int64_t blocks = 0, prev = 0;
        for (int64_t b = 0; b < nSeq; ++b) {
            blocks += (actualSeqQLen[b] - prev + 255) / 256;
            prev = actualSeqQLen[b];
        }
        if (blocks > kStaticMaxBlocks) return FA_ERR_INNER_NULLPTR;  // scratch limit
    }

    void* scratch = nullptr;
    if (scratch_address(&scratch) != cudaSuccess || scratch == nullptr) return FA_ERR_CUDA;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    unsigned char* dev = static_cast<unsigned char*>(scratch);

    // What this call reads, and nothing more: the ticket counter (zero), the
    // offsets of its nSeq sequences and, for the tensor-core kernels, its
    // work table.
    const size_t tab_off = table_offset(nSeq);
    size_t bytes = kCuOffset + 2 * (nSeq + 1) * sizeof(int64_t);
    {
        std::lock_guard<std::mutex> lock(g_stage_mutex);
        std::memset(g_host_stage, 0, kCuOffset);  // ticket counter = 0
        int64_t* cu = reinterpret_cast<int64_t*>(g_host_stage + kCuOffset);
        cu[0] = 0;
        cu[nSeq + 1] = 0;
        for (int64_t b = 0; b < nSeq; ++b) {
            cu[b + 1] = actualSeqQLen[b];
            cu[nSeq + 2 + b] = actualSeqKvLen[b];
        }
        if (sm100) {
            const int64_t count = fa::varlen_table_len(cu, nSeq);
            std::memset(g_host_stage + bytes, 0, tab_off - bytes);  // the alignment gap
            fa::build_varlen_table(cu, cu + nSeq + 1, nSeq, pre_c, next_c, g_sort_stage,
                                   reinterpret_cast<int4*>(g_host_stage + tab_off));
            p.table_len = (int32_t)count;
            p.n_items = p.table_len * p.Nq;
            bytes = tab_off + count * sizeof(int4);
        }
        // Pageable source: staged before the call returns (under stream
        // capture the graph carries the bytes), so the staging buffer may be
        // reused once the lock is released.
        if (fa::upload_async(dev, g_host_stage, bytes, st) != cudaSuccess) return FA_ERR_CUDA;
    }
    p.cu_q = reinterpret_cast<const int64_t*>(dev + kCuOffset);
    p.cu_kv = p.cu_q + (nSeq + 1);
    cudaError_t err;
    if (sm100) {
        p.table = reinterpret_cast<const int4*>(dev + tab_off);
        int device = 0, sms = 0;
        if (cudaGetDevice(&device) != cudaSuccess ||
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, device) != cudaSuccess)
            return FA_ERR_CUDA;
        fa::plan_sm100_schedule(p, sms, false, 0);  // varlen items differ in cost: no split
        p.sched_counter = reinterpret_cast<int*>(dev);
        fa::TmaSet maps;
        if (fa::make_sm100_tmaps(p, &maps) != cudaSuccess) return FA_ERR_CUDA;
        err = fa::launch_sm100(p, maps, p.grid, st);
    } else {
        err = fa::launch_simt(p, st);
    }
    return err == cudaSuccess ? FA_SUCCESS : FA_ERR_CUDA;
}
