// Launch parameters shared by the host planner (api.cpp) and the kernels.
// Internal to the library; the public ABI is include/fa_fwd.h.
#pragma once
#include <cstdint>
#include <cuda_runtime.h>

namespace fa {

// Row addressing.  For every operand, element (b, n, i, d) of a sequence lives
// at  base + b*stride_b + n*stride_n + (seq_off_b + i)*stride_s + d
// where seq_off_b is the sequence's first token for the packed TND layout
// (from the cumulative lengths) and 0 otherwise (stride_b is 0 for TND).
struct FaParams {
    const void* q;
    const void* k;
    const void* v;
    void* o;
    float* smax;
    float* ssum;
    const void* pse;      // dense bias (query dtype) or fp32 ALiBi slopes
    const uint8_t* mask;  // nonzero = excluded; read only when mask_on
    const float* sink;    // fp32 [Nq] or nullptr
    const void* qr;       // queryRope (query layout, head dim Dr) or nullptr
    const void* kr;       // keyRope (key layout, head dim Dr) or nullptr

    int64_t q_b, q_n, q_s;
    int64_t k_b, k_n, k_s;
    int64_t v_b, v_n, v_s;
    int64_t o_b, o_n, o_s;
    int64_t qr_b, qr_n, qr_s;
    int64_t kr_b, kr_n, kr_s;
    int64_t st_b, st_n, st_s;       // statistics; the 8 lanes are contiguous
    int64_t pse_b, pse_n, pse_i;    // dense bias strides (column stride 1); ALiBi: pse_b, pse_n
    int64_t mask_b, mask_n, mask_i; // mask strides (column stride 1), broadcast dims have 0

    const int64_t* cu_q;   // device, [B+1] with a leading 0 (TND only)
    const int64_t* cu_kv;

    int32_t B, Nq, Nkv, group;  // group = Nq / Nkv
    int32_t D, Dv;
    int32_t Dr;                 // rope head dim (0 without queryRope/keyRope): S = Q K^T + Qr Kr^T
    int32_t Sq, Skv;            // sequence lengths (TND: the longest)
    int32_t pre, next;          // band, clamped to +-(Sq + Skv + 1)
    float scale;                // scaleValue in fp32
    float scale_log2;           // scaleValue * log2(e) in fp32 (tcgen05 path)
    int32_t pse_type;           // 0 none, 1 dense, 2 ALiBi slopes
    int32_t mask_on;
    int32_t has_sink;
    int32_t varlen;
    int32_t dtype;              // FA_F32 / FA_F16 / FA_BF16

    // tcgen05 path: persistent schedule
    int32_t n_items;            // work items of (b, n, 256-row query block)
    int32_t n_qb;               // query blocks per (b, n) for the dense layouts
    int32_t items_per_n_block;  // dense: B * Nq
    int32_t head_group;         // dense: heads whose items run together, so that their K/V stay in L2
    const int4* table;          // TND: {b, qb, q_len, kv_len} per (sequence, block), heads implied
    int32_t table_len;
    int32_t neg_scale;          // scaleValue < 0: the kernel negates K inside the MMA
    int32_t Tq, Tkv;            // rows of the query / key tensors (TND: packed tokens; else Sq / Skv)
    int32_t mask_cols;          // allocated width of a mask row (columns readable from mask)
    int32_t o_vec;              // output rows allow 16-byte stores
    int32_t o_vec32;            // output rows allow 32-byte stores
    int32_t st_vec32;           // the 8 lanes of a statistics row allow 32-byte stores
    int32_t mask_vec;           // mask rows allow 16-byte loads
    int32_t pse_vec;            // dense bias rows allow 16-byte loads
    int32_t pse_tma;            // head dim 64: bias blocks come by TMA (set at launch from TmaSet::pse_ok)
    // dense bias layouts besides [B|1, N|1, Sq, Skv]:
    int32_t pse_rows1024;       // [B|1, N|1, 1024, Skv]: the last 1024 rows of the (lower-triangular) bias
    int32_t pse_flat;           // TND [sum_b N*Sq_b*Skv_b]: each sequence's [N, Sq_b, Skv_b] block in turn
    const int64_t* pse_off;     // pse_flat: device, element offset of sequence b's block
    int32_t alibi_delta;        // kvStartIdx - qStartIdx: ALiBi distance |i - j - delta| (global positions)
    int32_t debug_stall;        // failure injection: the MMA warp waits on a barrier never signalled

    // Schedule: tickets [0, n_whole) are whole work items; ticket
    // n_whole + u*n_pieces + j is piece j (a contiguous share of the key
    // blocks) of work item n_whole + u.  CTAs take tickets round-robin, or,
    // when items differ in cost, the next one from an atomic counter.
    int* sched_counter;         // device, zero at launch
    int32_t n_tickets;
    int32_t n_whole;
    int32_t n_pieces;           // 0 when no item is split
    int32_t grid;               // CTAs of the tcgen05 kernel
    int32_t dynamic;            // 1: tickets from sched_counter; 0: round-robin
    float* part;                // split items: [item u][piece j][256 rows][D + 4] fp32:
                                // O relative to m_used, then m_run, m_used, l (log2 units)
};

// fp32 words per row of a partial result
inline int part_row_words(int d) { return d + 4; }

#ifdef __CUDACC__
// Dense bias row of query row i (in-sequence index) for (b, n), as a pointer
// to element [i][0] and the number of readable columns.  The compressed form
// holds the bias rows Sq-1024 .. Sq-1; a row above them reads compressed row
// 0 shifted along its diagonal (bias[i][j] = c[0][j + Sq - 1024 - i]), which
// is the same value for a bias that depends on i - j only.
template <typename T>
__device__ __forceinline__ const T* pse_row_ptr(const FaParams& p, int b, int n, int q_len, int kv_len, int i,
                                                int* cols) {
    const T* base = static_cast<const T*>(p.pse);
    if (p.pse_flat) {
        *cols = kv_len;
        return base + p.pse_off[b] + (static_cast<int64_t>(n) * q_len + i) * kv_len;
    }
    base += b * p.pse_b + n * p.pse_n;
    if (p.pse_rows1024) {
        const int first = q_len - 1024;
        const int r = i >= first ? i - first : 0;
        const int shift = i >= first ? 0 : first - i;
        *cols = kv_len - shift;
        return base + static_cast<int64_t>(r) * p.pse_i + shift;
    }
    *cols = kv_len;
    return base + static_cast<int64_t>(i) * p.pse_i;
}
#endif

// fa_lse_merge: partial results of one query set over disjoint key sets.
// Rows are addressed as (b, n, s) with element strides (TND: b = 0, s = token).
struct MergeParams {
    static constexpr int kMax = 16;
    int32_t count;
    const void* out[kMax];
    const float* smax[kMax];
    const float* ssum[kMax];
    int64_t o_b[kMax], o_n[kMax], o_s[kMax];
    int64_t st_b[kMax], st_n[kMax], st_s[kMax];
    void* res_o;
    float* res_max;
    float* res_sum;
    int64_t r_o_b, r_o_n, r_o_s, r_st_b, r_st_n, r_st_s;
    const float* sink;  // fp32 [N] or nullptr
    int32_t B, N, S, Dv, dtype;
};
cudaError_t launch_lse_merge(const MergeParams& mp, cudaStream_t stream);

enum KernelKind { KERNEL_SIMT = 0, KERNEL_SM100 = 1 };

// Tensor-map descriptors (CUtensorMap is 128 bytes, 64-byte aligned).
struct alignas(64) TmaDesc {
    uint64_t opaque[16];
};
// Q, K, V and (with rope) queryRope, keyRope; without rope qr/kr repeat q/k
// and are never read.
// pse: a dense bias tensor [B|1, N|1, Sq, Skv] in boxes of 64 columns x 128
// rows (pse_ok = 0 when there is none or it is not TMA-legal: the kernel then
// reads bias rows itself).
struct TmaSet {
    TmaDesc q, k, v, qr, kr, pse;
    int32_t pse_ok;
};

// Varlen work table of the tcgen05 kernels: one entry {b, qb, q_len, kv_len}
// per (sequence b, 256-row query block qb), longest first -- by the number of
// 128-key blocks the block's two query tiles touch under the band
// -pre <= j - i <= next -- with ties in (sequence, block) order.  cu_q and
// cu_kv are cumulative lengths with a leading 0 (B + 1 entries each).
struct VarlenEntry {
    int64_t cost;
    int64_t order;
    int4 e;
};
int64_t varlen_table_len(const int64_t* cu_q, int64_t B);
// Writes varlen_table_len() entries to `out`, using `scratch` (as many
// VarlenEntry) for the sort; allocates nothing.
void build_varlen_table(const int64_t* cu_q, const int64_t* cu_kv, int64_t B, int64_t pre, int64_t next,
                        VarlenEntry* scratch, int4* out);
// A tensor-map dimension of `size` elements with an element stride of
// `stride` (16-bit elements): legal for TMA when the size is 1, or the byte
// stride is positive, a multiple of 16 and below 2^40.
bool tma_dim_ok(int64_t stride, int64_t size);

cudaError_t launch_simt(const FaParams& p, cudaStream_t stream);
cudaError_t launch_sm100(const FaParams& p, const TmaSet& maps, int num_sms, cudaStream_t stream);
// Schedule of the tcgen05 kernel (fills grid, n_whole, n_pieces, n_tickets
// from n_items): one CTA per SM, and, when every work item costs the same
// (`uniform`, item_kv_blocks 128-key blocks each) and the last wave is short,
// the last wave's items split into key pieces.  Returns the bytes of partial
// results the split needs (0 without a split).
uint64_t plan_sm100_schedule(FaParams& p, int num_sms, bool uniform, int item_kv_blocks);
// Encodes the Q/K/V (and rope) tensor maps for the tcgen05 kernel.
cudaError_t make_sm100_tmaps(const FaParams& p, TmaSet* maps);
uint64_t read_and_clear_device_error(cudaError_t* err);
// Host-to-device copy of a small table: cudaMemcpyAsync, or, while `stream`
// is being captured into a CUDA graph, copy kernels that carry the bytes in
// their launch parameters (the graph keeps them; the host source may go).
cudaError_t upload_async(void* dst, const void* src, size_t bytes, cudaStream_t stream);

}  // namespace fa
