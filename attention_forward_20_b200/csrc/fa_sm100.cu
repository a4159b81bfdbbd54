// tcgen05 attention forward for sm_100a (fp16 / bf16 inputs, head dim 64 or 128).
//
// What it computes is the forward and sink formulas of the
// aclnnFlashAttentionVarLenScoreV5 page ("计算公式"), tiled with the
// FlashAttention online softmax (aclnnFlashAttentionScore, "功能描述").
//
// One persistent CTA per SM walks a static list of work items; an item is one
// (batch, query head, 256-row query block), split into two 128-row query tiles
// that ping-pong on the tensor core:
//
//   warps 0-3  softmax tile 0   (thread r owns TMEM lane r = query row r)
//   warps 4-7  softmax tile 1
//   warp  8    TMA producer     (Q tiles, then K and V 128-row blocks into a ring)
//   warp  9    MMA issuer       (S = Q·Kᵀ and O += P·V with tcgen05.mma)
//   warps 10-11 idle (they complete the third warpgroup)
//
// The launch gives every thread the same register budget; setmaxnreg then
// moves registers from the producer/MMA warpgroup (kOtherRegs) to the two
// softmax warpgroups (kSoftmaxRegs), which hold a whole 128-column S row.
//
// TMEM (512 columns): S_t at columns [128t, 128t+128) as fp32; P_t (fp16/bf16,
// two per column) overwrites the first 64 of them and is the A operand of
// P·V; O_t at [256 + t*D, 256 + (t+1)*D) as fp32.
//
// Softmax runs in the log2 domain: x = s * scale * log2(e) (+ bias * log2(e)),
// p = 2^(x - m_used).  The running row max m_run is exact; m_used, the max the
// exponentials are taken against, only moves (rescaling l and O) when m_run
// exceeds it by more than 8, so that p <= 2^8 and most blocks skip the O
// rescale.  The epilogue folds in the sink (max and denominator) and converts
// the statistics back to natural-log units.
//
// Every wait is bounded (mbar_wait): on a timeout the CTA records the failure
// in a device error word, drains its in-flight copies and MMAs, frees TMEM and
// exits.
#include "fa_params.h"
#include "sm100_ptx.cuh"

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <math_constants.h>

#include <mutex>
#include <type_traits>

namespace fa {

__device__ unsigned long long g_fa_error;

namespace {
using namespace ptx;

constexpr int kTileM = 128;     // query rows per tile (one TMEM lane each)
constexpr int kTileN = 128;     // keys per block
constexpr int kQBlock = 256;    // query rows per work item (two tiles)
constexpr int kThreads = 384;   // three warpgroups
// Per-thread registers after setmaxnreg: softmax warpgroups / producer-MMA
// warpgroup.  The producer and MMA warps of the rope, ALiBi-ramp and
// bias-buffer kernels keep more state.
template <bool kMoreOther>
constexpr uint32_t kSoftmaxRegs = kMoreOther ? 216 : 224;
template <bool kMoreOther>
constexpr uint32_t kOtherRegs = kMoreOther ? 72 : 56;
// setmaxnreg hands out what the launch reserved: 384 threads x 168 registers
// (the allocation unit is 8 registers per thread; 176 x 384 exceeds 64K)
static_assert(2 * 128 * kSoftmaxRegs<false> + 128 * kOtherRegs<false> <= (65536 / kThreads) / 8 * 8 * kThreads &&
                  2 * 128 * kSoftmaxRegs<true> + 128 * kOtherRegs<true> <= (65536 / kThreads) / 8 * 8 * kThreads,
              "register split exceeds the launch's reservation");
constexpr int kLoadWarp = 8;
constexpr int kMmaWarp = 9;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.69314718055994531f;
constexpr float kRescaleThreshold = 8.0f;

// Column pairs, of every 8 in a score row, whose exponentials run on the FMA
// pipe (exp2_fma2) instead of MUFU, by padded head dim: MUFU bounds the
// softmax at every head dim (16 exponentials per clock per SM), the FMA pipe
// has room beside it.
#ifndef FA_POLY_PAIRS_64
#define FA_POLY_PAIRS_64 0
#endif
#ifndef FA_POLY_PAIRS_128
#define FA_POLY_PAIRS_128 0
#endif
#ifndef FA_POLY_PAIRS_256
#define FA_POLY_PAIRS_256 0
#endif
template <int D>
constexpr int kPolyPairs = D <= 64 ? FA_POLY_PAIRS_64 : (D <= 128 ? FA_POLY_PAIRS_128 : FA_POLY_PAIRS_256);
static_assert(kPolyPairs<64> >= 0 && kPolyPairs<64> <= 8 && kPolyPairs<128> >= 0 && kPolyPairs<128> <= 8 &&
                  kPolyPairs<256> >= 0 && kPolyPairs<256> <= 8,
              "poly pairs per 8");
constexpr int kSched = 4;            // ticket slots between the TMA warp and the other warps
constexpr int kTicketEnd = -1;       // no work left
constexpr int kTicketAbort = -2;     // a bounded wait gave up
constexpr int kTicketReaders = 9;    // the MMA warp and the eight softmax warps
constexpr int kMergeThreads = 256;

// wait sites recorded in the error word
enum : int {
    kSiteQEmpty = 1, kSiteKvEmpty, kSiteQFull, kSiteKvFull, kSitePFull,
    kSiteSFull, kSiteOFull, kSiteDrain, kSiteInjected, kSiteSched
};

// kRope: queryRope/keyRope with a head dim of 64 — one 128-byte chunk more
// in every Q tile (after its D columns) and, for K, in a two-slot ring of
// its own that fills with K under K's barrier.
// kAug (ALiBi slopes, head dim 64): the column ramp of the ALiBi bias comes
// out of the S MMA as one more K-step of 16: a chunk after Q's D columns
// holds, in every row, the slope (over scale) split into three terms, and a
// fixed chunk holds, for key c of the block, (c, c, c); so S gains
// slope/scale * c and a block left of every row's diagonal needs no bias
// work in the softmax (its per-row part joins the max and the shift).
// kTmaBias (dense bias tensor, head dim 64): the bias block of each query
// tile comes into shared memory by TMA (two 64-column boxes, two buffers per
// tile) instead of per-thread row loads; the K/V ring has 4 slots then.
template <int D, bool kRope = false, bool kAug = false, bool kTmaBias = false>
struct Cfg {
    static constexpr int kChunks = D / 64;             // 128-byte swizzle chunks per row
    static constexpr int kChunkBytes = kTileM * 128;   // one chunk of a 128-row tile
    static constexpr int kTileBytes = kTileM * D * 2;  // one K or V tile
    static constexpr int kQTileBytes = kTileBytes + ((kRope || kAug) ? kChunkBytes : 0);
    static constexpr int kRopeSlots = kRope ? 2 : 0;
    static constexpr int kAugBytes = kAug ? kChunkBytes : 0;  // the fixed (c, c, c) key chunk
    static constexpr int kStages = (D == 128) ? (kRope ? 3 : 4) : (kTmaBias ? 4 : 8);  // K/V ring slots
    static constexpr int kBiasTileBytes = kTileM * kTileN * 2;                     // one 128 x 128 block
    static constexpr int kBiasBytes = kTmaBias ? 4 * kBiasTileBytes : 0;          // 2 tiles x 2 buffers
    static constexpr int kSmemBytes =
        2 * kQTileBytes + kStages * kTileBytes + kRopeSlots * kChunkBytes + kAugBytes + kBiasBytes + 1024;
    static constexpr uint32_t kTmemCols = 512;
};
constexpr uint32_t kOCol = 256;  // TMEM column of O (S and P use 0..255)
static_assert(Cfg<128, true>::kSmemBytes + 1024 <= 227 * 1024, "rope tiles exceed shared memory");
static_assert(Cfg<64, true>::kSmemBytes + 1024 <= 227 * 1024, "rope tiles exceed shared memory");
static_assert(Cfg<64, false, true>::kSmemBytes + 1024 <= 227 * 1024, "ALiBi ramp chunks exceed shared memory");
static_assert(Cfg<64, false, false, true>::kSmemBytes + 1024 <= 227 * 1024, "bias buffers exceed shared memory");
template <int D, int kBias, bool kRope>
constexpr bool kAugRamp = kBias == 2 && D == 64 && !kRope;
template <int D, int kBias, bool kRope>
constexpr bool kTmaBiasK = kBias == 1 && D == 64 && !kRope;
// compressed-bias windows (in the bias buffers): 160 fp32 per copy, 4 copies per warp
constexpr int kWinLen = 160;
constexpr int kWinBytes = 4 * kWinLen * 4;
static_assert(8 * kWinBytes <= 4 * kTileM * kTileN * 2, "windows exceed the bias buffers");

__device__ __forceinline__ float to_f(__half x) { return __half2float(x); }
__device__ __forceinline__ float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }
__device__ __forceinline__ uint16_t bits16(__half x) { return __half_as_ushort(x); }
__device__ __forceinline__ uint16_t bits16(__nv_bfloat16 x) { return __bfloat16_as_ushort(x); }
template <typename T>
__device__ __forceinline__ T from_bits16(uint16_t b);
template <>
__device__ __forceinline__ __half from_bits16<__half>(uint16_t b) { return __ushort_as_half(b); }
template <>
__device__ __forceinline__ __nv_bfloat16 from_bits16<__nv_bfloat16>(uint16_t b) { return __ushort_as_bfloat16(b); }

// Row r's 16-byte piece k (k < 8) of a 128-byte-swizzled 128-row chunk.
__device__ __forceinline__ uint32_t sw128_offset(int r, int k) { return r * 128 + ((k ^ (r & 7)) << 4); }

struct Barriers {
    uint64_t q_full[2], q_empty[2], s_full[2], p_full[2], o_full[2];
    uint64_t p_half[2];    // two-tile kernel: the first 64 keys' half of P_t is in TMEM
    uint64_t bias_full[2][2], bias_empty[2][2];  // kTmaBias: tile t's bias buffers
    uint64_t kv_full[8], kv_empty[8];
    uint64_t kr_empty[2];  // keyRope slots (the K load's kv_full also covers its keyRope chunk)
    uint64_t pv_done;      // wide kernel: one completion per key block's P·V
    uint64_t sched_full[kSched], sched_empty[kSched];
    uint64_t drain;
    uint64_t never;  // failure injection: initialised, never arrived on
    int ticket[kSched];
};

struct Item {
    int b, n, nk, qb, q_len, kv_len;
    int64_t q_off, kv_off;
};

// The dynamic schedule's hand-off slots: the ticket and its decoded item (the
// TMA warp pays for the varlen table and offset loads, the others read smem).
struct TicketSlots {
    Item item[kSched];
};

// Work item -> (batch, head, query block).  Dense layouts: groups of
// p.head_group heads; inside a group the query blocks go from the last (the
// most keys under a causal band) to the first, heads fastest.  TND: the host
// table lists (sequence, block) longest first; heads fastest.
__device__ __forceinline__ Item decode_item(const FaParams& p, int item) {
    Item it;
    if (p.varlen) {
        const int e = item / p.Nq;
        it.n = item - e * p.Nq;
        const int4 t = p.table[e];
        it.b = t.x;
        it.qb = t.y;
        it.q_len = t.z;
        it.kv_len = t.w;
        it.q_off = p.cu_q[it.b];
        it.kv_off = p.cu_kv[it.b];
    } else {
        const int bn_total = p.B * p.Nq;
        const int hg = p.head_group;
        const int per_group = hg * p.n_qb;
        const int g = item / per_group;
        const int within = item - g * per_group;
        const int g_heads = min(hg, bn_total - g * hg);
        const int level = within / g_heads;
        const int bn = g * hg + (within - level * g_heads);
        it.qb = p.n_qb - 1 - level;
        it.b = bn / p.Nq;
        it.n = bn - it.b * p.Nq;
        it.q_len = p.Sq;
        it.kv_len = p.Skv;
        it.q_off = 0;
        it.kv_off = 0;
    }
    it.nk = it.n / p.group;
    return it;
}

// Key blocks [lo, hi] that query tile t of the item touches under the band
// -pre <= j - i <= next; lo > hi when none.  `valid` says the tile has rows.
struct TileRange {
    int valid, lo, hi;
    __device__ __forceinline__ bool active() const { return valid && hi >= lo; }
    __device__ __forceinline__ bool has(int jb) const { return valid && jb >= lo && jb <= hi; }
};

__device__ __forceinline__ TileRange tile_range(const FaParams& p, const Item& it, int t) {
    TileRange r{0, 0, -1};
    const int r0 = it.qb * kQBlock + t * kTileM;
    if (r0 >= it.q_len) return r;
    r.valid = 1;
    const int r1 = min(it.q_len, r0 + kTileM) - 1;
    const int j_lo = max(0, r0 - p.pre);
    const int j_hi = min(it.kv_len - 1, r1 + p.next);
    if (j_hi >= j_lo) {
        r.lo = j_lo / kTileN;
        r.hi = j_hi / kTileN;
    }
    return r;
}

// What a ticket stands for: a whole work item, or piece `piece` of split
// item number `tail` (counted among the split ones), whose tiles then only
// cover that piece's share of the item's key blocks.
struct Work {
    Item it;
    TileRange tr[2];
    int piece;  // -1: the whole item
    int tail;
};

__device__ __forceinline__ int item_of_ticket(const FaParams& p, int ticket) {
    return ticket < p.n_whole ? ticket : p.n_whole + (ticket - p.n_whole) / p.n_pieces;
}

__device__ __forceinline__ Work work_of(const FaParams& p, int ticket, const Item& it) {
    Work w;
    w.piece = -1;
    w.tail = 0;
    if (ticket >= p.n_whole) {
        const int u = ticket - p.n_whole;
        w.tail = u / p.n_pieces;
        w.piece = u - w.tail * p.n_pieces;
    }
    w.it = it;
    w.tr[0] = tile_range(p, w.it, 0);
    w.tr[1] = tile_range(p, w.it, 1);
    if (w.piece >= 0 && (w.tr[0].active() || w.tr[1].active())) {
        const int lo = w.tr[0].active() ? (w.tr[1].active() ? min(w.tr[0].lo, w.tr[1].lo) : w.tr[0].lo) : w.tr[1].lo;
        const int hi = w.tr[0].active() ? (w.tr[1].active() ? max(w.tr[0].hi, w.tr[1].hi) : w.tr[0].hi) : w.tr[1].hi;
        const int n = hi - lo + 1;
        const int c0 = lo + (w.piece * n) / p.n_pieces;
        const int c1 = lo + ((w.piece + 1) * n) / p.n_pieces - 1;
        for (int t = 0; t < 2; ++t) {
            if (w.tr[t].active()) {
                w.tr[t].lo = max(w.tr[t].lo, c0);
                w.tr[t].hi = min(w.tr[t].hi, c1);
                if (w.tr[t].hi < w.tr[t].lo) {  // no block of this tile in the piece
                    w.tr[t].lo = 0;
                    w.tr[t].hi = -1;
                }
            }
        }
    }
    return w;
}

__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort, int site) {
    const bool ok = mbar_wait(bar, parity, abort, site);
    return __all_sync(0xffffffffu, ok);
}

// Tickets.  Equal-cost items (p.dynamic == 0) go round-robin: the k-th ticket
// of CTA c is c + k * gridDim.x, which every warp computes for itself.
// Otherwise the TMA warp takes the next ticket from the global counter as soon
// as it has issued the loads of the previous one, and hands it to the MMA warp
// and the softmax warps through kSched shared-memory slots.
__device__ __forceinline__ int static_ticket(const FaParams& p, uint32_t& k, Item& it) {
    const int tk = blockIdx.x + static_cast<int>(k++) * gridDim.x;
    if (tk >= p.n_tickets) return kTicketEnd;
    it = decode_item(p, item_of_ticket(p, tk));
    return tk;
}
__device__ __forceinline__ int take_ticket_global(const FaParams& p, Barriers& bars, TicketSlots& slots, uint32_t& k,
                                                  Item& it, volatile int* abort) {
    if (!p.dynamic) return static_ticket(p, k, it);
    const uint32_t slot = k % kSched;
    if (!warp_wait(&bars.sched_empty[slot], ((k / kSched) & 1) ^ 1, abort, kSiteSched)) return kTicketAbort;
    int tk = 0;
    if ((threadIdx.x & 31) == 0) {
        tk = atomicAdd(p.sched_counter, 1);
        if (tk >= p.n_tickets) tk = kTicketEnd;
    }
    tk = __shfl_sync(0xffffffffu, tk, 0);
    if (tk >= 0) it = decode_item(p, item_of_ticket(p, tk));
    if ((threadIdx.x & 31) == 0) {
        bars.ticket[slot] = tk;
        if (tk >= 0) slots.item[slot] = it;
        mbar_arrive(&bars.sched_full[slot]);
    }
    ++k;
    return tk;
}
__device__ __forceinline__ int take_ticket_local(const FaParams& p, Barriers& bars, const TicketSlots& slots,
                                                 uint32_t& k, Item& it, volatile int* abort) {
    if (!p.dynamic) return static_ticket(p, k, it);
    const uint32_t slot = k % kSched;
    if (!warp_wait(&bars.sched_full[slot], (k / kSched) & 1, abort, kSiteSched)) return kTicketAbort;
    const int tk = *reinterpret_cast<volatile int*>(&bars.ticket[slot]);
    if (tk >= 0) it = slots.item[slot];
    __syncwarp();
    if ((threadIdx.x & 31) == 0) mbar_arrive(&bars.sched_empty[slot]);
    ++k;
    return tk;
}

// ---------------------------------------------------------------------------
// TMA producer (one warp: every lane follows the schedule and waits, so all
// operands stay warp-uniform; one elected lane issues the copies)
// ---------------------------------------------------------------------------
template <typename T, int D, bool kRope, bool kAug, bool kTmaBias>
__device__ void run_producer(const FaParams& p, const CUtensorMap* tq, const CUtensorMap* tk,
                             const CUtensorMap* tv, const CUtensorMap* tqr, const CUtensorMap* tkr,
                             const CUtensorMap* tpse, uint8_t* sQ, uint8_t* sKV, uint8_t* sKr, uint8_t* sBias,
                             Barriers& bars, TicketSlots& slots, volatile int* abort) {
    using C = Cfg<D, kRope, kAug, kTmaBias>;
    uint32_t kv_fill = 0, q_fill[2] = {0, 0}, k_sched = 0, kr_fill = 0, b_fill[2] = {0, 0};
    bool ok = true;
    const int v_chunks = (p.Dv + 63) / 64;

    auto load_chunks = [&](const CUtensorMap* tm, uint8_t* dst, uint64_t* bar, int chunks, int row, int head,
                           int b, int64_t seq_off) {
        for (int c = 0; c < chunks; ++c) {
            if (p.varlen)
                tma_load_3d(dst + c * C::kChunkBytes, tm, bar, c * 64, (int)(seq_off + row), head);
            else
                tma_load_4d(dst + c * C::kChunkBytes, tm, bar, c * 64, row, head, b);
        }
    };
    auto load_tile = [&](const CUtensorMap* tm, uint8_t* dst, uint64_t* bar, int row, int head, int b,
                         int64_t seq_off) { load_chunks(tm, dst, bar, C::kChunks, row, head, b, seq_off); };

    while (ok) {
        Item tit;
        const int ticket = take_ticket_global(p, bars, slots, k_sched, tit, abort);
        if (ticket == kTicketAbort) { ok = false; break; }
        if (ticket == kTicketEnd) break;
        const Work wk = work_of(p, ticket, tit);
        const Item it = wk.it;
        const TileRange tr[2] = {wk.tr[0], wk.tr[1]};
        if (!tr[0].active() && !tr[1].active()) continue;
        const int lo = tr[0].active() ? (tr[1].active() ? min(tr[0].lo, tr[1].lo) : tr[0].lo) : tr[1].lo;
        const int hi = tr[0].active() ? (tr[1].active() ? max(tr[0].hi, tr[1].hi) : tr[0].hi) : tr[1].hi;

        auto load_q = [&](int t) -> bool {
            if (!warp_wait(&bars.q_empty[t], (q_fill[t] & 1) ^ 1, abort, kSiteQEmpty)) return false;
            if constexpr (kAug) {
                // the item's slope in every row of the ramp chunk (three terms
                // whose sum is slope·log2(e)/|scale|, negated with the scale,
                // as the MMA then negates K), made visible to the tensor core
                const float a = (p.neg_scale ? -1.f : 1.f) *
                                static_cast<const float*>(p.pse)[it.b * p.pse_b + it.n * p.pse_n] * kLog2e /
                                p.scale_log2;
                const T a0 = static_cast<T>(a);
                const T a1 = static_cast<T>(a - to_f(a0));
                const T a2 = static_cast<T>(a - to_f(a0) - to_f(a1));
                const uint32_t w0 = static_cast<uint32_t>(bits16(a0)) | (static_cast<uint32_t>(bits16(a1)) << 16);
                const uint32_t w1 = static_cast<uint32_t>(bits16(a2));
                const uint32_t base = smem_u32(sQ + t * C::kQTileBytes + C::kTileBytes);
                for (int r = threadIdx.x & 31; r < kTileM; r += 32) st_shared_v4(base + sw128_offset(r, 0), w0, w1, 0u, 0u);
                fence_proxy_async_smem();
                __syncwarp();
            }
            if (elect_one()) {
                mbar_arrive_expect_tx(&bars.q_full[t], kAug ? C::kTileBytes : C::kQTileBytes);
                load_tile(tq, sQ + t * C::kQTileBytes, &bars.q_full[t], it.qb * kQBlock + t * kTileM, it.n, it.b,
                          it.q_off);
                if constexpr (kRope)
                    load_chunks(tqr, sQ + t * C::kQTileBytes + C::kTileBytes, &bars.q_full[t], 1,
                                it.qb * kQBlock + t * kTileM, it.n, it.b, it.q_off);
            }
            __syncwarp();
            ++q_fill[t];
            return true;
        };
        // K tiles: all kChunks chunks (columns past D read as zero); V tiles:
        // the chunks that hold its Dv columns.
        auto load_kv = [&](const CUtensorMap* tm, int jb, bool is_k) -> bool {
            const bool with_rope = is_k;
            const int chunks = is_k ? C::kChunks : v_chunks;
            const int slot = kv_fill % C::kStages;
            if (!warp_wait(&bars.kv_empty[slot], ((kv_fill / C::kStages) & 1) ^ 1, abort, kSiteKvEmpty))
                return false;
            const uint32_t rs = kr_fill % 2;
            if (kRope && with_rope &&
                !warp_wait(&bars.kr_empty[rs], ((kr_fill / 2) & 1) ^ 1, abort, kSiteKvEmpty))
                return false;
            if (elect_one()) {
                mbar_arrive_expect_tx(&bars.kv_full[slot],
                                      chunks * C::kChunkBytes + (kRope && with_rope ? C::kChunkBytes : 0));
                load_chunks(tm, sKV + slot * C::kTileBytes, &bars.kv_full[slot], chunks, jb * kTileN, it.nk, it.b,
                            it.kv_off);
                if (kRope && with_rope)
                    load_chunks(tkr, sKr + rs * C::kChunkBytes, &bars.kv_full[slot], 1, jb * kTileN, it.nk, it.b,
                                it.kv_off);
            }
            __syncwarp();
            ++kv_fill;
            if (kRope && with_rope) ++kr_fill;
            return true;
        };

        // kTmaBias: tile t's bias block [rows of the tile] x [128 keys of
        // block jb] into its next buffer (broadcast dimensions read index 0)
        auto load_bias = [&](int t, int jb) -> bool {
            const uint32_t slot = b_fill[t] & 1;
            if (!warp_wait(&bars.bias_empty[t][slot], ((b_fill[t] >> 1) & 1) ^ 1, abort, kSiteKvEmpty)) return false;
            if (elect_one()) {
                uint8_t* dst = sBias + (t * 2 + slot) * C::kBiasTileBytes;
                const int row = it.qb * kQBlock + t * kTileM;
                const int nb = p.pse_n ? it.n : 0, bb = p.pse_b ? it.b : 0;
                // the second box only when it starts inside the keys (columns
                // past the keys are masked; the first box always starts inside)
                const bool second = jb * kTileN + 64 < p.Skv;
                mbar_arrive_expect_tx(&bars.bias_full[t][slot], second ? C::kBiasTileBytes : C::kBiasTileBytes / 2);
                tma_load_4d(dst, tpse, &bars.bias_full[t][slot], jb * kTileN, row, nb, bb);
                if (second)
                    tma_load_4d(dst + C::kBiasTileBytes / 2, tpse, &bars.bias_full[t][slot], jb * kTileN + 64, row, nb,
                                bb);
            }
            __syncwarp();
            ++b_fill[t];
            return true;
        };

        if (tr[0].active() && !load_q(0)) { ok = false; break; }
        for (int jb = lo; ok && jb <= hi; ++jb) {
            if (!load_kv(tk, jb, true)) { ok = false; break; }
            if (jb == lo && tr[1].active() && !load_q(1)) { ok = false; break; }
            if (kTmaBias && p.pse_tma) {
                for (int t = 0; t < 2 && ok; ++t)
                    if (tr[t].has(jb) && !load_bias(t, jb)) ok = false;
                if (!ok) break;
            }
            if (!load_kv(tv, jb, false)) { ok = false; break; }
        }
    }

    // Drain: the latest fill of every slot (and Q buffer) must have landed
    // before the CTA may exit; earlier fills of a slot completed before the
    // slot could be refilled.
    for (int s = 0; s < C::kStages; ++s) {
        if ((uint32_t)s < kv_fill) {
            const uint32_t last = kv_fill - 1 - ((kv_fill - 1 - s) % C::kStages);
            mbar_wait_drain(&bars.kv_full[s], (last / C::kStages) & 1, abort, kSiteDrain);
        }
    }
    for (int t = 0; t < 2; ++t)
        if (q_fill[t]) mbar_wait_drain(&bars.q_full[t], (q_fill[t] - 1) & 1, abort, kSiteDrain);
    for (int t = 0; t < 2; ++t)
        for (uint32_t k = 0; k < 2; ++k)
            if (k < b_fill[t]) {
                const uint32_t last = b_fill[t] - 1 - ((b_fill[t] - 1 - k) % 2);
                mbar_wait_drain(&bars.bias_full[t][k], (last >> 1) & 1, abort, kSiteDrain);
            }
}

// ---------------------------------------------------------------------------
// MMA issuer (one warp, converged: descriptors and TMEM addresses are
// warp-uniform values; one elected lane issues each tcgen05 instruction, the
// same lane every time, so its commits cover its MMAs)
// ---------------------------------------------------------------------------
template <typename T, int D, bool kRope, bool kAug, bool kTmaBias>
__device__ void run_mma(const FaParams& p, uint8_t* sQ, uint8_t* sKV, uint8_t* sKr, uint8_t* sAug, Barriers& bars,
                        const TicketSlots& slots, uint32_t tmem, volatile int* abort) {
    using C = Cfg<D, kRope, kAug, kTmaBias>;
    constexpr bool kBf16 = std::is_same<T, __nv_bfloat16>::value;
    const uint32_t idesc_qk = idesc_f16(kBf16, kTileM, kTileN, false, false, p.neg_scale != 0);
    // P·V over the 64-column chunks that hold V's Dv columns
    const uint32_t idesc_pv = idesc_f16(kBf16, kTileM, ((p.Dv + 63) / 64) * 64, false, true, false);
    uint32_t kv_use = 0, q_use[2] = {0, 0}, p_cnt[2] = {0, 0}, k_sched = 0, kr_use = 0;
    bool ok = true;
    // Failure injection: a wait that can only end by running out of time.
    if (p.debug_stall && !warp_wait(&bars.never, 0, abort, kSiteInjected)) ok = false;

    auto wait_kv = [&](int* slot) -> bool {
        *slot = kv_use % C::kStages;
        const bool r = warp_wait(&bars.kv_full[*slot], (kv_use / C::kStages) & 1, abort, kSiteKvFull);
        ++kv_use;
        return r;
    };
    // One elected lane (elect.sync: the same lane every time in a converged
    // warp) issues every MMA and commit, so its commits track its MMAs; the
    // descriptors of the fixed shared-memory buffers are computed once, slot
    // k of the ring being kTileBytes further.
    auto commit = [&](uint64_t* bar) {
        if (elect_one()) tc_commit(bar);
        __syncwarp();
    };
    // S_t = Q_t · K^T: D/16 MMAs of K = 16; both operands K-major, 128-byte
    // swizzled, 8-row groups 1024 bytes apart, 64-column chunks one tile-chunk apart.
    // S_t = Q_t · K^T over D/16 K-steps, O_t (+)= P_t · V over 8 K-steps:
    // each group is one asm block issued by one lane.
    // With rope, 4 more K-steps over the queryRope / keyRope chunks accumulate
    // into the same S.
    constexpr uint64_t kSlotDesc = C::kTileBytes >> 4;  // descriptor start-address units of 16 bytes
    const uint64_t qdesc[2] = {sdesc_sw128(smem_u32(sQ), 1024, 16),
                               sdesc_sw128(smem_u32(sQ + C::kQTileBytes), 1024, 16)};
    const uint64_t kdesc0 = sdesc_sw128(smem_u32(sKV), 1024, 16);
    const uint64_t vdesc0 = sdesc_sw128(smem_u32(sKV), 1024, C::kChunkBytes);
    auto issue_qk = [&](int t, int slot, uint32_t rs) {
        const uint64_t qd = t ? qdesc[1] : qdesc[0];
        const uint64_t kd = kdesc0 + static_cast<uint64_t>(slot) * kSlotDesc;
        if (elect_one()) {
            if constexpr (D == 128)
                mma_ss_k128(tmem + t * kTileN, qd, kd, idesc_qk, 0u);
            else
                mma_ss_k64(tmem + t * kTileN, qd, kd, idesc_qk, 0u);
            if constexpr (kRope) {
                const uint64_t qrd = sdesc_sw128(smem_u32(sQ + t * C::kQTileBytes + C::kTileBytes), 1024, 16);
                const uint64_t krd = sdesc_sw128(smem_u32(sKr + rs * C::kChunkBytes), 1024, 16);
                mma_ss_k64(tmem + t * kTileN, qrd, krd, idesc_qk, 1u);
            }
            if constexpr (kAug) {
                const uint64_t qad = sdesc_sw128(smem_u32(sQ + t * C::kQTileBytes + C::kTileBytes), 1024, 16);
                mma_ss(tmem + t * kTileN, qad, sdesc_sw128(smem_u32(sAug), 1024, 16), idesc_qk, 1u);
            }
        }
        __syncwarp();
    };
    // O_t (+)= P_t · V over the block's keys 64h .. 64h+63: P columns 32h..,
    // V rows from 64h (4 K-steps of 16 keys, 2048 bytes each)
    auto issue_pv_half = [&](int t, int slot, int h, bool accumulate) {
        const uint64_t vd = vdesc0 + static_cast<uint64_t>(slot) * kSlotDesc + static_cast<uint64_t>(h) * (4 * 2048 / 16);
        if (elect_one())
            mma_ts_k64(tmem + kOCol + t * D, tmem + t * kTileN + 32 * h, vd, idesc_pv, accumulate ? 1u : 0u);
        __syncwarp();
    };

    while (ok) {
        Item tit;
        const int ticket = take_ticket_local(p, bars, slots, k_sched, tit, abort);
        if (ticket == kTicketAbort) { ok = false; break; }
        if (ticket == kTicketEnd) break;
        const Work wk = work_of(p, ticket, tit);
        const TileRange tr[2] = {wk.tr[0], wk.tr[1]};
        if (!tr[0].active() && !tr[1].active()) continue;
        const int lo = tr[0].active() ? (tr[1].active() ? min(tr[0].lo, tr[1].lo) : tr[0].lo) : tr[1].lo;
        const int hi = tr[0].active() ? (tr[1].active() ? max(tr[0].hi, tr[1].hi) : tr[0].hi) : tr[1].hi;

        for (int t = 0; t < 2; ++t)
            if (tr[t].active() && !warp_wait(&bars.q_full[t], q_use[t] & 1, abort, kSiteQFull)) ok = false;
        int sk;
        if (!ok || !wait_kv(&sk)) { ok = false; break; }
        tc_fence_after();
        uint32_t rs = kr_use % 2;
        for (int t = 0; t < 2; ++t) {
            if (tr[t].has(lo)) {
                issue_qk(t, sk, rs);
                commit(&bars.s_full[t]);
                if (lo == tr[t].hi) commit(&bars.q_empty[t]);
            }
        }
        commit(&bars.kv_empty[sk]);
        if constexpr (kRope) { commit(&bars.kr_empty[rs]); ++kr_use; }

        for (int jb = lo; jb <= hi; ++jb) {
            int sv, sk2 = 0;
            const bool has_next = jb < hi;
            if (!wait_kv(&sv) || (has_next && !wait_kv(&sk2))) { ok = false; break; }
            tc_fence_after();
            rs = kr_use % 2;
            for (int t = 0; t < 2; ++t) {
                if (tr[t].has(jb)) {
                    // the first half of P·V as soon as the softmax has stored
                    // that half of P, the second after the whole of P
                    if (!warp_wait(&bars.p_half[t], p_cnt[t] & 1, abort, kSitePFull)) { ok = false; break; }
                    tc_fence_after();
                    issue_pv_half(t, sv, 0, jb != tr[t].lo);
                    if (!warp_wait(&bars.p_full[t], p_cnt[t] & 1, abort, kSitePFull)) { ok = false; break; }
                    ++p_cnt[t];
                    tc_fence_after();
                    issue_pv_half(t, sv, 1, true);
                    if (jb == tr[t].hi) commit(&bars.o_full[t]);
                }
                if (has_next && tr[t].has(jb + 1)) {
                    issue_qk(t, sk2, rs);
                    commit(&bars.s_full[t]);
                    if (jb + 1 == tr[t].hi) commit(&bars.q_empty[t]);
                }
            }
            if (!ok) break;
            commit(&bars.kv_empty[sv]);
            if (has_next) commit(&bars.kv_empty[sk2]);
            if (kRope && has_next) { commit(&bars.kr_empty[rs]); ++kr_use; }
        }
        for (int t = 0; t < 2; ++t)
            if (tr[t].active()) ++q_use[t];
    }
    // Drain: every MMA this warp issued completes before TMEM is freed.
    commit(&bars.drain);
    __all_sync(0xffffffffu, mbar_wait_drain(&bars.drain, 0, abort, kSiteDrain));
}

// ---------------------------------------------------------------------------
// Wide kernel (head dims 129..256, zero-padded to 256): one query tile at a
// time.  TMEM: S in two buffers (columns 0 and 128) that alternate from key
// block to key block, O at 256..511.  Shared memory: the Q tile (64 KB) and a
// ring of kWideSlots half-tiles (128 rows x 128 columns, 32 KB): K of a block
// is two halves, V one or two (by Dv).  Ring order per tile: K_lo, K_lo+1,
// then V_j, K_j+2 for j = lo .. hi, which is the order the MMA warp uses them.
// ---------------------------------------------------------------------------
constexpr int kWideSlots = 5;
constexpr int kWideThreads = 192;  // softmax warps 0-3, TMA warp 4, MMA warp 5
constexpr int kWideLoadWarp = 4;
constexpr int kWideMmaWarp = 5;
constexpr int kHalfBytes = kTileM * 128 * 2;  // 128 rows x 128 columns
constexpr int kWideQBytes = kTileM * 256 * 2;
constexpr int kWideSmemBytes = kWideQBytes + kWideSlots * kHalfBytes + 1024;
static_assert(kWideSmemBytes + 1024 <= 227 * 1024, "wide kernel tiles exceed shared memory");

__device__ void run_producer_wide(const FaParams& p, const CUtensorMap* tq, const CUtensorMap* tk,
                                  const CUtensorMap* tv, uint8_t* sQ, uint8_t* sKV, Barriers& bars,
                                  TicketSlots& slots, volatile int* abort) {
    constexpr int kChunkBytes = kTileM * 128;
    uint32_t fill = 0, q_fill = 0, k_sched = 0;
    bool ok = true;
    const int v_halves = (p.Dv + 127) / 128;

    while (ok) {
        Item tit;
        const int ticket = take_ticket_global(p, bars, slots, k_sched, tit, abort);
        if (ticket == kTicketAbort) { ok = false; break; }
        if (ticket == kTicketEnd) break;
        const Work wk = work_of(p, ticket, tit);
        const Item it = wk.it;
        auto load_chunk = [&](const CUtensorMap* tm, uint8_t* dst, uint64_t* bar, int c, int row, int head) {
            if (p.varlen)
                tma_load_3d(dst, tm, bar, c * 64, (int)(it.kv_off + row), head);
            else
                tma_load_4d(dst, tm, bar, c * 64, row, head, it.b);
        };
        // one half (columns 128h .. 128h+127) of key block jb of K or V
        auto load_half = [&](const CUtensorMap* tm, int jb, int h) -> bool {
            const int slot = fill % kWideSlots;
            if (!warp_wait(&bars.kv_empty[slot], ((fill / kWideSlots) & 1) ^ 1, abort, kSiteKvEmpty)) return false;
            if (elect_one()) {
                mbar_arrive_expect_tx(&bars.kv_full[slot], kHalfBytes);
                uint8_t* dst = sKV + slot * kHalfBytes;
                load_chunk(tm, dst, &bars.kv_full[slot], 2 * h, jb * kTileN, it.nk);
                load_chunk(tm, dst + kChunkBytes, &bars.kv_full[slot], 2 * h + 1, jb * kTileN, it.nk);
            }
            __syncwarp();
            ++fill;
            return true;
        };
        auto load_k = [&](int jb) { return load_half(tk, jb, 0) && load_half(tk, jb, 1); };
        auto load_v = [&](int jb) {
            for (int h = 0; h < v_halves; ++h)
                if (!load_half(tv, jb, h)) return false;
            return true;
        };
        for (int tt = 0; tt < 2 && ok; ++tt) {
            const TileRange tr = tt ? wk.tr[1] : wk.tr[0];
            if (!tr.active()) continue;
            if (!warp_wait(&bars.q_empty[0], (q_fill & 1) ^ 1, abort, kSiteQEmpty)) { ok = false; break; }
            if (elect_one()) {
                mbar_arrive_expect_tx(&bars.q_full[0], kWideQBytes);
                const int row = it.qb * kQBlock + tt * kTileM;
                for (int c = 0; c < 4; ++c) {
                    if (p.varlen)
                        tma_load_3d(sQ + c * kChunkBytes, tq, &bars.q_full[0], c * 64, (int)(it.q_off + row), it.n);
                    else
                        tma_load_4d(sQ + c * kChunkBytes, tq, &bars.q_full[0], c * 64, row, it.n, it.b);
                }
            }
            __syncwarp();
            ++q_fill;
            if (!load_k(tr.lo) || (tr.lo + 1 <= tr.hi && !load_k(tr.lo + 1))) { ok = false; break; }
            for (int jb = tr.lo; jb <= tr.hi; ++jb) {
                if (!load_v(jb) || (jb + 2 <= tr.hi && !load_k(jb + 2))) { ok = false; break; }
            }
        }
    }
    // Drain: the latest fill of every slot and of Q has landed.
    for (int sl = 0; sl < kWideSlots; ++sl) {
        if ((uint32_t)sl < fill) {
            const uint32_t last = fill - 1 - ((fill - 1 - sl) % kWideSlots);
            mbar_wait_drain(&bars.kv_full[sl], (last / kWideSlots) & 1, abort, kSiteDrain);
        }
    }
    if (q_fill) mbar_wait_drain(&bars.q_full[0], (q_fill - 1) & 1, abort, kSiteDrain);
}

template <typename T>
__device__ void run_mma_wide(const FaParams& p, uint8_t* sQ, uint8_t* sKV, Barriers& bars, const TicketSlots& slots,
                             uint32_t tmem, volatile int* abort) {
    constexpr bool kBf16 = std::is_same<T, __nv_bfloat16>::value;
    constexpr int kChunkBytes = kTileM * 128;
    const uint32_t idesc_qk = idesc_f16(kBf16, kTileM, kTileN, false, false, p.neg_scale != 0);
    constexpr uint32_t idesc_pv = idesc_f16(kBf16, kTileM, 128, false, true, false);
    const int v_halves = (p.Dv + 127) / 128;
    uint32_t use = 0, q_use = 0, p_cnt0 = 0, p_cnt1 = 0, k_sched = 0, g = 0;
    bool ok = true;
    if (p.debug_stall && !warp_wait(&bars.never, 0, abort, kSiteInjected)) ok = false;

    auto wait_half = [&](int* slot) -> bool {
        *slot = use % kWideSlots;
        const bool r = warp_wait(&bars.kv_full[*slot], (use / kWideSlots) & 1, abort, kSiteKvFull);
        ++use;
        return r;
    };
    auto commit = [&](uint64_t* bar) {
        if (elect_one()) tc_commit(bar);
        __syncwarp();
    };
    // S_b = Q · K^T over 256 columns: K-steps 0..7 against K's first half,
    // 8..15 (Q chunks 2, 3) against its second half.
    auto qk = [&](uint32_t b) -> bool {
        int k0, k1;
        if (!wait_half(&k0) || !wait_half(&k1)) return false;
        tc_fence_after();
        const uint64_t qd0 = sdesc_sw128(smem_u32(sQ), 1024, 16);
        const uint64_t qd2 = sdesc_sw128(smem_u32(sQ + 2 * kChunkBytes), 1024, 16);
        const uint64_t kd0 = sdesc_sw128(smem_u32(sKV + k0 * kHalfBytes), 1024, 16);
        const uint64_t kd1 = sdesc_sw128(smem_u32(sKV + k1 * kHalfBytes), 1024, 16);
        if (elect_one()) {
            mma_ss_k128(tmem + b * kTileN, qd0, kd0, idesc_qk, 0u);
            mma_ss_k128(tmem + b * kTileN, qd2, kd1, idesc_qk, 1u);
        }
        __syncwarp();
        commit(&bars.s_full[b]);
        commit(&bars.kv_empty[k0]);
        commit(&bars.kv_empty[k1]);
        return true;
    };

    while (ok) {
        Item tit;
        const int ticket = take_ticket_local(p, bars, slots, k_sched, tit, abort);
        if (ticket == kTicketAbort) { ok = false; break; }
        if (ticket == kTicketEnd) break;
        const Work wk = work_of(p, ticket, tit);
        for (int tt = 0; tt < 2 && ok; ++tt) {
            const TileRange tr = tt ? wk.tr[1] : wk.tr[0];
            if (!tr.active()) continue;
            if (!warp_wait(&bars.q_full[0], q_use & 1, abort, kSiteQFull)) { ok = false; break; }
            ++q_use;
            if (!qk(g & 1)) { ok = false; break; }
            if (tr.lo == tr.hi) commit(&bars.q_empty[0]);
            if (tr.lo + 1 <= tr.hi) {
                if (!qk((g + 1) & 1)) { ok = false; break; }
                if (tr.lo + 1 == tr.hi) commit(&bars.q_empty[0]);
            }
            for (int jb = tr.lo; jb <= tr.hi; ++jb, ++g) {
                const uint32_t b = g & 1;
                int v0 = 0, v1 = 0;
                if (!wait_half(&v0) || (v_halves > 1 && !wait_half(&v1))) { ok = false; break; }
                const uint32_t pc = b ? p_cnt1 : p_cnt0;
                if (!warp_wait(&bars.p_full[b], pc & 1, abort, kSitePFull)) { ok = false; break; }
                if (b) ++p_cnt1; else ++p_cnt0;
                tc_fence_after();
                const uint32_t acc = jb != tr.lo ? 1u : 0u;
                const uint64_t vd0 = sdesc_sw128(smem_u32(sKV + v0 * kHalfBytes), 1024, kChunkBytes);
                if (elect_one()) mma_ts_k128(tmem + 256, tmem + b * kTileN, vd0, idesc_pv, acc);
                __syncwarp();
                if (v_halves > 1) {
                    const uint64_t vd1 = sdesc_sw128(smem_u32(sKV + v1 * kHalfBytes), 1024, kChunkBytes);
                    if (elect_one()) mma_ts_k128(tmem + 384, tmem + b * kTileN, vd1, idesc_pv, acc);
                    __syncwarp();
                }
                commit(&bars.pv_done);
                commit(&bars.kv_empty[v0]);
                if (v_halves > 1) commit(&bars.kv_empty[v1]);
                if (jb == tr.hi) commit(&bars.o_full[0]);
                if (jb + 2 <= tr.hi) {
                    // into the buffer whose P this block's P·V reads: issued after it
                    if (!qk(b)) { ok = false; break; }
                    if (jb + 2 == tr.hi) commit(&bars.q_empty[0]);
                }
            }
        }
    }
    commit(&bars.drain);
    __all_sync(0xffffffffu, mbar_wait_drain(&bars.drain, 0, abort, kSiteDrain));
}

// ---------------------------------------------------------------------------
// Softmax warpgroup t (128 threads; thread r owns query row r of the tile)
// ---------------------------------------------------------------------------

// Two floats rounded to T and packed, `lo` (the lower column) in the low half.
template <typename T>
__device__ __forceinline__ uint32_t pack2(float lo, float hi) {
    if constexpr (std::is_same<T, __nv_bfloat16>::value)
        return pack_bf16x2(lo, hi);
    else
        return pack_f16x2(lo, hi);
}

// Additive bias of 8 consecutive keys starting at j from a dense pse row (query dtype), in natural units.
template <typename T>
__device__ __forceinline__ void load_bias8(const T* row, int j, int kv_len, bool vec, float* out) {
    if (vec && j + 8 <= kv_len) {
        const uint4 u = __ldg(reinterpret_cast<const uint4*>(row + j));
        const T* h = reinterpret_cast<const T*>(&u);
#pragma unroll
        for (int e = 0; e < 8; ++e) out[e] = to_f(h[e]);
    } else {
#pragma unroll
        for (int e = 0; e < 8; ++e) out[e] = (j + e < kv_len) ? to_f(row[j + e]) : 0.f;
    }
}

// Additive bias of 16 consecutive keys starting at j (natural units): one
// 32-byte load when the row allows it, else two 8-key loads.
template <typename T>
__device__ __forceinline__ void load_bias16(const T* row, int j, int kv_len, bool vec32, bool vec, float* out) {
    if (vec32 && j + 16 <= kv_len) {
        uint32_t w[8];
        ld_global_nc_v8(row + j, w);
        const T* h = reinterpret_cast<const T*>(w);
#pragma unroll
        for (int e = 0; e < 16; ++e) out[e] = to_f(h[e]);
    } else {
        load_bias8(row, j, kv_len, vec, out);
        load_bias8(row, j + 8, kv_len, vec, out + 8);
    }
}

// Excluded flags (nonzero) of 16 consecutive keys starting at j from a mask row.
__device__ __forceinline__ uint32_t load_mask16(const uint8_t* row, int j, int cols, bool vec) {
    uint32_t bits = 0;
    if (vec && j + 16 <= cols) {
        const uint4 u = __ldg(reinterpret_cast<const uint4*>(row + j));
        const uint8_t* b = reinterpret_cast<const uint8_t*>(&u);
#pragma unroll
        for (int e = 0; e < 16; ++e) bits |= (b[e] != 0 ? 1u : 0u) << e;
    } else {
#pragma unroll
        for (int e = 0; e < 16; ++e)
            if (j + e < cols && row[j + e] != 0) bits |= 1u << e;
    }
    return bits;
}

// Final statistics of a row from its running max m_run, the max m_used that
// O and l are relative to, and l (all log2 units): the sink joins the max and
// the denominator; o_scale turns O into the output.
struct RowFinal {
    float m_f, l_f, o_scale;
};
__device__ __forceinline__ RowFinal finalize_row(const FaParams& p, const Item& it, float m_run, float m_used, float l) {
    RowFinal f;
    f.m_f = m_run;
    if (p.has_sink) {
        const float sk = p.sink[it.n] * kLog2e;
        f.m_f = fmaxf(m_run, sk);
        const float a = (m_used == -CUDART_INF_F) ? 0.f : ex2(m_used - f.m_f);
        f.l_f = l * a + ex2(sk - f.m_f);
        f.o_scale = a / f.l_f;
    } else {
        f.l_f = l * ((m_used == -CUDART_INF_F) ? 0.f : ex2(m_used - m_run));
        f.o_scale = (l > 0.f) ? 1.f / l : 0.f;
    }
    return f;
}

// 32 output columns of a row (fp32 bits in o) scaled, rounded to T and stored.
template <typename T>
__device__ __forceinline__ void store_out32(const FaParams& p, T* orow, int cc, const uint32_t (&o)[32], float o_scale) {
    uint32_t w[16];
#pragma unroll
    for (int e = 0; e < 16; ++e)
        w[e] = pack2<T>(__uint_as_float(o[2 * e]) * o_scale, __uint_as_float(o[2 * e + 1]) * o_scale);
    if (p.o_vec32) {  // whole 32-byte sectors: half the store requests of 16-byte stores
        st_global_v8(orow + cc, w);
        st_global_v8(orow + cc + 16, w + 8);
    } else if (p.o_vec) {
        uint4* dst = reinterpret_cast<uint4*>(orow + cc);
#pragma unroll
        for (int v = 0; v < 4; ++v) dst[v] = make_uint4(w[4 * v], w[4 * v + 1], w[4 * v + 2], w[4 * v + 3]);
    } else {
        uint32_t* dst = reinterpret_cast<uint32_t*>(orow + cc);
        if ((reinterpret_cast<uintptr_t>(dst) & 3u) == 0) {
#pragma unroll
            for (int e = 0; e < 16; ++e) dst[e] = w[e];
        } else {
            const T* h = reinterpret_cast<const T*>(w);
#pragma unroll
            for (int e = 0; e < 32; ++e) orow[cc + e] = h[e];
        }
    }
}

// The first 8*groups (< 32) output columns from cc of a row: the last, partial
// 32-column group of a value head dim that is a multiple of 8 only.
template <typename T>
__device__ __forceinline__ void store_out8s(const FaParams& p, T* orow, int cc, int groups, const uint32_t (&o)[32],
                                            float o_scale) {
#pragma unroll
    for (int g = 0; g < 3; ++g) {
        if (g >= groups) break;
        uint32_t w[4];
#pragma unroll
        for (int e = 0; e < 4; ++e)
            w[e] = pack2<T>(__uint_as_float(o[8 * g + 2 * e]) * o_scale, __uint_as_float(o[8 * g + 2 * e + 1]) * o_scale);
        if (p.o_vec) {
            *reinterpret_cast<uint4*>(orow + cc + 8 * g) = make_uint4(w[0], w[1], w[2], w[3]);
        } else {
            const T* h = reinterpret_cast<const T*>(w);
#pragma unroll
            for (int e = 0; e < 8; ++e) orow[cc + 8 * g + e] = h[e];
        }
    }
}

// softmaxMax (natural log units) and softmaxSum of query row i, all 8 lanes.
__device__ __forceinline__ void store_stats(const FaParams& p, const Item& it, int i, const RowFinal& f) {
    const int64_t so = it.b * p.st_b + it.n * p.st_n + (it.q_off + i) * p.st_s;
    const float m_nat = f.m_f * kLn2;
    if (p.st_vec32) {
        uint32_t wm[8], wl[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            wm[e] = __float_as_uint(m_nat);
            wl[e] = __float_as_uint(f.l_f);
        }
        st_global_v8(p.smax + so, wm);
        st_global_v8(p.ssum + so, wl);
        return;
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) {
        p.smax[so + e] = m_nat;
        p.ssum[so + e] = f.l_f;
    }
}

// kBias: 0 no bias, 1 dense bias tensor, 2 ALiBi slopes (one variant each, so
// that each kernel carries only its own bias code).
// Two-tile kernels: warpgroup t owns query tile t of every item, S_t at
// columns 128t, O_t at kOCol + tD.  kWide (head dims above 128): the one
// softmax warpgroup takes both tiles of an item in turn; S alternates between
// the buffers at columns 0 and 128 from one key block to the next, O is at
// kOCol, and a rescale of O first waits for the previous block's P·V (pv_done).
template <typename T, int D, int kBias, bool kWide = false>
__device__ void run_softmax(const FaParams& p, Barriers& bars, const TicketSlots& slots, uint32_t tmem,
                            volatile int* abort, int t, uint8_t* sBias = nullptr) {
    const int quad = (threadIdx.x >> 5) & 3;
    const int row = quad * 32 + (threadIdx.x & 31);
    const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
    const uint32_t tO = tmem + lane_off + kOCol + t * D;
    const float sl2 = p.scale_log2;
    const float abs_scale = fabsf(p.scale);  // the MMA negates K for a negative scale
    constexpr bool kAug = !kWide && kBias == 2 && D == 64;  // the ALiBi ramp comes out of the S MMA
    uint32_t s_cnt0 = 0, s_cnt1 = 0, o_cnt = 0, k_sched = 0, g_blk = 0, bf_cnt = 0;
    bool ok = true;
    const bool tma_bias = kBias == 1 && sBias != nullptr && p.pse_tma;  // bias blocks in shared memory

    while (ok) {
        Item tit;
        const int ticket = take_ticket_local(p, bars, slots, k_sched, tit, abort);
        if (ticket == kTicketAbort) { ok = false; break; }
        if (ticket == kTicketEnd) break;
        const Work wk = work_of(p, ticket, tit);
        const Item it = wk.it;
      for (int tt = kWide ? 0 : t; tt <= (kWide ? 1 : t); ++tt) {
        const TileRange tr = tt ? wk.tr[1] : wk.tr[0];  // a select: no indexing of wk by a runtime value
        if (!tr.valid) continue;
        const int r0 = it.qb * kQBlock + tt * kTileM;
        const int i = r0 + row;
        const bool row_ok = i < it.q_len;

        float slope_l2 = 0.f;
        const T* pse_row = nullptr;
        int pse_cols = 0;
        bool pse_vec = false, pse_vec32 = false;
        if constexpr (kBias == 2)
            slope_l2 = static_cast<const float*>(p.pse)[it.b * p.pse_b + it.n * p.pse_n] * kLog2e;
        if constexpr (kBias == 1)
            if (row_ok) {
                pse_row = pse_row_ptr<T>(p, it.b, it.n, it.q_len, it.kv_len, i, &pse_cols);
                pse_vec = p.pse_vec && (reinterpret_cast<uintptr_t>(pse_row) & 15u) == 0;
                pse_vec32 = p.pse_vec && (reinterpret_cast<uintptr_t>(pse_row) & 31u) == 0;
            }
        const uint8_t* mask_row =
            (p.mask_on && row_ok) ? p.mask + it.b * p.mask_b + it.n * p.mask_n + (int64_t)i * p.mask_i : nullptr;

        float m_run = -CUDART_INF_F, m_used = -CUDART_INF_F, l = 0.f;
        uint32_t wnext[3];  // compressed bias: the warp's window values of the coming block
        for (int jb = tr.lo; jb <= tr.hi; ++jb) {
            if constexpr (kBias == 1) {
                // the next block's bias row segment (256 bytes) on its way to L2
                const int jn = (jb + 1) * kTileN;
                if (pse_row && !tma_bias && jb < tr.hi && jn < pse_cols) {
                    prefetch_l2(pse_row + jn);
                    if (jn + 64 < pse_cols) prefetch_l2(pse_row + jn + 64);
                }
            }
            const uint32_t sb = kWide ? (g_blk & 1u) : static_cast<uint32_t>(t);
            const uint32_t sc = (kWide && sb) ? s_cnt1 : s_cnt0;
            if (!warp_wait(&bars.s_full[sb], sc & 1, abort, kSiteSFull)) { ok = false; break; }
            if (kWide && sb) ++s_cnt1; else ++s_cnt0;
            const uint32_t tS = tmem + lane_off + sb * kTileN;
            tc_fence_after();
            float s[128];
            {
                uint32_t sr[128];
                tmem_ld_x128(tS, sr);
#pragma unroll
                for (int c = 0; c < kTileN; ++c) s[c] = __uint_as_float(sr[c]);
            }
            const int j0 = jb * kTileN;
            const bool full = !p.mask_on && (j0 + kTileN <= it.kv_len) && (j0 - (r0 + kTileM - 1) >= -p.pre) &&
                              (j0 + kTileN - 1 - r0 <= p.next);

            // scores in the log2 domain (bias path) and the block's row max
            float m_blk;
            float row_off = 0.f;  // a per-row bias term kept out of s (added to the max and the shift)
            bool linear = false;
            bool scaled = kBias == 0;  // s still holds S (the max and the exponentials multiply by sl2)
            // after the bias: s in log2 units (ALiBi), natural units (bias tensor)
            if constexpr (kBias == 2) {
                // A block wholly on one side of every row's diagonal has
                // -slope·|i - j| = st·c - st·(i - j0) with st = ±slope: a ramp
                // over the columns plus a per-row constant.  With the ramp
                // from the MMA (kAug: S already holds slope·c / scale) a block
                // left of the diagonal needs nothing more.  When the band
                // keeps no key right of a row's diagonal (next + delta <= 0,
                // so j + delta <= i for every kept key), every block is
                // "below" for the keys it keeps, the diagonal block as well:
                // the keys past the diagonal are masked out anyway.
                const int j0g = j0 + p.alibi_delta;  // key positions relative to the query positions
                const bool below = j0g + kTileN - 1 <= r0 || (int64_t)p.next + p.alibi_delta <= 0;
                const bool above = !below && (j0g >= r0 + kTileM - 1 || (int64_t)p.alibi_delta - p.pre >= 0);
                linear = below || above;
                if (linear) {
                    const float st = below ? slope_l2 : -slope_l2;
                    row_off = -st * (float)(i - j0g);
                    if (kAug && below) scaled = true;
                }
                if (linear && !scaled) {
                    const float sr = (below ? slope_l2 : -slope_l2) - (kAug ? slope_l2 : 0.f);  // ramp still to apply
                    float t[8];  // ramp at columns c8 + h, four chains of column pairs
#pragma unroll
                    for (int h = 0; h < 8; ++h) t[h] = sr * (float)h;
                    const float step = 8.f * sr;
#pragma unroll
                    for (int c8 = 0; c8 < kTileN; c8 += 8) {
#pragma unroll
                        for (int h = 0; h < 8; h += 2) {
                            fma2(s[c8 + h], s[c8 + h + 1], s[c8 + h], s[c8 + h + 1], sl2, sl2, t[h], t[h + 1]);
                            add2(t[h], t[h + 1], step, step);
                        }
                    }
                }
            }
            uint32_t brow = 0;  // this thread's row of the block's bias buffer (tma_bias)
            if (tma_bias) {
                const uint32_t slot = bf_cnt & 1;
                if (!warp_wait(&bars.bias_full[t][slot], (bf_cnt >> 1) & 1, abort, kSiteKvFull)) { ok = false; break; }
                brow = smem_u32(sBias + (t * 2 + slot) * (kTileM * kTileN * 2)) + row * 128;
            }
            // Compressed bias, a warp whose 32 rows all lie above the stored
            // rows: row i reads stored row 0 at column j + first - i, so the
            // warp needs 159 consecutive stored values per key block.  They
            // go to shared memory (in the bias buffers, unused for this bias
            // form) as fp32, in four copies shifted by 0..3 values, so that
            // every row's 128 values are four-aligned runs of one copy.  Each
            // lane loads the next block's values while this block runs.
            uint32_t wrow = 0;  // this thread's run in the warp's window (0: no window)
            if (kBias == 1 && sBias != nullptr && p.pse_rows1024) {
                const int first = it.q_len - 1024;
                const int w0 = r0 + quad * 32;
                if (w0 + 31 < first) {
                    const int lane = threadIdx.x & 31;
                    const uint32_t wbase = smem_u32(sBias + (t * 4 + quad) * kWinBytes);
                    const T* srow = static_cast<const T*>(p.pse) + it.b * p.pse_b + it.n * p.pse_n;
                    const int col0 = j0 + first - w0 - 31;  // stored column of window value 0
                    // two stored values per register (raw 16-bit), zero outside the keys
                    auto window_pair = [&](int col_a, int col_b) -> uint32_t {
                        const uint32_t a = (col_a >= 0 && col_a < it.kv_len) ? bits16(srow[col_a]) : 0u;
                        const uint32_t b = (col_b >= 0 && col_b < it.kv_len) ? bits16(srow[col_b]) : 0u;
                        return a | (b << 16);
                    };
                    if (jb == tr.lo) {
#pragma unroll
                        for (int m = 0; m < 3; ++m)
                            wnext[m] = window_pair(col0 + lane + 64 * m, col0 + lane + 64 * m + 32);
                    }
                    __syncwarp();  // every lane has read the previous block's window
#pragma unroll
                    for (int m = 0; m < 6; ++m) {
                        const int x = lane + 32 * m;
                        if (x < kWinLen + 3) {
                            const uint32_t raw = (wnext[m >> 1] >> (16 * (m & 1))) & 0xffffu;
                            const float g = to_f(from_bits16<T>(static_cast<uint16_t>(raw)));
#pragma unroll
                            for (int k = 0; k < 4; ++k)
                                if (x - k >= 0 && x - k < kWinLen)
                                    asm volatile("st.shared.f32 [%0], %1;" ::"r"(wbase + (k * kWinLen + x - k) * 4),
                                                 "f"(g)
                                                 : "memory");
                        }
                    }
                    __syncwarp();
                    if (jb < tr.hi) {  // the next block's values, one block of keys on
#pragma unroll
                        for (int m = 0; m < 3; ++m)
                            wnext[m] = window_pair(col0 + kTileN + lane + 64 * m, col0 + kTileN + lane + 64 * m + 32);
                    }
                    const int x0 = 31 - lane;  // this row's first window value
                    wrow = wbase + ((x0 & 3) * kWinLen + (x0 & ~3)) * 4;
                }
            }
            if (kBias && !linear) {
                const float fi = (float)(i - j0 - p.alibi_delta);
#pragma unroll
                for (int c16 = 0; c16 < kTileN; c16 += 16) {
                    float bias[16];
                    if constexpr (kBias == 2) {
#pragma unroll
                        for (int e = 0; e < 16; ++e) {
                            const float cf = (float)(c16 + e);
                            bias[e] = -slope_l2 * (fabsf(fi - cf) + (kAug ? cf : 0.f));
                        }
                    } else if (tma_bias) {
                        // two 16-byte pieces of the row in a 128-byte-swizzled 64-column box
#pragma unroll
                        for (int k2 = 0; k2 < 2; ++k2) {
                            const int k = ((c16 & 63) >> 3) + k2;
                            const uint4 u = ld_shared_v4(brow + (c16 >> 6) * (kTileM * 128) + ((k ^ (row & 7)) << 4));
                            const T* h = reinterpret_cast<const T*>(&u);
#pragma unroll
                            for (int e = 0; e < 8; ++e) bias[8 * k2 + e] = to_f(h[e]);
                        }
                    } else if (wrow) {
#pragma unroll
                        for (int q4 = 0; q4 < 4; ++q4) {
                            const uint4 u = ld_shared_v4(wrow + (c16 + 4 * q4) * 4);
                            bias[4 * q4] = __uint_as_float(u.x);
                            bias[4 * q4 + 1] = __uint_as_float(u.y);
                            bias[4 * q4 + 2] = __uint_as_float(u.z);
                            bias[4 * q4 + 3] = __uint_as_float(u.w);
                        }
                    } else if (pse_row) {
                        load_bias16(pse_row, j0 + c16, pse_cols, pse_vec32, pse_vec, bias);
                    } else {
#pragma unroll
                        for (int e = 0; e < 16; ++e) bias[e] = 0.f;
                    }
                    // ALiBi terms are in log2 units; a bias tensor's are
                    // natural, so its scores stay natural (unit = log2 e)
                    const float sm = kBias == 2 ? sl2 : abs_scale;
#pragma unroll
                    for (int e = 0; e < 16; e += 2)
                        fma2(s[c16 + e], s[c16 + e + 1], s[c16 + e], s[c16 + e + 1], sm, sm, bias[e], bias[e + 1]);
                }
            }
            if (tma_bias) {  // the buffer may be refilled
                mbar_arrive(&bars.bias_empty[t][bf_cnt & 1]);
                ++bf_cnt;
            }
            if (!full) {
                // keys of this row kept by the sequence end and the band:
                // columns [c_lo, c_hi] of the block (empty when c_hi < c_lo)
                const int c_lo = max(0, i - p.pre - j0);
                const int c_hi = min(min(kTileN - 1, it.kv_len - 1 - j0), i + p.next - j0);
                // kept: 0 <= c - c_lo <= c_hi - c_lo, one unsigned compare
                // (nothing kept: c - (kTileN + 1) wraps above a span of 0)
                const bool any = c_hi >= c_lo;
                const uint32_t span = any ? static_cast<uint32_t>(c_hi - c_lo) : 0u;
                const int base = any ? c_lo : kTileN + 1;
                const bool lo_zero = __all_sync(0xffffffffu, c_lo == 0);  // every lane (mask_row may differ)
                if (mask_row) {
#pragma unroll
                    for (int c16 = 0; c16 < kTileN; c16 += 16) {
                        const uint32_t excl = load_mask16(mask_row, j0 + c16, p.mask_cols, p.mask_vec != 0);
#pragma unroll
                        for (int e = 0; e < 16; ++e) {
                            const int c = c16 + e;
                            const bool keep = static_cast<uint32_t>(c - base) <= span && ((excl >> e) & 1u) == 0u;
                            s[c] = keep ? s[c] : -CUDART_INF_F;
                        }
                    }
                } else if (lo_zero) {
                    // the usual partial block (a causal diagonal, the keys'
                    // end): one compare and one select per column
#pragma unroll
                    for (int c = 0; c < kTileN; ++c) s[c] = c <= c_hi ? s[c] : -CUDART_INF_F;
                } else {
#pragma unroll
                    for (int c = 0; c < kTileN; ++c)
                        s[c] = static_cast<uint32_t>(c - base) <= span ? s[c] : -CUDART_INF_F;
                }
            }
            {
                // eight chains: columns 0..15 seed them, pairs of 16..127 feed them
                float mc[8];
#pragma unroll
                for (int h = 0; h < 8; ++h) mc[h] = fmaxf(s[2 * h], s[2 * h + 1]);
#pragma unroll
                for (int c = 16; c < kTileN; c += 16)
#pragma unroll
                    for (int h = 0; h < 8; ++h) mc[h] = max3(mc[h], s[c + 2 * h], s[c + 2 * h + 1]);
                m_blk = max3(max3(mc[0], mc[1], mc[2]), max3(mc[3], mc[4], mc[5]), fmaxf(mc[6], mc[7]));
                if (scaled) m_blk *= sl2;
                if (kBias == 1) m_blk *= kLog2e;
                m_blk += row_off;
            }

            const float m_new = fmaxf(m_run, m_blk);
            const bool need = (m_new - m_used) > kRescaleThreshold;  // false while both are -inf
            const float alpha = need ? ex2(m_used - m_new) : 1.f;    // 0 when m_used is -inf
            if (need) {
                l *= alpha;
                m_used = m_new;
            }
            m_run = m_new;
            const float shift = (m_used == -CUDART_INF_F) ? 0.f : m_used;

            // p = 2^(x - shift), two columns per packed FMA / ADD / convert;
            // kPolyPairs of every 8 column pairs take the FMA-pipe exponential
            // (spread over the 8), the others MUFU's ex2
            float l0 = 0.f, l1 = 0.f, l2 = 0.f, l3 = 0.f;
            const float mult = scaled ? sl2 : (kBias == 1 ? kLog2e : 1.f);
            const float nshift = row_off - shift;
            // Rescale O_t by alpha before this block's P·V reaches it.  Two
            // tiles: O_t is stable, the commit behind this block's S_t covered
            // the last P·V.  Wide: wait for the previous block's P·V first.
            const bool rescale = jb > tr.lo && __any_sync(0xffffffffu, need);
            auto rescale_o = [&]() {
#pragma unroll
                for (int cc = 0; cc < D; cc += 32) {
                    if (cc >= p.Dv) break;
                    uint32_t o[32];
                    tmem_ld_x32(tO + cc, o);
#pragma unroll
                    for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
                    tmem_st_x32(tO + cc, o);
                }
            };
            // P goes to TMEM in two halves of 64 columns (only one half's
            // packed values live at a time).  Two tiles: p_half releases the
            // first half's P·V (over keys 0..63) while the second half of
            // the exponentials runs.
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                uint32_t pk[32];
#pragma unroll
                for (int c4 = 0; c4 < 64; c4 += 4) {
                    const int c = 64 * h + c4;
                    float x0, x1, x2, x3, e0, e1, e2, e3;
                    fma2(x0, x1, s[c], s[c + 1], mult, mult, nshift, nshift);
                    fma2(x2, x3, s[c + 2], s[c + 3], mult, mult, nshift, nshift);
                    constexpr int P = kPolyPairs<D>;
                    if (((c / 2) * P) % 8 < P) {
                        exp2_fma2(x0, x1, e0, e1);
                    } else {
                        e0 = ex2(x0);
                        e1 = ex2(x1);
                    }
                    if (((c / 2 + 1) * P) % 8 < P) {
                        exp2_fma2(x2, x3, e2, e3);
                    } else {
                        e2 = ex2(x2);
                        e3 = ex2(x3);
                    }
                    add2(l0, l1, e0, e1);
                    add2(l2, l3, e2, e3);
                    pk[c4 / 2] = pack2<T>(e0, e1);
                    pk[c4 / 2 + 1] = pack2<T>(e2, e3);
                }
                tmem_st_x32(tS + 32 * h, pk);
                if constexpr (!kWide) {
                    if (h == 0) {
                        if (rescale) rescale_o();
                        tmem_wait_st();
                        tc_fence_before();
                        mbar_arrive(&bars.p_half[sb]);
                    }
                }
            }
            l += (l0 + l1) + (l2 + l3);
            if (kWide && rescale) {
                if (!warp_wait(&bars.pv_done, (g_blk - 1) & 1, abort, kSiteOFull)) { ok = false; break; }
                tc_fence_after();
                rescale_o();
            }
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(&bars.p_full[sb]);
            if (kWide) ++g_blk;
        }
        if (!ok) break;

        // ---- epilogue: sink, normalisation, statistics ----------------------
        const bool has_blocks = tr.hi >= tr.lo;
        if (has_blocks) {
            if (!warp_wait(&bars.o_full[t], o_cnt & 1, abort, kSiteOFull)) { ok = false; break; }
            ++o_cnt;
            tc_fence_after();
        }
        if (wk.piece >= 0) {
            // A piece of a split item: keep O_t (relative to m_used) and the
            // row's m_run, m_used, l for the merge.
            float* prow = p.part + ((static_cast<size_t>(wk.tail) * p.n_pieces + wk.piece) * kQBlock + tt * kTileM + row) *
                                       static_cast<size_t>(D + 4);
#pragma unroll 1
            for (int cc = 0; cc < D; cc += 32) {
                uint32_t o[32];
                if (has_blocks) {
                    tmem_ld_x32(tO + cc, o);
                } else {
#pragma unroll
                    for (int e = 0; e < 32; ++e) o[e] = 0u;
                }
                float4* dst = reinterpret_cast<float4*>(prow + cc);
#pragma unroll
                for (int v = 0; v < 8; ++v)
                    dst[v] = make_float4(__uint_as_float(o[4 * v]), __uint_as_float(o[4 * v + 1]),
                                         __uint_as_float(o[4 * v + 2]), __uint_as_float(o[4 * v + 3]));
            }
            *reinterpret_cast<float4*>(prow + D) = make_float4(m_run, m_used, l, 0.f);
            continue;
        }
        const RowFinal f = finalize_row(p, it, m_run, m_used, l);
        T* orow = static_cast<T*>(p.o) + it.b * p.o_b + it.n * p.o_n + (it.q_off + i) * p.o_s;
#pragma unroll 1
        for (int cc = 0; cc < p.Dv; cc += 32) {
            uint32_t o[32];
            if (has_blocks) {
                tmem_ld_x32(tO + cc, o);
            } else {
#pragma unroll
                for (int e = 0; e < 32; ++e) o[e] = 0u;
            }
            if (!row_ok) continue;
            if (cc + 32 <= p.Dv)
                store_out32<T>(p, orow, cc, o, f.o_scale);
            else
                store_out8s<T>(p, orow, cc, (p.Dv - cc) / 8, o, f.o_scale);
        }
        if (row_ok) store_stats(p, it, i, f);
      }
    }
}

// ---------------------------------------------------------------------------
// Merge of split items: the online-softmax combination of the pieces' partial
// results (applied to whole pieces instead of key blocks), then the same row
// finish as the softmax epilogue.  One thread per (query row, 8 output
// columns): a warp reads two rows' partials in 32-byte runs.
// ---------------------------------------------------------------------------
template <typename T, int D>
__global__ void __launch_bounds__(kMergeThreads) fa_merge_kernel(const FaParams p) {
    constexpr int kGroups = D / 8;
    const int n_split = (p.n_tickets - p.n_whole) / p.n_pieces;
    const int idx = blockIdx.x * kMergeThreads + threadIdx.x;
    if (idx >= n_split * kQBlock * kGroups) return;
    const int g = idx % kGroups;
    if (8 * g >= p.Dv) return;  // padding columns of a value head dim below D
    const int rr = idx / kGroups;
    const int r = rr % kQBlock, u = rr / kQBlock;
    const Item it = decode_item(p, p.n_whole + u);
    const int i = it.qb * kQBlock + r;
    if (i >= it.q_len) return;
    const size_t words = D + 4;
    const float* base = p.part + (static_cast<size_t>(u) * p.n_pieces * kQBlock + r) * words;
    const size_t piece_stride = static_cast<size_t>(kQBlock) * words;
    float m_run = -CUDART_INF_F, m_used = -CUDART_INF_F;
    for (int j = 0; j < p.n_pieces; ++j) {
        const float4 st = *reinterpret_cast<const float4*>(base + j * piece_stride + D);
        m_run = fmaxf(m_run, st.x);
        m_used = fmaxf(m_used, st.y);
    }
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    float l = 0.f;
    if (m_used != -CUDART_INF_F) {
#pragma unroll 4
        for (int j = 0; j < p.n_pieces; ++j) {
            const float* pr = base + j * piece_stride;
            const float4 st = *reinterpret_cast<const float4*>(pr + D);
            const float4 o0 = *reinterpret_cast<const float4*>(pr + 8 * g);
            const float4 o1 = *reinterpret_cast<const float4*>(pr + 8 * g + 4);
            // a piece that saw no key of this row has m_used = -inf: weight 0
            const float w = (st.y == -CUDART_INF_F) ? 0.f : ex2(st.y - m_used);
            l = fmaf(st.z, w, l);
            acc[0] = fmaf(o0.x, w, acc[0]);
            acc[1] = fmaf(o0.y, w, acc[1]);
            acc[2] = fmaf(o0.z, w, acc[2]);
            acc[3] = fmaf(o0.w, w, acc[3]);
            acc[4] = fmaf(o1.x, w, acc[4]);
            acc[5] = fmaf(o1.y, w, acc[5]);
            acc[6] = fmaf(o1.z, w, acc[6]);
            acc[7] = fmaf(o1.w, w, acc[7]);
        }
    }
    const RowFinal f = finalize_row(p, it, m_run, m_used, l);
    T* orow = static_cast<T*>(p.o) + it.b * p.o_b + it.n * p.o_n + (it.q_off + i) * p.o_s + 8 * g;
    uint32_t w4[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) w4[e] = pack2<T>(acc[2 * e] * f.o_scale, acc[2 * e + 1] * f.o_scale);
    if (p.o_vec) {
        *reinterpret_cast<uint4*>(orow) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
    } else {
        const T* h = reinterpret_cast<const T*>(w4);
#pragma unroll
        for (int e = 0; e < 8; ++e) orow[e] = h[e];
    }
    if (g == 0) store_stats(p, it, i, f);
}

// ---------------------------------------------------------------------------
// Kernel
// ---------------------------------------------------------------------------
template <typename T, int D, int kBias, bool kRope>
__global__ void __launch_bounds__(kThreads, 1)
    fa_fwd_sm100_kernel(const __grid_constant__ CUtensorMap tmap_q, const __grid_constant__ CUtensorMap tmap_k,
                        const __grid_constant__ CUtensorMap tmap_v, const __grid_constant__ CUtensorMap tmap_qr,
                        const __grid_constant__ CUtensorMap tmap_kr, const __grid_constant__ CUtensorMap tmap_pse,
                        const FaParams p) {
    constexpr bool kAug = kAugRamp<D, kBias, kRope>;
    constexpr bool kTmaBias = kTmaBiasK<D, kBias, kRope>;
    using C = Cfg<D, kRope, kAug, kTmaBias>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sQ = smem;
    uint8_t* sKV = smem + 2 * C::kQTileBytes;
    uint8_t* sKr = sKV + C::kStages * C::kTileBytes;
    uint8_t* sAug = sKr + C::kRopeSlots * C::kChunkBytes;
    uint8_t* sBias = sAug + C::kAugBytes;
    __shared__ Barriers bars;
    __shared__ TicketSlots slots;
    __shared__ uint32_t tmem_base;
    __shared__ int abort_flag;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int t = 0; t < 2; ++t) {
            mbar_init(&bars.q_full[t], 1);
            mbar_init(&bars.q_empty[t], 1);
            mbar_init(&bars.s_full[t], 1);
            mbar_init(&bars.p_full[t], kTileM);
            mbar_init(&bars.p_half[t], kTileM);
            for (int k = 0; k < 2; ++k) {
                mbar_init(&bars.bias_full[t][k], 1);
                mbar_init(&bars.bias_empty[t][k], kTileM);
            }
            mbar_init(&bars.o_full[t], 1);
        }
        for (int s = 0; s < C::kStages; ++s) {
            mbar_init(&bars.kv_full[s], 1);
            mbar_init(&bars.kv_empty[s], 1);
        }
        for (int r = 0; r < 2; ++r) mbar_init(&bars.kr_empty[r], 1);
        for (int k = 0; k < kSched; ++k) {
            mbar_init(&bars.sched_full[k], 1);
            mbar_init(&bars.sched_empty[k], kTicketReaders);
        }
        mbar_init(&bars.drain, 1);
        mbar_init(&bars.never, 1);
        abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == kLoadWarp && lane == 0) {
        prefetch_tmap(&tmap_q);
        prefetch_tmap(&tmap_k);
        prefetch_tmap(&tmap_v);
        if (kRope) {
            prefetch_tmap(&tmap_qr);
            prefetch_tmap(&tmap_kr);
        }
        if (kTmaBias && p.pse_tma) prefetch_tmap(&tmap_pse);
    }
    if (warp == kMmaWarp) {
        tmem_alloc(&tmem_base, C::kTmemCols);
        tmem_relinquish();
    }
    if constexpr (kAug) {
        // ALiBi ramp chunks: the Q tiles' ramp chunks zero (the producer
        // writes each item's slope terms into piece 0 of every row); the
        // fixed key chunk (c, c, c) in piece 0 of row c, zero elsewhere
        if (threadIdx.x < 2 * kTileM) {
            const int t = threadIdx.x / kTileM, r = threadIdx.x % kTileM;
            const uint32_t qa = smem_u32(sQ + t * C::kQTileBytes + C::kTileBytes) + r * 128;
            for (int k = 0; k < 8; ++k) st_shared_v4(qa + k * 16, 0u, 0u, 0u, 0u);
            if (t == 0) {
                const uint32_t ka = smem_u32(sAug);
                const uint32_t cc = static_cast<uint32_t>(bits16(static_cast<T>(static_cast<float>(r))));
                for (int k = 0; k < 8; ++k) st_shared_v4(ka + sw128_offset(r, k), 0u, 0u, 0u, 0u);
                st_shared_v4(ka + sw128_offset(r, 0), cc | (cc << 16), cc, 0u, 0u);
            }
        }
        fence_proxy_async_smem();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_base;

    if (warp < 8) {
        setmaxnreg_inc<kSoftmaxRegs<kRope || kAug || kTmaBias>>();
        run_softmax<T, D, kBias>(p, bars, slots, tmem, &abort_flag, warp >> 2, kTmaBias ? sBias : nullptr);
    } else {
        setmaxnreg_dec<kOtherRegs<kRope || kAug || kTmaBias>>();
        if (warp == kLoadWarp)
            run_producer<T, D, kRope, kAug, kTmaBias>(p, &tmap_q, &tmap_k, &tmap_v, &tmap_qr, &tmap_kr, &tmap_pse, sQ,
                                                      sKV, sKr, sBias, bars, slots, &abort_flag);
        else if (warp == kMmaWarp)
            run_mma<T, D, kRope, kAug, kTmaBias>(p, sQ, sKV, sKr, sAug, bars, slots, tmem, &abort_flag);
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == kMmaWarp) tmem_dealloc(tmem, C::kTmemCols);
    if (threadIdx.x == 0 && abort_flag != 0)
        atomicCAS(&g_fa_error, 0ull, (static_cast<unsigned long long>(abort_flag) << 32) | (blockIdx.x + 1u));
}

// Wide kernel: head dims 129..256 (see run_producer_wide).
template <typename T, int kBias>
__global__ void __launch_bounds__(kWideThreads, 1)
    fa_fwd_sm100_wide_kernel(const __grid_constant__ CUtensorMap tmap_q, const __grid_constant__ CUtensorMap tmap_k,
                             const __grid_constant__ CUtensorMap tmap_v, const FaParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sQ = smem;
    uint8_t* sKV = smem + kWideQBytes;
    __shared__ Barriers bars;
    __shared__ TicketSlots slots;
    __shared__ uint32_t tmem_base;
    __shared__ int abort_flag;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        mbar_init(&bars.q_full[0], 1);
        mbar_init(&bars.q_empty[0], 1);
        mbar_init(&bars.o_full[0], 1);
        for (int b = 0; b < 2; ++b) {
            mbar_init(&bars.s_full[b], 1);
            mbar_init(&bars.p_full[b], kTileM);
        }
        for (int sl = 0; sl < kWideSlots; ++sl) {
            mbar_init(&bars.kv_full[sl], 1);
            mbar_init(&bars.kv_empty[sl], 1);
        }
        for (int k = 0; k < kSched; ++k) {
            mbar_init(&bars.sched_full[k], 1);
            mbar_init(&bars.sched_empty[k], 5);  // the MMA warp and the four softmax warps
        }
        mbar_init(&bars.pv_done, 1);
        mbar_init(&bars.drain, 1);
        mbar_init(&bars.never, 1);
        abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == kWideLoadWarp && lane == 0) {
        prefetch_tmap(&tmap_q);
        prefetch_tmap(&tmap_k);
        prefetch_tmap(&tmap_v);
    }
    if (warp == kWideMmaWarp) {
        tmem_alloc(&tmem_base, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_base;

    if (warp < 4)
        run_softmax<T, 256, kBias, true>(p, bars, slots, tmem, &abort_flag, 0);
    else if (warp == kWideLoadWarp)
        run_producer_wide(p, &tmap_q, &tmap_k, &tmap_v, sQ, sKV, bars, slots, &abort_flag);
    else if (warp == kWideMmaWarp)
        run_mma_wide<T>(p, sQ, sKV, bars, slots, tmem, &abort_flag);

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == kWideMmaWarp) tmem_dealloc(tmem, 512);
    if (threadIdx.x == 0 && abort_flag != 0)
        atomicCAS(&g_fa_error, 0ull, (static_cast<unsigned long long>(abort_flag) << 32) | (blockIdx.x + 1u));
}

template <typename T, int kBias>
cudaError_t launch_wide(const FaParams& p, const TmaSet& maps, cudaStream_t stream) {
    auto kern = fa_fwd_sm100_wide_kernel<T, kBias>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kWideSmemBytes);
    if (e != cudaSuccess) return e;
    if (p.grid <= 0) return cudaSuccess;
    auto map = [](const TmaDesc& d) -> const CUtensorMap& { return *reinterpret_cast<const CUtensorMap*>(&d); };
    kern<<<p.grid, kWideThreads, kWideSmemBytes, stream>>>(map(maps.q), map(maps.k), map(maps.v), p);
    e = cudaGetLastError();
    if (e != cudaSuccess || p.n_pieces == 0) return e;
    const int n_split = (p.n_tickets - p.n_whole) / p.n_pieces;
    const int merge_threads = n_split * kQBlock * (256 / 8);
    fa_merge_kernel<T, 256><<<(merge_threads + kMergeThreads - 1) / kMergeThreads, kMergeThreads, 0, stream>>>(p);
    return cudaGetLastError();
}

template <typename T, int D, int kBias, bool kRope = false>
cudaError_t launch_t(const FaParams& p, const TmaSet& maps, int num_sms, cudaStream_t stream) {
    using C = Cfg<D, kRope, kAugRamp<D, kBias, kRope>, kTmaBiasK<D, kBias, kRope>>;
    auto kern = fa_fwd_sm100_kernel<T, D, kBias, kRope>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
    if (e != cudaSuccess) return e;
    // setmaxnreg.inc can only hand out what the launch reserved: refuse to
    // launch (instead of waiting forever) if the compiled register count is
    // below the split's total.
    cudaFuncAttributes attr{};
    e = cudaFuncGetAttributes(&attr, kern);
    if (e != cudaSuccess) return e;
    constexpr bool kMore = kRope || kAugRamp<D, kBias, kRope> || kTmaBiasK<D, kBias, kRope>;
    if (static_cast<uint64_t>(attr.numRegs) * kThreads < 2ull * 128 * kSoftmaxRegs<kMore> + 128ull * kOtherRegs<kMore>)
        return cudaErrorLaunchOutOfResources;
    (void)num_sms;
    if (p.grid <= 0) return cudaSuccess;
    auto map = [](const TmaDesc& d) -> const CUtensorMap& { return *reinterpret_cast<const CUtensorMap*>(&d); };
    FaParams pl = p;
    pl.pse_tma = (kTmaBiasK<D, kBias, kRope> && maps.pse_ok) ? 1 : 0;
    kern<<<p.grid, kThreads, C::kSmemBytes, stream>>>(map(maps.q), map(maps.k), map(maps.v), map(maps.qr),
                                                      map(maps.kr), map(maps.pse), pl);
    e = cudaGetLastError();
    if (e != cudaSuccess || p.n_pieces == 0) return e;
    const int n_split = (p.n_tickets - p.n_whole) / p.n_pieces;
    const int merge_threads = n_split * kQBlock * (D / 8);
    fa_merge_kernel<T, D><<<(merge_threads + kMergeThreads - 1) / kMergeThreads, kMergeThreads, 0, stream>>>(p);
    return cudaGetLastError();
}

template <typename T>
cudaError_t launch_d(const FaParams& p, const TmaSet& maps, int num_sms, cudaStream_t stream) {
    // pse_type is 0 whenever realShift is absent; rope (bf16 only, no
    // realShift) has kernels of its own
    // head dims up to 64 run on the 64-column kernels, up to 128 on the
    // 128-column ones, up to 256 on the wide kernel (columns past D and Dv
    // load as zero)
    if (p.D > 128) {
        if (p.pse_type == 2) return launch_wide<T, 2>(p, maps, stream);
        if (p.pse_type == 1) return launch_wide<T, 1>(p, maps, stream);
        return launch_wide<T, 0>(p, maps, stream);
    }
    if constexpr (std::is_same<T, __nv_bfloat16>::value) {
        if (p.Dr) {
            if (p.D > 64) return launch_t<T, 128, 0, true>(p, maps, num_sms, stream);
            return launch_t<T, 64, 0, true>(p, maps, num_sms, stream);
        }
    }
    if (p.D > 64) {
        if (p.pse_type == 2) return launch_t<T, 128, 2>(p, maps, num_sms, stream);
        if (p.pse_type == 1) return launch_t<T, 128, 1>(p, maps, num_sms, stream);
        return launch_t<T, 128, 0>(p, maps, num_sms, stream);
    }
    if (p.pse_type == 2) return launch_t<T, 64, 2>(p, maps, num_sms, stream);
    if (p.pse_type == 1) return launch_t<T, 64, 1>(p, maps, num_sms, stream);
    return launch_t<T, 64, 0>(p, maps, num_sms, stream);
}

// ---------------------------------------------------------------------------
// Tensor maps (host)
// ---------------------------------------------------------------------------
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q{};
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &f, 12000, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(f);
    });
    return fn;
}

// Byte stride of a dimension; a size-1 dimension's stride never matters, so
// any legal value (16) stands in for it.
cuuint64_t stride_bytes(int64_t elems, int64_t size) {
    return size == 1 ? 16 : static_cast<cuuint64_t>(elems) * 2;
}

// Box of 64 columns (128 bytes, the swizzle span) x 128 rows; 128-byte swizzle;
// out-of-range rows, and columns past `cols` (a head dim below the kernel's
// 64 / 128), read as zero.
cudaError_t encode(TmaDesc* out, const FaParams& p, const void* base, int cols, int rows, int heads,
                   int64_t s_stride, int64_t n_stride, int64_t b_stride) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return cudaErrorNotSupported;
    const CUtensorMapDataType dt = p.dtype == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
    CUresult r;
    if (p.varlen) {
        const cuuint64_t dims[3] = {(cuuint64_t)cols, (cuuint64_t)rows, (cuuint64_t)heads};
        const cuuint64_t strides[2] = {stride_bytes(s_stride, rows), stride_bytes(n_stride, heads)};
        const cuuint32_t box[3] = {64, 128, 1};
        const cuuint32_t es[3] = {1, 1, 1};
        r = fn(reinterpret_cast<CUtensorMap*>(out), dt, 3, const_cast<void*>(base), dims, strides, box, es,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    } else {
        const cuuint64_t dims[4] = {(cuuint64_t)cols, (cuuint64_t)rows, (cuuint64_t)heads, (cuuint64_t)p.B};
        const cuuint64_t strides[3] = {stride_bytes(s_stride, rows), stride_bytes(n_stride, heads),
                                       stride_bytes(b_stride, p.B)};
        const cuuint32_t box[4] = {64, 128, 1, 1};
        const cuuint32_t es[4] = {1, 1, 1, 1};
        r = fn(reinterpret_cast<CUtensorMap*>(out), dt, 4, const_cast<void*>(base), dims, strides, box, es,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    }
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

}  // namespace

cudaError_t make_sm100_tmaps(const FaParams& p, TmaSet* maps) {
    cudaError_t e = encode(&maps->q, p, p.q, p.D, p.Tq, p.Nq, p.q_s, p.q_n, p.q_b);
    if (e == cudaSuccess) e = encode(&maps->k, p, p.k, p.D, p.Tkv, p.Nkv, p.k_s, p.k_n, p.k_b);
    if (e == cudaSuccess) e = encode(&maps->v, p, p.v, p.Dv, p.Tkv, p.Nkv, p.v_s, p.v_n, p.v_b);
    if (e != cudaSuccess) return e;
    // a dense bias [B|1, N|1, Sq, Skv] (not the compressed or flattened forms):
    // 64 x 128 boxes for the head-dim-64 kernels' bias buffers
    maps->pse = maps->q;
    maps->pse_ok = 0;
    if (p.pse_type == 1 && !p.pse_rows1024 && !p.pse_flat && !p.varlen &&
        (reinterpret_cast<uintptr_t>(p.pse) & 15u) == 0 && p.pse_i % 8 == 0 && p.pse_n % 8 == 0 && p.pse_b % 8 == 0) {
        EncodeTiledFn fn = encode_fn();
        const cuuint64_t nb = p.pse_n ? (cuuint64_t)p.Nq : 1, bb = p.pse_b ? (cuuint64_t)p.B : 1;
        const cuuint64_t dims[4] = {(cuuint64_t)p.Skv, (cuuint64_t)p.Sq, nb, bb};
        const cuuint64_t strides[3] = {stride_bytes(p.pse_i, p.Sq), p.pse_n ? (cuuint64_t)p.pse_n * 2 : 16,
                                       p.pse_b ? (cuuint64_t)p.pse_b * 2 : 16};
        const cuuint32_t box[4] = {64, 128, 1, 1};
        const cuuint32_t es[4] = {1, 1, 1, 1};
        const CUtensorMapDataType dt =
            p.dtype == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
        if (fn && fn(reinterpret_cast<CUtensorMap*>(&maps->pse), dt, 4, const_cast<void*>(p.pse), dims, strides, box,
                     es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS)
            maps->pse_ok = 1;
        else
            maps->pse = maps->q;
    }
    if (p.Dr) {
        e = encode(&maps->qr, p, p.qr, p.Dr, p.Tq, p.Nq, p.qr_s, p.qr_n, p.qr_b);
        if (e == cudaSuccess) e = encode(&maps->kr, p, p.kr, p.Dr, p.Tkv, p.Nkv, p.kr_s, p.kr_n, p.kr_b);
    } else {
        maps->qr = maps->q;
        maps->kr = maps->k;
    }
    return e;
}

uint64_t plan_sm100_schedule(FaParams& p, int num_sms, bool uniform, int item_kv_blocks) {
    p.grid = p.n_items < num_sms ? p.n_items : num_sms;
    p.n_whole = p.n_tickets = p.n_items;
    p.n_pieces = 0;
    p.dynamic = uniform ? 0 : 1;  // unequal items: CTAs take the next ticket when free
    if (!uniform || p.grid <= 0 || p.n_items <= p.grid) return 0;
    // Equal items leave a last wave of n_items % grid items on a few SMs; split
    // those items into key pieces so that the last wave spreads over the grid.
    const int tail = p.n_items % p.grid;
    if (tail == 0) return 0;
    int pieces = p.grid / tail;
    if (pieces > item_kv_blocks) pieces = item_kv_blocks;
    if (pieces < 2) return 0;
    p.n_whole = p.n_items - tail;
    p.n_pieces = pieces;
    p.n_tickets = p.n_whole + tail * pieces;
    const int d_pad = p.D > 128 ? 256 : (p.D > 64 ? 128 : 64);
    return static_cast<uint64_t>(tail) * pieces * kQBlock * part_row_words(d_pad) * sizeof(float);
}

cudaError_t launch_sm100(const FaParams& p, const TmaSet& maps, int num_sms, cudaStream_t stream) {
    if (p.dtype == 2) return launch_d<__nv_bfloat16>(p, maps, num_sms, stream);
    return launch_d<__half>(p, maps, num_sms, stream);
}

uint64_t read_and_clear_device_error(cudaError_t* err) {
    unsigned long long word = 0, zero = 0;
    cudaError_t e = cudaDeviceSynchronize();
    if (e == cudaSuccess) e = cudaMemcpyFromSymbol(&word, g_fa_error, sizeof(word));
    if (e == cudaSuccess && word) e = cudaMemcpyToSymbol(g_fa_error, &zero, sizeof(zero));
    if (err) *err = e;
    return word;
}

}  // namespace fa
