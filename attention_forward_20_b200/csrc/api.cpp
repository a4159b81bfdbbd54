// Host side of the C ABI: argument validation, layout -> stride resolution,
// kernel choice, the varlen work table, and the launch.
//
// Validation follows the two-stage contract of the aclnnFlashAttentionScore and
// aclnnFlashAttentionVarLenScoreV5 pages ("返回值": 161001 for a NULL required
// argument, 161002 for an unsupported dtype or format, 561103 for a shape or
// attribute out of range; "约束说明" for the shape limits, the GQA ratio, the
// band intersection rule and the cumulative actualSeq*Len form).
#include "fa_fwd.h"
#include "fa_params.h"

#include <algorithm>
#include <cmath>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <new>
#include <string>
#include <vector>

struct fa_executor {
    fa::FaParams p;
    int kind = fa::KERNEL_SIMT;
    std::vector<int64_t> cu;   // TND: cu_q[B+1] then cu_kv[B+1], each with a leading 0
    std::vector<int4> table;   // TND, tcgen05 kernel: one entry per (sequence, query block)
    uint64_t off_cu = 0;
    uint64_t off_table = 0;
    uint64_t off_part = 0;
    uint64_t ws_bytes = 0;
    std::string desc;
};

namespace {

enum Layout { L_BSH, L_SBH, L_BSND, L_BNSD, L_TND };

constexpr int64_t kMaxB = 20000;       // aclnnFlashAttentionVarLenScoreV5, 约束说明: B 1~20000
constexpr int64_t kMaxN = 256;         // N 1~256
constexpr int64_t kMaxS = 1 << 20;     // S, T 1~1M
constexpr int64_t kMaxD = 256;         // this library: head dim up to 256
constexpr int kQBlock = 256;           // tcgen05 kernel: two 128-row query tiles per work item
constexpr int kKvBlock = 128;
constexpr uint64_t kScheduleHeader = 256; // tcgen05 kernel: ticket counter at workspace offset 0
constexpr int kDefaultSms = 148;          // B200

bool parse_layout(const char* s, Layout* out) {
    if (s == nullptr) return false;
    static const struct { const char* name; Layout l; } names[] = {
        {"BSH", L_BSH}, {"SBH", L_SBH}, {"BSND", L_BSND}, {"BNSD", L_BNSD}, {"TND", L_TND}};
    for (const auto& n : names)
        if (std::strcmp(s, n.name) == 0) { *out = n.l; return true; }
    return false;
}

bool is_float_dtype(int32_t d) { return d == FA_F32 || d == FA_F16 || d == FA_BF16; }

// Logical view of a query/key/value/out tensor: sizes and element strides of
// (b, n, s); the head-dim stride is 1.
struct View {
    int64_t B = 0, N = 0, S = 0, D = 0;
    int64_t sb = 0, sn = 0, ss = 0;
};

// heads > 0: the head count is known (query); else head_dim > 0 is known
// (key from query's D, value from key's head count via heads).
fa_status make_view(const fa_tensor* t, Layout L, int64_t heads, int64_t head_dim, View* v) {
    const bool four = (L == L_BSND || L == L_BNSD);
    if (t->ndim != (four ? 4 : 3)) return FA_ERR_INNER_NULLPTR;
    for (int i = 0; i < t->ndim; ++i)
        if (t->shape[i] < 1 || t->strides[i] < 0) return FA_ERR_INNER_NULLPTR;
    if (t->strides[t->ndim - 1] != 1) return FA_ERR_INNER_NULLPTR;
    const int64_t* sh = t->shape;
    const int64_t* st = t->strides;
    switch (L) {
        case L_BNSD: *v = {sh[0], sh[1], sh[2], sh[3], st[0], st[1], st[2]}; break;
        case L_BSND: *v = {sh[0], sh[2], sh[1], sh[3], st[0], st[2], st[1]}; break;
        case L_TND:  *v = {0, sh[1], sh[0], sh[2], 0, st[1], st[0]}; break;
        case L_BSH:
        case L_SBH: {
            const int64_t H = sh[2];
            int64_t N, D;
            if (heads > 0) { if (H % heads) return FA_ERR_INNER_NULLPTR; N = heads; D = H / heads; }
            else { if (head_dim <= 0 || H % head_dim) return FA_ERR_INNER_NULLPTR; D = head_dim; N = H / head_dim; }
            if (L == L_BSH) *v = {sh[0], N, sh[1], D, st[0], D, st[1]};
            else            *v = {sh[1], N, sh[0], D, st[1], D, st[0]};
            break;
        }
    }
    return FA_SUCCESS;
}

bool same_shape(const fa_tensor* t, std::initializer_list<int64_t> dims) {
    if (t->ndim != (int)dims.size()) return false;
    int i = 0;
    for (int64_t d : dims) if (t->shape[i++] != d) return false;
    return true;
}

int64_t clamp64(int64_t x, int64_t lo, int64_t hi) { return x < lo ? lo : (x > hi ? hi : x); }

// 128-key blocks of the union of the two tiles' key ranges of the query block
// starting at row r0 (0 when neither tile has a key).
int64_t union_blocks(int64_t r0, int64_t q_len, int64_t kv_len, int64_t pre, int64_t next) {
    const int64_t r1 = std::min(q_len, r0 + 256) - 1;
    if (r1 < r0 || kv_len <= 0) return 0;
    const int64_t lo = std::max<int64_t>(0, r0 - pre);
    const int64_t hi = std::min<int64_t>(kv_len - 1, r1 + next);
    if (hi < lo) return 0;
    return hi / kKvBlock - lo / kKvBlock + 1;
}

// Number of 128-key blocks that 128-row query tile [r0, r0+128) touches,
// for the LPT ordering of the varlen work table.
int64_t kv_blocks_for_tile(int64_t r0, int64_t q_len, int64_t kv_len, int64_t pre, int64_t next) {
    const int64_t r1 = std::min(q_len, r0 + 128) - 1;
    if (r1 < r0 || kv_len <= 0) return 0;
    const int64_t lo = std::max<int64_t>(0, r0 - pre);
    const int64_t hi = std::min<int64_t>(kv_len - 1, r1 + next);
    if (hi < lo) return 0;
    return hi / kKvBlock - lo / kKvBlock + 1;
}

}  // namespace

namespace fa {

int64_t varlen_table_len(const int64_t* cu_q, int64_t B) {
    int64_t n = 0;
    for (int64_t b = 0; b < B; ++b) n += (cu_q[b + 1] - cu_q[b] + kQBlock - 1) / kQBlock;
    return n;
}

void build_varlen_table(const int64_t* cu_q, const int64_t* cu_kv, int64_t B, int64_t pre, int64_t next,
                        VarlenEntry* scratch, int4* out) {
    int64_t count = 0;
    for (int64_t b = 0; b < B; ++b) {
        const int64_t ql = cu_q[b + 1] - cu_q[b];
        const int64_t kl = cu_kv[b + 1] - cu_kv[b];
        for (int64_t qb = 0; qb * kQBlock < ql; ++qb) {
            const int64_t cost = kv_blocks_for_tile(qb * kQBlock, ql, kl, pre, next) +
                                 kv_blocks_for_tile(qb * kQBlock + 128, ql, kl, pre, next);
            scratch[count] = {cost, count, make_int4((int)b, (int)qb, (int)ql, (int)kl)};
            ++count;
        }
    }
    // a total order (cost, then position), so an in-place sort gives one result
    std::sort(scratch, scratch + count, [](const VarlenEntry& a, const VarlenEntry& c) {
        return a.cost != c.cost ? a.cost > c.cost : a.order < c.order;
    });
    for (int64_t e = 0; e < count; ++e) out[e] = scratch[e].e;
}

bool tma_dim_ok(int64_t stride, int64_t size) {
    if (size == 1) return true;
    const int64_t bytes = stride * 2;
    return stride > 0 && bytes % 16 == 0 && bytes < (int64_t(1) << 40);
}

}  // namespace fa

extern "C" fa_status fa_fwd_get_workspace_size_v5(
    const fa_tensor* query, const fa_tensor* queryRope, const fa_tensor* key, const fa_tensor* keyRope,
    const fa_tensor* value,
    const fa_tensor* realShift, const fa_tensor* attenMask, const fa_tensor* sink,
    const int64_t* actualSeqQLen, int64_t nSeqQ,
    const int64_t* actualSeqKvLen, int64_t nSeqKv,
    const int64_t* qStartIdx, int64_t nQStartIdx,
    const int64_t* kvStartIdx, int64_t nKvStartIdx,
    double scaleValue, double keepProb, int64_t preTokens, int64_t nextTokens,
    int64_t headNum, const char* inputLayout, int64_t innerPrecise,
    int64_t maskMode, int64_t pseType, const char* softmaxOutLayout,
    const fa_tensor* softmaxMax, const fa_tensor* softmaxSum, const fa_tensor* attentionOut,
    uint64_t* workspaceSize, fa_executor** executor) {
    if (executor) *executor = nullptr;
    // ---- 161001: required arguments -------------------------------------
    if (!query || !key || !value || !softmaxMax || !softmaxSum || !attentionOut || !workspaceSize ||
        !executor)
        return FA_ERR_PARAM_NULLPTR;
    if (!query->data || !key->data || !value->data || !softmaxMax->data || !softmaxSum->data ||
        !attentionOut->data)
        return FA_ERR_PARAM_NULLPTR;
    if ((realShift && !realShift->data) || (attenMask && !attenMask->data) || (sink && !sink->data))
        return FA_ERR_PARAM_NULLPTR;
    if ((queryRope && !queryRope->data) || (keyRope && !keyRope->data)) return FA_ERR_PARAM_NULLPTR;
    const bool rope = queryRope != nullptr;

    // ---- 161002: dtypes and format strings ------------------------------
    Layout L;
    if (!parse_layout(inputLayout, &L)) return FA_ERR_PARAM_INVALID;
    const char* sol = softmaxOutLayout ? softmaxOutLayout : "";
    const bool stats_same_as_input = std::strcmp(sol, "same_as_input") == 0;
    if (!stats_same_as_input && sol[0] != '\0') return FA_ERR_PARAM_INVALID;
    const int32_t dt = query->dtype;
    if (!is_float_dtype(dt) || key->dtype != dt || value->dtype != dt || attentionOut->dtype != dt)
        return FA_ERR_PARAM_INVALID;
    if (softmaxMax->dtype != FA_F32 || softmaxSum->dtype != FA_F32) return FA_ERR_PARAM_INVALID;
    if (attenMask && attenMask->dtype != FA_U8 && attenMask->dtype != FA_BOOL) return FA_ERR_PARAM_INVALID;
    if (sink && sink->dtype != FA_F32) return FA_ERR_PARAM_INVALID;
    // queryRope / keyRope: BFLOAT16 only, the dtype of query/key/value
    // (aclnnFlashAttentionVarLenScoreV5, parameter list)
    if ((queryRope && (queryRope->dtype != FA_BF16 || dt != FA_BF16)) ||
        (keyRope && (keyRope->dtype != FA_BF16 || dt != FA_BF16)))
        return FA_ERR_PARAM_INVALID;
    if (realShift) {
        if (pseType == FA_PSE_DENSE && realShift->dtype != dt) return FA_ERR_PARAM_INVALID;
        if (pseType == FA_PSE_ALIBI && realShift->dtype != FA_F32) return FA_ERR_PARAM_INVALID;
    }

    // ---- 561103: attributes ----------------------------------------------
    if (keepProb != 1.0) return FA_ERR_INNER_NULLPTR;
    if (!std::isfinite(scaleValue) || scaleValue == 0.0) return FA_ERR_INNER_NULLPTR;
    if (innerPrecise < 0 || innerPrecise > 2) return FA_ERR_INNER_NULLPTR;
    if (maskMode != FA_MASK_TENSOR && maskMode != FA_MASK_BAND) return FA_ERR_INNER_NULLPTR;
    if (headNum < 1 || headNum > kMaxN) return FA_ERR_INNER_NULLPTR;
    if (realShift == nullptr) {
        if (pseType != FA_PSE_NONE && pseType != FA_PSE_DENSE) return FA_ERR_INNER_NULLPTR;
    } else if (pseType != FA_PSE_DENSE && pseType != FA_PSE_ALIBI) {
        return FA_ERR_INNER_NULLPTR;
    }

    // ---- 561103: shapes ---------------------------------------------------
    View qv, kv, vv, ov;
    fa_status s;
    if ((s = make_view(query, L, headNum, 0, &qv)) != FA_SUCCESS) return s;
    if ((s = make_view(key, L, 0, qv.D, &kv)) != FA_SUCCESS) return s;
    if ((s = make_view(value, L, kv.N, 0, &vv)) != FA_SUCCESS) return s;
    if (qv.N != headNum) return FA_ERR_INNER_NULLPTR;
    if (kv.D != qv.D || vv.N != kv.N || kv.N < 1 || qv.N % kv.N != 0) return FA_ERR_INNER_NULLPTR;
    if (vv.D > qv.D || qv.D > kMaxD) return FA_ERR_INNER_NULLPTR;
    if (L != L_TND && (kv.B != qv.B || vv.B != qv.B || vv.S != kv.S)) return FA_ERR_INNER_NULLPTR;
    if (L == L_TND && vv.S != kv.S) return FA_ERR_INNER_NULLPTR;
    if ((s = make_view(attentionOut, L, headNum, 0, &ov)) != FA_SUCCESS) return s;
    if (ov.N != qv.N || ov.S != qv.S || ov.D != vv.D || (L != L_TND && ov.B != qv.B))
        return FA_ERR_INNER_NULLPTR;
    if (qv.S > kMaxS || kv.S > kMaxS) return FA_ERR_INNER_NULLPTR;
    // rope: both or neither; no realShift with it (same page: realShiftOptional
    // is incompatible with queryRope/keyRope); the query's / key's layout,
    // sizes and head counts with a head dim Dr of their own; D + Dr <= 256.
    View qrv, krv;
    if (rope || keyRope) {
        if (!queryRope || !keyRope || realShift) return FA_ERR_INNER_NULLPTR;
        if ((s = make_view(queryRope, L, headNum, 0, &qrv)) != FA_SUCCESS) return s;
        if ((s = make_view(keyRope, L, kv.N, 0, &krv)) != FA_SUCCESS) return s;
        if (qrv.N != qv.N || qrv.S != qv.S || qrv.B != qv.B || krv.N != kv.N || krv.S != kv.S || krv.B != kv.B ||
            krv.D != qrv.D || qv.D + qrv.D > kMaxD)
            return FA_ERR_INNER_NULLPTR;
    }

    auto* ex = new (std::nothrow) fa_executor();
    if (!ex) return FA_ERR_INNER_NULLPTR;
    fa::FaParams& p = ex->p;
    std::memset(&p, 0, sizeof(p));
    auto fail = [&](fa_status st) { delete ex; return st; };

    int64_t B, max_q, max_kv;
    if (L == L_TND) {
        if (!actualSeqQLen || !actualSeqKvLen) return fail(FA_ERR_PARAM_NULLPTR);
        if (nSeqQ < 1 || nSeqQ > kMaxB || nSeqKv != nSeqQ) return fail(FA_ERR_INNER_NULLPTR);
        B = nSeqQ;
        ex->cu.assign(2 * (B + 1), 0);
        max_q = max_kv = 0;
        for (int64_t b = 0; b < B; ++b) {
            const int64_t cq = actualSeqQLen[b], ck = actualSeqKvLen[b];
            if (cq < ex->cu[b] || ck < ex->cu[B + 1 + b]) return fail(FA_ERR_INNER_NULLPTR);
            ex->cu[b + 1] = cq;
            ex->cu[B + 2 + b] = ck;
            max_q = std::max(max_q, cq - ex->cu[b]);
            max_kv = std::max(max_kv, ck - ex->cu[B + 1 + b]);
        }
        if (ex->cu[B] != qv.S || ex->cu[2 * B + 1] != kv.S) return fail(FA_ERR_INNER_NULLPTR);
    } else {
        if (actualSeqQLen || actualSeqKvLen) return fail(FA_ERR_INNER_NULLPTR);
        B = qv.B;
        if (B > kMaxB) return fail(FA_ERR_INNER_NULLPTR);
        max_q = qv.S;
        max_kv = kv.S;
    }

    // statistics: [B, N, Sq, 8]; TND: [N, T, 8] ("") or [T, N, 8] ("same_as_input")
    for (const fa_tensor* st : {softmaxMax, softmaxSum}) {
        bool ok;
        if (L != L_TND) ok = same_shape(st, {B, qv.N, qv.S, 8});
        else if (stats_same_as_input) ok = same_shape(st, {qv.S, qv.N, 8});
        else ok = same_shape(st, {qv.N, qv.S, 8});
        if (!ok || st->strides[st->ndim - 1] != 1) return fail(FA_ERR_INNER_NULLPTR);
        for (int i = 0; i < st->ndim; ++i) if (st->strides[i] < 0) return fail(FA_ERR_INNER_NULLPTR);
    }
    if (softmaxMax->strides[0] != softmaxSum->strides[0] || softmaxMax->strides[1] != softmaxSum->strides[1] ||
        (L != L_TND && softmaxMax->strides[2] != softmaxSum->strides[2]))
        return fail(FA_ERR_INNER_NULLPTR);

    // band: -pre <= j - i <= next; the two bounds must intersect
    const int64_t lim = max_q + max_kv + 1;
    if (clamp64(preTokens, -lim, lim) + clamp64(nextTokens, -lim, lim) < 0) return fail(FA_ERR_INNER_NULLPTR);
    // Global positions (qStartIdx / kvStartIdx, one value or one per sequence):
    // the band and ALiBi see qStart + i and kvStart + j, i.e. j - i shifted by
    // delta = kvStart - qStart, the same for every sequence of the call.
    int64_t delta = 0;
    {
        const int64_t nseq = (L == L_TND) ? B : 1;
        auto start_at = [&](const int64_t* a, int64_t n, int64_t b, int64_t* v) {
            if (!a || n == 0) { *v = 0; return true; }
            if (n == 1) { *v = a[0]; return true; }
            if (n != nseq) return false;
            *v = a[b];
            return true;
        };
        for (int64_t b = 0; b < nseq; ++b) {
            int64_t qs, ks;
            if (!start_at(qStartIdx, nQStartIdx, b, &qs) || !start_at(kvStartIdx, nKvStartIdx, b, &ks) || qs < 0 ||
                ks < 0 || qs > kMaxS * 64 || ks > kMaxS * 64)
                return fail(FA_ERR_INNER_NULLPTR);
            if (b == 0) delta = ks - qs;
            else if (ks - qs != delta) return fail(FA_ERR_INNER_NULLPTR);
        }
    }
    // -pre <= (j + delta) - i <= next  <=>  -(pre + delta) <= j - i <= next - delta
    auto shifted = [&](int64_t bound, int64_t d) {
        return bound >= lim ? lim : clamp64(clamp64(bound, -lim, lim) + d, -lim, lim);
    };
    const int64_t pre_c = shifted(preTokens, delta);
    const int64_t next_c = shifted(nextTokens, -delta);
    p.alibi_delta = (int32_t)delta;

    // sink
    if (sink && (!same_shape(sink, {qv.N}) || sink->strides[0] != 1)) return fail(FA_ERR_INNER_NULLPTR);

    // position bias
    if (realShift && pseType == FA_PSE_DENSE && L == L_TND) {
        // [pseTotalLen]: sequence b's [N, Sq_b, Skv_b] block after those of
        // sequences 0 .. b-1 (aclnnFlashAttentionVarLenScoreV5, realShiftOptional)
        int64_t total = 0;
        std::vector<int64_t> offs(B);
        for (int64_t b = 0; b < B; ++b) {
            offs[b] = total;
            total += qv.N * (ex->cu[b + 1] - ex->cu[b]) * (ex->cu[B + 2 + b] - ex->cu[B + 1 + b]);
        }
        if (realShift->ndim != 1 || realShift->shape[0] != total || (total > 1 && realShift->strides[0] != 1))
            return fail(FA_ERR_INNER_NULLPTR);
        ex->cu.insert(ex->cu.end(), offs.begin(), offs.end());  // copied to the workspace with the offsets
        p.pse_flat = 1;
    } else if (realShift && pseType == FA_PSE_DENSE) {
        if (realShift->ndim != 4) return fail(FA_ERR_INNER_NULLPTR);
        const int64_t* sh = realShift->shape;
        // [B|1, N|1, Sq, Skv], or the compressed [B|1, N|1, 1024, Skv] (the last
        // 1024 rows of a lower-triangular bias; Sq > 1024, Sq = Skv, keys at or
        // left of the diagonal only: same page, realShiftOptional notes)
        const bool rows1024 = sh[2] == 1024 && qv.S > 1024 && qv.S == kv.S && next_c <= 0;
        if (!(sh[0] == 1 || sh[0] == B) || !(sh[1] == 1 || sh[1] == qv.N) || (sh[2] != qv.S && !rows1024) ||
            sh[3] != kv.S || realShift->strides[3] != 1)
            return fail(FA_ERR_INNER_NULLPTR);
        p.pse_b = sh[0] == 1 ? 0 : realShift->strides[0];
        p.pse_n = sh[1] == 1 ? 0 : realShift->strides[1];
        p.pse_i = realShift->strides[2];
        p.pse_rows1024 = rows1024 ? 1 : 0;
    } else if (realShift && pseType == FA_PSE_ALIBI) {
        if (same_shape(realShift, {qv.N}) && realShift->strides[0] == 1) {
            p.pse_b = 0; p.pse_n = 1;
        } else if (same_shape(realShift, {B, qv.N}) && realShift->strides[1] == 1) {
            p.pse_b = realShift->strides[0]; p.pse_n = 1;
        } else {
            return fail(FA_ERR_INNER_NULLPTR);
        }
    }

    // mask: [B,N,Sq,Skv], [B,1,Sq,Skv], [1,1,Sq,Skv], [Sq,Skv]; TND only [Sq,Skv]
    if (attenMask) {
        const fa_tensor* m = attenMask;
        if (m->strides[m->ndim - 1] != 1) return fail(FA_ERR_INNER_NULLPTR);
        if (m->ndim == 2) {
            const bool ok = (L == L_TND) ? (m->shape[0] >= max_q && m->shape[1] >= max_kv)
                                         : (m->shape[0] == qv.S && m->shape[1] == kv.S);
            if (!ok) return fail(FA_ERR_INNER_NULLPTR);
            p.mask_b = 0; p.mask_n = 0; p.mask_i = m->strides[0];
        } else if (m->ndim == 4 && L != L_TND) {
            const int64_t* sh = m->shape;
            const bool ok = (sh[0] == B || sh[0] == 1) && (sh[1] == qv.N || sh[1] == 1) &&
                            sh[2] == qv.S && sh[3] == kv.S;
            if (!ok) return fail(FA_ERR_INNER_NULLPTR);
            p.mask_b = sh[0] == 1 ? 0 : m->strides[0];
            p.mask_n = sh[1] == 1 ? 0 : m->strides[1];
            p.mask_i = m->strides[2];
        } else {
            return fail(FA_ERR_INNER_NULLPTR);
        }
    }

    // ---- parameter block ---------------------------------------------------
    p.q = query->data; p.k = key->data; p.v = value->data; p.o = attentionOut->data;
    p.smax = static_cast<float*>(softmaxMax->data);
    p.ssum = static_cast<float*>(softmaxSum->data);
    p.pse = realShift ? realShift->data : nullptr;
    p.mask = attenMask ? static_cast<const uint8_t*>(attenMask->data) : nullptr;
    p.sink = sink ? static_cast<const float*>(sink->data) : nullptr;
    p.q_b = qv.sb; p.q_n = qv.sn; p.q_s = qv.ss;
    p.k_b = kv.sb; p.k_n = kv.sn; p.k_s = kv.ss;
    p.v_b = vv.sb; p.v_n = vv.sn; p.v_s = vv.ss;
    p.o_b = ov.sb; p.o_n = ov.sn; p.o_s = ov.ss;
    if (rope) {
        p.qr = queryRope->data; p.kr = keyRope->data;
        p.qr_b = qrv.sb; p.qr_n = qrv.sn; p.qr_s = qrv.ss;
        p.kr_b = krv.sb; p.kr_n = krv.sn; p.kr_s = krv.ss;
        p.Dr = (int32_t)qrv.D;
    }
    if (L != L_TND) {
        p.st_b = softmaxMax->strides[0]; p.st_n = softmaxMax->strides[1]; p.st_s = softmaxMax->strides[2];
    } else if (stats_same_as_input) {
        p.st_b = 0; p.st_s = softmaxMax->strides[0]; p.st_n = softmaxMax->strides[1];
    } else {
        p.st_b = 0; p.st_n = softmaxMax->strides[0]; p.st_s = softmaxMax->strides[1];
    }
    p.B = (int32_t)B; p.Nq = (int32_t)qv.N; p.Nkv = (int32_t)kv.N; p.group = (int32_t)(qv.N / kv.N);
    p.D = (int32_t)qv.D; p.Dv = (int32_t)vv.D;
    p.Sq = (int32_t)max_q; p.Skv = (int32_t)max_kv;
    p.pre = (int32_t)pre_c; p.next = (int32_t)next_c;
    p.scale = (float)scaleValue;
    p.scale_log2 = (float)(std::fabs(scaleValue) * 1.4426950408889634);
    p.neg_scale = scaleValue < 0 ? 1 : 0;
    p.pse_type = realShift ? (int32_t)pseType : 0;
    p.mask_on = (attenMask && maskMode == FA_MASK_TENSOR) ? 1 : 0;
    p.has_sink = sink ? 1 : 0;
    p.varlen = L == L_TND ? 1 : 0;
    p.dtype = dt;
    // Failure injection for tests of the bounded waits (see fa_device_error).
    const char* stall = std::getenv("FA_DEBUG_STALL");
    p.debug_stall = (stall && std::atoi(stall) != 0) ? 1 : 0;

    p.Tq = (int32_t)qv.S;
    p.Tkv = (int32_t)kv.S;
    p.mask_cols = attenMask ? (int32_t)attenMask->shape[attenMask->ndim - 1] : 0;
    auto aligned16 = [](const void* ptr) { return (reinterpret_cast<uintptr_t>(ptr) & 15u) == 0; };
    p.o_vec = aligned16(p.o) && p.o_b % 8 == 0 && p.o_n % 8 == 0 && p.o_s % 8 == 0;
    auto aligned32 = [](const void* ptr) { return (reinterpret_cast<uintptr_t>(ptr) & 31u) == 0; };
    p.o_vec32 = aligned32(p.o) && p.o_b % 16 == 0 && p.o_n % 16 == 0 && p.o_s % 16 == 0;
    p.st_vec32 = aligned32(p.smax) && aligned32(p.ssum) && p.st_b % 8 == 0 && p.st_n % 8 == 0 && p.st_s % 8 == 0;
    p.mask_vec = attenMask && aligned16(p.mask) && p.mask_b % 16 == 0 && p.mask_n % 16 == 0 && p.mask_i % 16 == 0;
    // 16-byte bias loads: the kernels also check each row's start
    p.pse_vec = realShift && pseType == FA_PSE_DENSE && aligned16(p.pse) && p.pse_b % 8 == 0 &&
                p.pse_n % 8 == 0 && p.pse_i % 8 == 0;

    // ---- kernel choice -------------------------------------------------------
    // tcgen05 needs fp16/bf16, D <= 256, and TMA-legal operands:
    // 16-byte aligned bases and, for every dimension longer than 1, a positive
    // byte stride that is a multiple of 16 and below 2^40.
    using fa::tma_dim_ok;
    bool tma_ok = aligned16(p.q) && aligned16(p.k) && aligned16(p.v);
    const int64_t qB = L == L_TND ? 1 : B;
    tma_ok = tma_ok && tma_dim_ok(p.q_s, qv.S) && tma_dim_ok(p.q_n, qv.N) && tma_dim_ok(p.q_b, qB);
    tma_ok = tma_ok && tma_dim_ok(p.k_s, kv.S) && tma_dim_ok(p.k_n, kv.N) && tma_dim_ok(p.k_b, qB);
    tma_ok = tma_ok && tma_dim_ok(p.v_s, vv.S) && tma_dim_ok(p.v_n, vv.N) && tma_dim_ok(p.v_b, qB);
    // rope on the tcgen05 path: one 64-column chunk more in Q and K
    if (rope)
        tma_ok = tma_ok && p.Dr == 64 && aligned16(p.qr) && aligned16(p.kr) && tma_dim_ok(p.qr_s, qv.S) &&
                 tma_dim_ok(p.qr_n, qv.N) && tma_dim_ok(p.qr_b, qB) && tma_dim_ok(p.kr_s, kv.S) &&
                 tma_dim_ok(p.kr_n, kv.N) && tma_dim_ok(p.kr_b, qB);
    // head dims: D <= 256 and Dv <= D, multiples of 8 (whole 16-byte pieces of
    // a row), run zero-padded to 64, 128 or 256 columns (rope: D <= 128)
    const bool dims_ok = qv.D <= 256 && qv.D % 8 == 0 && vv.D % 8 == 0 && (!rope || qv.D <= 128);
    const bool sm100 = (dt == FA_F16 || dt == FA_BF16) && dims_ok && tma_ok;
    ex->kind = sm100 ? fa::KERNEL_SM100 : fa::KERNEL_SIMT;

    // ---- workspace: schedule counter, cumulative lengths, varlen work
    // table, partial results of split items ----------------------------------
    uint64_t off = 0;
    if (sm100) off = kScheduleHeader;  // the ticket counter, zeroed before every launch
    if (L == L_TND) {
        ex->off_cu = off;
        off += ex->cu.size() * sizeof(int64_t);
        off = (off + 255) & ~uint64_t(255);
    }
    if (sm100) {
        if (L == L_TND) {
            const int64_t len = fa::varlen_table_len(ex->cu.data(), B);
            std::vector<fa::VarlenEntry> scratch(len);
            ex->table.resize(len);
            fa::build_varlen_table(ex->cu.data(), ex->cu.data() + B + 1, B, pre_c, next_c, scratch.data(),
                                   ex->table.data());
            ex->off_table = off;
            off += ex->table.size() * sizeof(int4);
            p.table_len = (int32_t)ex->table.size();
            p.n_items = p.table_len * p.Nq;
        } else {
            p.n_qb = (int32_t)((max_q + kQBlock - 1) / kQBlock);
            p.items_per_n_block = (int32_t)(B * qv.N);
            // 16 heads of K/V at D <= 128 (2 MB each at 4096 keys) stay in L2;
            // the one-tile kernel for larger D streams them twice per item, 4 heads
            p.head_group = qv.D > 128 ? 4 : 16;
            p.n_items = p.n_qb * p.items_per_n_block;
        }
        // Equal-cost items (every query block touches the same number of key
        // blocks) may have their last wave split into key pieces.
        bool uniform = L != L_TND;
        int64_t item_blocks = 0;
        if (uniform) {
            auto cost = [&](int64_t r0) {
                return kv_blocks_for_tile(r0, max_q, max_kv, pre_c, next_c) +
                       kv_blocks_for_tile(r0 + 128, max_q, max_kv, pre_c, next_c);
            };
            item_blocks = union_blocks(0, max_q, max_kv, pre_c, next_c);
            const int64_t c0 = cost(0);
            for (int64_t qb = 1; uniform && qb < p.n_qb; ++qb)
                uniform = cost(qb * kQBlock) == c0 && union_blocks(qb * kQBlock, max_q, max_kv, pre_c, next_c) == item_blocks;
        }
        // SM count of the current device (an attribute query, no device work);
        // without a device the plan assumes a full B200.  Any grid is correct:
        // the SM count only shapes the schedule.
        int dev = 0, sms = 0;
        if (cudaGetDevice(&dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0) {
            (void)cudaGetLastError();
            sms = kDefaultSms;
        }
        const uint64_t part_bytes = fa::plan_sm100_schedule(p, sms, uniform, (int)item_blocks);
        if (part_bytes) {
            off = (off + 255) & ~uint64_t(255);
            ex->off_part = off;
            off += part_bytes;
        }
    }
    ex->ws_bytes = off;
    *workspaceSize = off;

    char buf[256];
    std::snprintf(buf, sizeof(buf),
                  "kernel=%s dtype=%s D=%d Dv=%d Dr=%d B=%d Nq=%d Nkv=%d Sq=%d Skv=%d varlen=%d items=%d grid=%d "
                  "dynamic=%d split_items=%d pieces=%d ws=%llu",
                  sm100 ? "sm100_tcgen05" : "simt_fp32acc", dt == FA_F32 ? "f32" : dt == FA_F16 ? "f16" : "bf16",
                  p.D, p.Dv, p.Dr, p.B, p.Nq, p.Nkv, p.Sq, p.Skv, p.varlen, p.n_items, p.grid,
                  p.dynamic, p.n_items - p.n_whole, p.n_pieces, (unsigned long long)off);
    ex->desc = buf;
    (void)innerPrecise;
    *executor = ex;
    return FA_SUCCESS;
}

extern "C" fa_status fa_fwd_get_workspace_size(
    const fa_tensor* query, const fa_tensor* key, const fa_tensor* value,
    const fa_tensor* realShift, const fa_tensor* attenMask, const fa_tensor* sink,
    const int64_t* actualSeqQLen, int64_t nSeqQ,
    const int64_t* actualSeqKvLen, int64_t nSeqKv,
    double scaleValue, double keepProb, int64_t preTokens, int64_t nextTokens,
    int64_t headNum, const char* inputLayout, int64_t innerPrecise,
    int64_t maskMode, int64_t pseType, const char* softmaxOutLayout,
    const fa_tensor* softmaxMax, const fa_tensor* softmaxSum, const fa_tensor* attentionOut,
    uint64_t* workspaceSize, fa_executor** executor) {
    return fa_fwd_get_workspace_size_v5(query, nullptr, key, nullptr, value, realShift, attenMask, sink, actualSeqQLen, nSeqQ,
                                        actualSeqKvLen, nSeqKv, nullptr, 0, nullptr, 0, scaleValue, keepProb,
                                        preTokens, nextTokens, headNum, inputLayout, innerPrecise, maskMode, pseType,
                                        softmaxOutLayout, softmaxMax, softmaxSum, attentionOut, workspaceSize,
                                        executor);
}

extern "C" fa_status fa_fwd(void* workspace, uint64_t workspaceSize, fa_executor* executor, void* stream) {
    if (!executor) return FA_ERR_PARAM_NULLPTR;
    fa_executor* ex = executor;
    auto done = [&](fa_status st) { delete ex; return st; };
    if (workspaceSize < ex->ws_bytes) return done(FA_ERR_WORKSPACE);
    if (ex->ws_bytes > 0 && !workspace) return done(FA_ERR_PARAM_NULLPTR);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    char* ws = static_cast<char*>(workspace);
    fa::FaParams p = ex->p;
    if (!ex->cu.empty()) {
        // Pageable source, staged before the call returns (or, under stream
        // capture, carried by the graph), so the executor may be freed right after.
        if (fa::upload_async(ws + ex->off_cu, ex->cu.data(), ex->cu.size() * sizeof(int64_t), st) != cudaSuccess)
            return done(FA_ERR_CUDA);
        p.cu_q = reinterpret_cast<const int64_t*>(ws + ex->off_cu);
        p.cu_kv = p.cu_q + (p.B + 1);
        if (p.pse_flat) p.pse_off = p.cu_q + 2 * (p.B + 1);
    }
    if (!ex->table.empty()) {
        if (fa::upload_async(ws + ex->off_table, ex->table.data(), ex->table.size() * sizeof(int4), st) !=
            cudaSuccess)
            return done(FA_ERR_CUDA);
        p.table = reinterpret_cast<const int4*>(ws + ex->off_table);
    }
    cudaError_t err;
    if (ex->kind == fa::KERNEL_SM100) {
        p.sched_counter = reinterpret_cast<int*>(ws);
        p.part = ex->off_part ? reinterpret_cast<float*>(ws + ex->off_part) : nullptr;
        if (p.grid > 0 && p.dynamic && cudaMemsetAsync(ws, 0, sizeof(int), st) != cudaSuccess) return done(FA_ERR_CUDA);
        fa::TmaSet maps;
        if (fa::make_sm100_tmaps(p, &maps) != cudaSuccess) return done(FA_ERR_CUDA);
        err = fa::launch_sm100(p, maps, p.grid, st);
    } else {
        err = fa::launch_simt(p, st);
    }
    return done(err == cudaSuccess ? FA_SUCCESS : FA_ERR_CUDA);
}

extern "C" fa_status fa_lse_merge(const fa_tensor* const* outs, const fa_tensor* const* softmaxMaxes,
                                  const fa_tensor* const* softmaxSums, int64_t count, const fa_tensor* sink,
                                  int64_t headNum, const char* inputLayout, const char* softmaxOutLayout,
                                  const int64_t* actualSeqQLen, int64_t nSeq, const fa_tensor* attentionOut,
                                  const fa_tensor* softmaxMax, const fa_tensor* softmaxSum, void* stream) {
    if (!outs || !softmaxMaxes || !softmaxSums || !attentionOut || !softmaxMax || !softmaxSum)
        return FA_ERR_PARAM_NULLPTR;
    if (!attentionOut->data || !softmaxMax->data || !softmaxSum->data || (sink && !sink->data))
        return FA_ERR_PARAM_NULLPTR;
    if (count < 1 || count > fa::MergeParams::kMax) return FA_ERR_INNER_NULLPTR;
    for (int64_t k = 0; k < count; ++k)
        if (!outs[k] || !softmaxMaxes[k] || !softmaxSums[k] || !outs[k]->data || !softmaxMaxes[k]->data ||
            !softmaxSums[k]->data)
            return FA_ERR_PARAM_NULLPTR;
    Layout L;
    if (!parse_layout(inputLayout, &L)) return FA_ERR_PARAM_INVALID;
    const char* sol = softmaxOutLayout ? softmaxOutLayout : "";
    const bool same_as_input = std::strcmp(sol, "same_as_input") == 0;
    if (!same_as_input && sol[0] != '\0') return FA_ERR_PARAM_INVALID;
    const int32_t dt = attentionOut->dtype;
    if (!is_float_dtype(dt) || (sink && sink->dtype != FA_F32)) return FA_ERR_PARAM_INVALID;
    if (headNum < 1 || headNum > kMaxN) return FA_ERR_INNER_NULLPTR;
    View ov;
    if (make_view(attentionOut, L, headNum, 0, &ov) != FA_SUCCESS) return FA_ERR_INNER_NULLPTR;
    const int64_t B = L == L_TND ? 1 : ov.B;
    if (L == L_TND && actualSeqQLen && (nSeq < 1 || actualSeqQLen[nSeq - 1] != ov.S)) return FA_ERR_INNER_NULLPTR;
    if (sink && (!same_shape(sink, {headNum}) || sink->strides[0] != 1)) return FA_ERR_INNER_NULLPTR;

    // statistics strides (b, n, s) of a [.., 8] tensor of this layout
    auto stat_strides = [&](const fa_tensor* st, int64_t* sb, int64_t* sn, int64_t* ss) {
        if (st->dtype != FA_F32 || !st->data || st->strides[st->ndim - 1] != 1) return false;
        if (L != L_TND) {
            if (!same_shape(st, {ov.B, headNum, ov.S, 8})) return false;
            *sb = st->strides[0]; *sn = st->strides[1]; *ss = st->strides[2];
        } else if (same_as_input) {
            if (!same_shape(st, {ov.S, headNum, 8})) return false;
            *sb = 0; *ss = st->strides[0]; *sn = st->strides[1];
        } else {
            if (!same_shape(st, {headNum, ov.S, 8})) return false;
            *sb = 0; *sn = st->strides[0]; *ss = st->strides[1];
        }
        return true;
    };
    fa::MergeParams mp;
    std::memset(&mp, 0, sizeof(mp));
    mp.count = (int32_t)count;
    for (int64_t k = 0; k < count; ++k) {
        View v;
        if (outs[k]->dtype != dt || make_view(outs[k], L, headNum, 0, &v) != FA_SUCCESS || v.N != ov.N ||
            v.S != ov.S || v.D != ov.D || (L != L_TND && v.B != ov.B))
            return FA_ERR_INNER_NULLPTR;
        int64_t a, b, c, a2, b2, c2;
        if (!stat_strides(softmaxMaxes[k], &a, &b, &c) || !stat_strides(softmaxSums[k], &a2, &b2, &c2) ||
            a != a2 || b != b2 || c != c2)
            return FA_ERR_INNER_NULLPTR;
        mp.out[k] = outs[k]->data;
        mp.smax[k] = static_cast<const float*>(softmaxMaxes[k]->data);
        mp.ssum[k] = static_cast<const float*>(softmaxSums[k]->data);
        mp.o_b[k] = v.sb; mp.o_n[k] = v.sn; mp.o_s[k] = v.ss;
        mp.st_b[k] = a; mp.st_n[k] = b; mp.st_s[k] = c;
    }
    int64_t a, b, c, a2, b2, c2;
    if (!stat_strides(softmaxMax, &a, &b, &c) || !stat_strides(softmaxSum, &a2, &b2, &c2) || a != a2 || b != b2 ||
        c != c2)
        return FA_ERR_INNER_NULLPTR;
    mp.res_o = attentionOut->data;
    mp.res_max = static_cast<float*>(softmaxMax->data);
    mp.res_sum = static_cast<float*>(softmaxSum->data);
    mp.r_o_b = ov.sb; mp.r_o_n = ov.sn; mp.r_o_s = ov.ss;
    mp.r_st_b = a; mp.r_st_n = b; mp.r_st_s = c;
    mp.sink = sink ? static_cast<const float*>(sink->data) : nullptr;
    mp.B = (int32_t)B; mp.N = (int32_t)headNum; mp.S = (int32_t)ov.S; mp.Dv = (int32_t)ov.D; mp.dtype = dt;
    return fa::launch_lse_merge(mp, static_cast<cudaStream_t>(stream)) == cudaSuccess ? FA_SUCCESS : FA_ERR_CUDA;
}

extern "C" void fa_executor_destroy(fa_executor* executor) { delete executor; }

extern "C" const char* fa_executor_describe(const fa_executor* executor) {
    return executor ? executor->desc.c_str() : "";
}

extern "C" fa_status fa_device_error(uint64_t* detail) {
    cudaError_t err = cudaSuccess;
    const uint64_t word = fa::read_and_clear_device_error(&err);
    if (detail) *detail = word;
    if (err != cudaSuccess) return FA_ERR_CUDA;
    return word ? FA_ERR_DEVICE_TIMEOUT : FA_SUCCESS;
}

extern "C" const char* fa_status_string(fa_status status) {
    switch (status) {
        case FA_SUCCESS: return "FA_SUCCESS";
        case FA_ERR_PARAM_NULLPTR: return "FA_ERR_PARAM_NULLPTR (161001): a required argument is NULL";
        case FA_ERR_PARAM_INVALID: return "FA_ERR_PARAM_INVALID (161002): unsupported dtype or format";
        case FA_ERR_INNER_NULLPTR: return "FA_ERR_INNER_NULLPTR (561103): shape or attribute out of range";
        case FA_ERR_CUDA: return "FA_ERR_CUDA (561200): CUDA call or kernel launch failed";
        case FA_ERR_WORKSPACE: return "FA_ERR_WORKSPACE (561201): workspace too small";
        case FA_ERR_DEVICE_TIMEOUT: return "FA_ERR_DEVICE_TIMEOUT (561202): a kernel wait ran out of time";
        default: return "unknown fa_status";
    }
}
