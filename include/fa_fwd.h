/*
 * fa_fwd.h — C ABI of the B200 (sm_100a) FlashAttention self-attention forward.
 *
 * The operation (aclnnFlashAttentionVarLenScoreV5 page, "计算公式": the forward
 * formula and the sink formula; aclnnFlashAttentionScore page, parameter list):
 *
 *   for every batch b and query head n, with i a query row and j a key row of
 *   that sequence:
 *     s_ij    = scaleValue * <q_i, k_j> + pse_ij
 *     keep_ij = (-preTokens <= j - i <= nextTokens) && !attenMask_ij
 *     m_i     = max({s_ij : keep_ij} U {sink_n})
 *     l_i     = sum_keep exp(s_ij - m_i) + exp(sink_n - m_i)
 *     out_i   = sum_keep exp(s_ij - m_i) v_j / l_i
 *   softmaxMax_i = m_i (natural-log units), softmaxSum_i = l_i, each written to
 *   all 8 lanes of the trailing axis.  The sink terms are absent without a
 *   sink.  A row with nothing kept gets out = 0, m = -inf, l = 0 (with a sink:
 *   out = 0, m = sink_n, l = 1).
 *
 * Two-stage call, as on both operator pages ("接口原型" / "函数原型"):
 *   1. fa_fwd_get_workspace_size() validates every argument on the host, plans
 *      the launch and returns the device workspace size and an executor.  It
 *      touches no device memory and enqueues nothing; its only CUDA calls read
 *      the current device's SM count (cudaGetDevice, cudaDeviceGetAttribute),
 *      and without a device it plans for a 148-SM B200.
 *   2. fa_fwd() enqueues the work on `stream` and consumes the executor.
 *
 * Workspace contents (tcgen05 kernel; the CUDA-core kernel needs none): a
 * ticket counter (zeroed by fa_fwd on the stream when the schedule uses it),
 * for TND the cumulative offsets and the list of work items, and, when the
 * last wave of equal-cost work items is split along the keys, the pieces'
 * partial results (fp32 O rows with their max and sum) that a second, small
 * kernel merges.  Nothing in it has to be initialised by the caller.
 *
 * All floating-point accumulation is fp32.  Q·Kᵀ and P·V run on the tcgen05
 * tensor cores for fp16/bf16 inputs whose head dims (D, and Dv <= D) are
 * multiples of 8 up to 256: zero-padded to 64 or 128 columns on a kernel that
 * holds two 128-row query tiles, to 256 on a one-tile kernel.  fp32 inputs and
 * other head dims up to 256 run on an exact-FFMA CUDA-core kernel.
 */
#ifndef FA_FWD_H
#define FA_FWD_H

#include <stdint.h>

#if defined(__GNUC__)
#define FA_API __attribute__((visibility("default")))
#else
#define FA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* ---------------------------------------------------------------------------
 * Status codes.  The first three carry the numbers of the pages' aclnn return
 * codes (aclnnFlashAttentionScore "返回值"; aclnnFlashAttentionVarLenScoreV5
 * return-code table).  The rest are this library's own.
 * ------------------------------------------------------------------------- */
typedef int32_t fa_status;
#define FA_SUCCESS 0
#define FA_ERR_PARAM_NULLPTR 161001   /* a required input, output or out-pointer is NULL      */
#define FA_ERR_PARAM_INVALID 161002   /* a dtype or a layout/format string is not supported   */
#define FA_ERR_INNER_NULLPTR 561103   /* a shape or attribute is out of the supported range   */
#define FA_ERR_CUDA 561200            /* a CUDA runtime call or the kernel launch failed      */
#define FA_ERR_WORKSPACE 561201       /* workspace smaller than fa_fwd_get_workspace_size said */
#define FA_ERR_DEVICE_TIMEOUT 561202  /* a kernel wait ran past its limit (see fa_device_error) */

/* Element types of fa_tensor.dtype. */
#define FA_F32 0
#define FA_F16 1
#define FA_BF16 2
#define FA_U8 3
#define FA_BOOL 4

/* Position-bias kinds for pseType (the pages leave pseType's values undefined;
 * these are this library's). */
#define FA_PSE_NONE 0   /* realShift must be NULL (1 is also accepted with NULL) */
#define FA_PSE_DENSE 1  /* realShift [B or 1, N or 1, Sq, Skv], query dtype, added after scaling */
#define FA_PSE_ALIBI 2  /* realShift fp32 slopes [N] or [B, N]: pse_ij = -slope * |i - j|     */

/* Mask modes for maskMode (the pages' sparseMode numbering is defined in a
 * section they do not include; these are this library's). */
#define FA_MASK_TENSOR 0  /* attenMask, when given, is read element by element, and the band applies */
#define FA_MASK_BAND 1    /* the caller asserts attenMask equals the preTokens/nextTokens band; the
                             kernel does not read attenMask and skips tiles outside the band */

/* A strided tensor view.  `data` is a device pointer, borrowed (the caller owns
 * the memory and keeps it valid until the work on the stream has finished).
 * Strides count elements, not bytes.  The innermost stride must be 1.  Up to 8
 * dimensions. */
typedef struct fa_tensor {
    void* data;
    int32_t dtype;
    int32_t ndim;
    int64_t shape[8];
    int64_t strides[8];
} fa_tensor;

/* Opaque plan made by stage 1 (aclOpExecutor on the pages). */
typedef struct fa_executor fa_executor;

/* Stage 1.  Validates, plans, and reports the workspace size.
 *
 * query / key / value: device tensors, dtype FA_F32, FA_F16 or FA_BF16 (all
 *   three equal), layout `inputLayout`:
 *     "BNSD" [B, N, S, D]   "BSND" [B, S, N, D]   "BSH" [B, S, N*D]
 *     "SBH"  [S, B, N*D]    "TND"  [T, N, D] (T = sequences packed back to back)
 *   key/value may have fewer heads than query (Nq % Nkv == 0; query head n
 *   reads key/value head n / (Nq/Nkv)).  value's head dim may be smaller than
 *   the query/key head dim.
 * realShift: optional bias, see FA_PSE_*; NULL for none.  A dense bias is
 *   [B|1, N|1, Sq, Skv]; or its last 1024 rows [B|1, N|1, 1024, Skv] when
 *   Sq > 1024, Sq == Skv and the band is lower-triangular (nextTokens <= 0):
 *   row i < Sq-1024 then reads stored row 0 along its diagonal,
 *   bias[i][j] = stored[0][j + Sq - 1024 - i]; with "TND" it is the 1-D
 *   [sum_b N*Sq_b*Skv_b], sequence b's [N, Sq_b, Skv_b] block after those of
 *   sequences 0..b-1 (aclnnFlashAttentionVarLenScoreV5, realShiftOptional).
 * attenMask: optional FA_U8/FA_BOOL, nonzero = excluded.  Shapes [B,N,Sq,Skv],
 *   [B,1,Sq,Skv], [1,1,Sq,Skv] or [Sq,Skv]; with "TND" only [Sq,Skv] indexed by
 *   in-sequence positions (Sq, Skv at least the longest sequence).
 * sink: optional fp32 [headNum], one logit per query head, not scaled.
 * actualSeqQLen / actualSeqKvLen: host int64 arrays of nSeqQ == nSeqKv == B
 *   entries, cumulative lengths without a leading 0 ([2,2,0,2,2] is passed as
 *   [2,4,4,6,8]); required with "TND", must be NULL otherwise; the last entry
 *   equals T of query (resp. key/value).  Zero-length sequences are allowed.
 * scaleValue: finite and nonzero.  keepProb: must be 1.0 (no dropout).
 * preTokens / nextTokens: the band -preTokens <= j - i <= nextTokens, inclusive,
 *   counted from the start of each sequence; INT64_MAX for no bound.
 *   preTokens + nextTokens must be >= 0.
 * headNum: N of query, 1..256.  innerPrecise: 0, 1 or 2 (accepted; the
 *   arithmetic is always fp32 and empty rows always get the defined values).
 * maskMode: FA_MASK_TENSOR or FA_MASK_BAND.  pseType: FA_PSE_*.
 * softmaxOutLayout: NULL/"" or "same_as_input".  With "TND" the statistics are
 *   [N, T, 8] for "" and [T, N, 8] for "same_as_input"; other layouts always
 *   use [B, N, Sq, 8].
 * softmaxMax / softmaxSum: fp32 outputs of that shape.  attentionOut: query's
 *   dtype and layout with value's head dim.
 * workspaceSize / executor: out-pointers.  On success *executor owns host
 *   memory until fa_fwd() or fa_executor_destroy() releases it.
 *
 * Returns FA_SUCCESS, FA_ERR_PARAM_NULLPTR, FA_ERR_PARAM_INVALID or
 * FA_ERR_INNER_NULLPTR; on error *executor is set to NULL.  Thread-safe; the
 * only CUDA calls read the current device's SM count (no device work; with no
 * device the plan assumes a 148-SM B200). */
FA_API fa_status fa_fwd_get_workspace_size(
    const fa_tensor* query, const fa_tensor* key, const fa_tensor* value,
    const fa_tensor* realShift, const fa_tensor* attenMask, const fa_tensor* sink,
    const int64_t* actualSeqQLen, int64_t nSeqQ,
    const int64_t* actualSeqKvLen, int64_t nSeqKv,
    double scaleValue, double keepProb, int64_t preTokens, int64_t nextTokens,
    int64_t headNum, const char* inputLayout, int64_t innerPrecise,
    int64_t maskMode, int64_t pseType, const char* softmaxOutLayout,
    const fa_tensor* softmaxMax, const fa_tensor* softmaxSum, const fa_tensor* attentionOut,
    uint64_t* workspaceSize, fa_executor** executor);

/* Stage 1 with the rope term and global positions
 * (aclnnFlashAttentionVarLenScoreV5GetWorkspaceSize's further arguments).
 *
 * queryRope / keyRope (optional, together; the page's forward formula
 * scale*(query key^T + queryRope keyRope^T) + pse): BFLOAT16 tensors (query,
 * key and value must then be BFLOAT16 too; else 161002) in inputLayout with
 * the sizes and head counts of query / key and a head dim Dr of their own
 * (BSH/SBH: H = heads * Dr); D + Dr <= 256.  Not with realShift (the page:
 * incompatible), pseType 0 or 1.  A mismatch returns 561103.  Dr = 64 with
 * D <= 128 runs on the tensor cores; other sizes on the CUDA-core kernel.
 *
 * qStartIdxOptional / kvStartIdxOptional: the start, in the whole sequence, of
 * the query and key/value chunk this call sees.  The band and an ALiBi bias
 * are evaluated at global positions qStart + i and kvStart + j:
 *   keep iff -preTokens <= (kvStart + j) - (qStart + i) <= nextTokens,
 *   ALiBi pse = -slope * |(qStart + i) - (kvStart + j)|;
 * attenMask and a dense realShift stay indexed by in-chunk positions.
 * qStartIdx / kvStartIdx: host int64, NULL (0), one value, or one per
 * sequence (nQStartIdx / nKvStartIdx entries, "TND" only for more than one);
 * kvStart - qStart must be the same for every sequence (else 561103).  All
 * other arguments and the return values are those of
 * fa_fwd_get_workspace_size, which equals this call with queryRope, keyRope,
 * qStartIdx and kvStartIdx all NULL. */
FA_API fa_status fa_fwd_get_workspace_size_v5(
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
    uint64_t* workspaceSize, fa_executor** executor);

/* Stage 2.  Enqueues the forward on `stream` (a cudaStream_t; NULL = the
 * legacy default stream) on the current device and returns without waiting.
 * `workspace` is caller-owned device memory of at least the size stage 1
 * returned (NULL allowed when that size is 0); it must stay untouched until
 * the stream work has finished.  The executor is consumed and freed on every
 * return path, success or error.
 * The call may be captured into a CUDA graph (stream capture on `stream`):
 * it then enqueues only capturable work, and the per-call tables (varlen
 * offsets and work table) travel in the graph, so the graph replays
 * correctly after the executor is gone; the workspace must stay allocated
 * for as long as the graph is replayed.
 * Returns FA_SUCCESS, FA_ERR_PARAM_NULLPTR (executor NULL, or workspace NULL
 * with a nonzero size), FA_ERR_WORKSPACE or FA_ERR_CUDA. */
FA_API fa_status fa_fwd(void* workspace, uint64_t workspaceSize, fa_executor* executor, void* stream);

/* Merge of partial results (the step after a forward split along the keys,
 * e.g. context parallelism: key/value chunks on different GPUs, each run with
 * its kvStartIdx).  outs[k], softmaxMaxes[k], softmaxSums[k] (k < count,
 * 1 <= count <= 16) are the attentionOut / softmaxMax / softmaxSum of the same
 * queries over disjoint key sets, computed without a sink; the result over
 * the union of the key sets, with the optional sink added once, is
 *   M   = max(max_k m_k over rows with l_k > 0, sink_n)
 *   l   = sum_k l_k e^(m_k - M) + e^(sink_n - M)
 *   out = sum_k l_k e^(m_k - M) out_k / l
 * (the online-softmax update of the forward formula, applied to whole partial
 * results; softmaxMax/softmaxSum in natural-log units as the forward writes
 * them).  A row with no key in any part gets out = 0, m = -inf, l = 0 (with a
 * sink: m = sink, l = 1).
 * Tensors are device tensors in `inputLayout` with headNum query heads, all
 * outs[k] and attentionOut of one dtype and shape; statistics fp32 of the
 * forward's statistics shape for that layout and softmaxOutLayout.
 * actualSeqQLen (TND, optional): host cumulative lengths, checked against T.
 * Enqueued on `stream`; no workspace.  Returns FA_SUCCESS,
 * FA_ERR_PARAM_NULLPTR, FA_ERR_PARAM_INVALID, FA_ERR_INNER_NULLPTR or
 * FA_ERR_CUDA.  (No page defines this call; the pages define the statistics
 * it consumes and name the split scenario that needs it.) */
FA_API fa_status fa_lse_merge(const fa_tensor* const* outs, const fa_tensor* const* softmaxMaxes,
                              const fa_tensor* const* softmaxSums, int64_t count, const fa_tensor* sink,
                              int64_t headNum, const char* inputLayout, const char* softmaxOutLayout,
                              const int64_t* actualSeqQLen, int64_t nSeq, const fa_tensor* attentionOut,
                              const fa_tensor* softmaxMax, const fa_tensor* softmaxSum, void* stream);

/* Releases an executor that will not be passed to fa_fwd().  NULL is a no-op. */
FA_API void fa_executor_destroy(fa_executor* executor);

/* Static description of the plan ("kernel=... grid=... items=..."), valid
 * while the executor lives.  For logging and tests. */
FA_API const char* fa_executor_describe(const fa_executor* executor);

/* Reads and clears the current device's kernel error word.  Every wait in the
 * tcgen05 kernel has a time limit (about 2 s); a wait that runs out records an
 * error here and the kernel returns early instead of hanging.  The raw word
 * holds the wait site in its high 32 bits and 1 + the CTA index in its low 32
 * bits.  Synchronises the device.  Returns FA_SUCCESS, FA_ERR_DEVICE_TIMEOUT or
 * FA_ERR_CUDA; when `detail` is not NULL it receives the raw word (0 when
 * clean).  For tests of this path, the environment variable FA_DEBUG_STALL=1
 * (read by fa_fwd_get_workspace_size) makes the kernel wait on a barrier that
 * is never signalled. */
FA_API fa_status fa_device_error(uint64_t* detail);

/* The packed-TND (varlen) forward for callers that cannot allocate device
 * memory.  The operator pages have no counterpart of this call.
 *
 * The ordinary varlen call needs a caller-allocated workspace for its
 * per-call scratch (cumulative sequence offsets and the work-item table).
 * Callers that must not call cudaMalloc -- code running while a stream is
 * captured, or a runtime whose device memory is all handed out up front --
 * cannot provide one.  This call keeps that scratch in a fixed static device
 * array of the library instead and allocates nothing: no cudaMalloc/cudaFree,
 * no workspace, no host heap.  Inputs and outputs are passed as for
 * fa_fwd_get_workspace_size with inputLayout "TND" (no realShift, no
 * attenMask, keepProb 1); the work is enqueued on `stream`.
 *
 * Limit: nSeq <= 2048 sequences (with T <= 1M tokens, as for every call);
 * more sequences return FA_ERR_INNER_NULLPTR before any device work.  The
 * static array (about 130 KB: the offsets and up to 6144 work items) is held
 * on every GPU that loads the library until the process exits.
 *
 * The first call on a device looks up the array's device address (with that
 * device current) and keeps it once the lookup succeeds; make that first call
 * before any stream capture.  Every call overwrites the part of the array it reads, so nothing
 * needs clearing, but calls whose work overlaps on the GPU (other streams,
 * other host threads) race on the shared array.  Under stream capture the
 * offsets and table travel in the graph (copy kernels that carry the bytes in
 * their launch parameters), so each replay writes its own table back into the
 * array first; replays, like calls, must not overlap on the GPU.
 * Each call uploads only what it reads (the ticket counter, its nSeq + 1
 * offsets per side and its work table).  Kernel choice is fa_fwd's:
 * fp16/bf16 with head dims that are multiples of 8 up to 256 run on the
 * tensor cores (the two-tile kernel up to 128, the one-tile kernel above),
 * fp32 and other head dims on the CUDA-core kernel.
 *
 * Returns FA_SUCCESS, FA_ERR_PARAM_NULLPTR, FA_ERR_PARAM_INVALID,
 * FA_ERR_INNER_NULLPTR or FA_ERR_CUDA. */
FA_API fa_status fa_fwd_varlen_static(
    const fa_tensor* query, const fa_tensor* key, const fa_tensor* value, const fa_tensor* sink,
    const int64_t* actualSeqQLen, const int64_t* actualSeqKvLen, int64_t nSeq,
    double scaleValue, int64_t preTokens, int64_t nextTokens, int64_t headNum,
    const char* softmaxOutLayout, const fa_tensor* softmaxMax, const fa_tensor* softmaxSum,
    const fa_tensor* attentionOut, void* stream);

/* Human-readable name of a status code (static string). */
FA_API const char* fa_status_string(fa_status status);

#ifdef __cplusplus
}
#endif

#endif /* FA_FWD_H */
