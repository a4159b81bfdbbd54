"""B200 (sm_100a) FlashAttention self-attention forward.

Thin Python binding over the C ABI of include/fa_fwd.h (libfa_fwd.so, loaded
with ctypes).  PyTorch is used only to allocate device memory and to find the
current CUDA stream; every step of the computation runs in the library's CUDA
kernels.  There is no CPU fallback: CPU tensors, or a missing library, raise.

Entry points:
  fa_fwd(...)                  the two-stage operator call (both stages)
  attention_forward(...)       [B,S,N,D] / [B,N,S,D] convenience form
  attention_forward_varlen(...) packed [T,N,D] with cu_seqlens
  plan(...)                    stage 1 only: validation, workspace size, plan text
  device_error()               reads and clears the kernel error word
"""
import ctypes

import torch

from . import _abi
from ._abi import (  # noqa: F401
    FA_SUCCESS, FA_ERR_PARAM_NULLPTR, FA_ERR_PARAM_INVALID, FA_ERR_INNER_NULLPTR,
    FA_ERR_CUDA, FA_ERR_WORKSPACE, FA_ERR_DEVICE_TIMEOUT,
    FA_PSE_NONE, FA_PSE_DENSE, FA_PSE_ALIBI, FA_MASK_TENSOR, FA_MASK_BAND,
    INT64_MAX, FaError,
)

_DTYPE_CODES = {
    torch.float32: _abi.FA_F32,
    torch.float16: _abi.FA_F16,
    torch.bfloat16: _abi.FA_BF16,
    torch.uint8: _abi.FA_U8,
    torch.bool: _abi.FA_BOOL,
}


def _ft(t):
    if t is None:
        return None
    if t.dtype not in _DTYPE_CODES:
        raise TypeError(f"unsupported dtype {t.dtype}")
    return _abi.make_tensor(t.data_ptr(), _DTYPE_CODES[t.dtype], t.shape, t.stride())


def _ptr(ft):
    return ctypes.byref(ft) if ft is not None else None


def _i64_array(values):
    if values is None:
        return None, 0
    vals = [int(x) for x in (values.tolist() if torch.is_tensor(values) else values)]
    arr = (ctypes.c_int64 * max(1, len(vals)))(*vals)
    return arr, len(vals)


def _head_dims(query, key, value, layout, head_num):
    """(D, Dv, Nkv) from the tensors' shapes in `layout`."""
    if layout in ("BSH", "SBH"):
        d = query.shape[2] // head_num
        n_kv = key.shape[2] // d
        return d, value.shape[2] // n_kv, n_kv
    n_axis = {"BNSD": 1, "BSND": 2, "TND": 1}[layout]
    return query.shape[-1], value.shape[-1], key.shape[n_axis]


def _out_shapes(query, layout, head_num, dv, softmax_out_layout):
    qs = list(query.shape)
    if layout in ("BSH", "SBH"):
        out = qs[:2] + [head_num * dv]
    else:
        out = qs[:-1] + [dv]
    if layout == "BNSD":
        stats = [qs[0], head_num, qs[2], 8]
    elif layout == "BSND":
        stats = [qs[0], head_num, qs[1], 8]
    elif layout == "BSH":
        stats = [qs[0], head_num, qs[1], 8]
    elif layout == "SBH":
        stats = [qs[1], head_num, qs[0], 8]
    else:
        stats = [qs[0], head_num, 8] if softmax_out_layout == "same_as_input" else [head_num, qs[0], 8]
    return out, stats


def _stage1(query, key, value, out, smax, ssum, *, input_layout, head_num, scale, real_shift,
            pse_type, atten_mask, mask_mode, sink, actual_seq_qlen, actual_seq_kvlen,
            pre_tokens, next_tokens, keep_prob, inner_precise, softmax_out_layout,
            q_start_idx=None, kv_start_idx=None, query_rope=None, key_rope=None):
    lib = _abi.load()
    tq, tk, tv = _ft(query), _ft(key), _ft(value)
    tqr, tkr = _ft(query_rope), _ft(key_rope)
    tpse, tmask, tsink = _ft(real_shift), _ft(atten_mask), _ft(sink)
    to, tmax, tsum = _ft(out), _ft(smax), _ft(ssum)
    aq, nq = _i64_array(actual_seq_qlen)
    akv, nkv = _i64_array(actual_seq_kvlen)
    qst, nqst = _i64_array(_as_list(q_start_idx))
    kvst, nkvst = _i64_array(_as_list(kv_start_idx))
    ws = ctypes.c_uint64(0)
    ex = ctypes.c_void_p(None)
    status = lib.fa_fwd_get_workspace_size_v5(
        _ptr(tq), _ptr(tqr), _ptr(tk), _ptr(tkr), _ptr(tv), _ptr(tpse), _ptr(tmask), _ptr(tsink),
        aq, nq, akv, nkv, qst, nqst, kvst, nkvst,
        float(scale), float(keep_prob), int(pre_tokens), int(next_tokens),
        int(head_num), input_layout.encode(), int(inner_precise),
        int(mask_mode), int(pse_type), softmax_out_layout.encode(),
        _ptr(tmax), _ptr(tsum), _ptr(to), ctypes.byref(ws), ctypes.byref(ex))
    return status, ws.value, ex


def _as_list(x):
    """None, one int, or a sequence of ints -> None or a list."""
    if x is None:
        return None
    if isinstance(x, int):
        return [x]
    return [int(v) for v in x]


def _defaults(query, key, value, input_layout, head_num, scale, real_shift, pse_type):
    d, dv, _ = _head_dims(query, key, value, input_layout, head_num)
    if scale is None:
        scale = d ** -0.5
    if pse_type is None:
        pse_type = FA_PSE_NONE if real_shift is None else (FA_PSE_DENSE if real_shift.dim() == 4 else FA_PSE_ALIBI)
    return d, dv, scale, pse_type


def fa_fwd(query, key, value, *, input_layout, head_num, scale=None, real_shift=None, pse_type=None,
           atten_mask=None, mask_mode=FA_MASK_TENSOR, sink=None, actual_seq_qlen=None,
           actual_seq_kvlen=None, pre_tokens=INT64_MAX, next_tokens=INT64_MAX, keep_prob=1.0,
           inner_precise=0, softmax_out_layout="", out=None, softmax_max=None, softmax_sum=None,
           q_start_idx=None, kv_start_idx=None, query_rope=None, key_rope=None):
    """The operator: returns (attention_out, softmax_max, softmax_sum).

    Arguments mirror fa_fwd_get_workspace_size_v5 (include/fa_fwd.h).  Tensors
    must be CUDA tensors on one device; actual_seq_* are host sequences of
    cumulative lengths without a leading zero; q_start_idx / kv_start_idx are
    None, one int or one int per sequence; query_rope / key_rope (bf16, the
    query's / key's layout with their own head dim) add
    scale * query_rope key_rope^T to the scores.  The default scale is
    D ** -0.5 with D the query's head dim, rope or not.  The work is
    enqueued on the current stream of the query's device.
    """
    if not query.is_cuda:
        raise ValueError("fa_fwd runs on CUDA tensors only (no CPU path)")
    _, dv, scale, pse_type = _defaults(query, key, value, input_layout, head_num, scale, real_shift, pse_type)
    out_shape, stats_shape = _out_shapes(query, input_layout, head_num, dv, softmax_out_layout)
    dev = query.device
    if out is None:
        out = torch.empty(out_shape, dtype=query.dtype, device=dev)
    if softmax_max is None:
        softmax_max = torch.empty(stats_shape, dtype=torch.float32, device=dev)
    if softmax_sum is None:
        softmax_sum = torch.empty(stats_shape, dtype=torch.float32, device=dev)
    status, ws_bytes, ex = _stage1(
        query, key, value, out, softmax_max, softmax_sum, input_layout=input_layout,
        head_num=head_num, scale=scale, real_shift=real_shift, pse_type=pse_type,
        atten_mask=atten_mask, mask_mode=mask_mode, sink=sink, actual_seq_qlen=actual_seq_qlen,
        actual_seq_kvlen=actual_seq_kvlen, pre_tokens=pre_tokens, next_tokens=next_tokens,
        keep_prob=keep_prob, inner_precise=inner_precise, softmax_out_layout=softmax_out_layout,
        q_start_idx=q_start_idx, kv_start_idx=kv_start_idx, query_rope=query_rope, key_rope=key_rope)
    if status != FA_SUCCESS:
        raise FaError(status, "fa_fwd_get_workspace_size_v5")
    ws = torch.empty(max(1, ws_bytes), dtype=torch.uint8, device=dev) if ws_bytes else None
    stream = torch.cuda.current_stream(dev).cuda_stream
    status = _abi.load().fa_fwd(ctypes.c_void_p(ws.data_ptr() if ws is not None else None),
                                ctypes.c_uint64(ws_bytes), ex, ctypes.c_void_p(stream))
    if status != FA_SUCCESS:
        raise FaError(status, "fa_fwd")
    return out, softmax_max, softmax_sum


def plan(query, key, value, *, input_layout, head_num, scale=None, real_shift=None, pse_type=None,
         atten_mask=None, mask_mode=FA_MASK_TENSOR, sink=None, actual_seq_qlen=None,
         actual_seq_kvlen=None, pre_tokens=INT64_MAX, next_tokens=INT64_MAX, keep_prob=1.0,
         inner_precise=0, softmax_out_layout="", out=None, softmax_max=None, softmax_sum=None,
         q_start_idx=None, kv_start_idx=None, query_rope=None, key_rope=None):
    """Stage 1 only (no device work): returns (status, workspace_bytes, plan_text)."""
    _, dv, scale, pse_type = _defaults(query, key, value, input_layout, head_num, scale, real_shift, pse_type)
    out_shape, stats_shape = _out_shapes(query, input_layout, head_num, dv, softmax_out_layout)
    dev = query.device
    if out is None:
        out = torch.empty(out_shape, dtype=query.dtype, device=dev)
    if softmax_max is None:
        softmax_max = torch.empty(stats_shape, dtype=torch.float32, device=dev)
    if softmax_sum is None:
        softmax_sum = torch.empty(stats_shape, dtype=torch.float32, device=dev)
    status, ws_bytes, ex = _stage1(
        query, key, value, out, softmax_max, softmax_sum, input_layout=input_layout,
        head_num=head_num, scale=scale, real_shift=real_shift, pse_type=pse_type,
        atten_mask=atten_mask, mask_mode=mask_mode, sink=sink, actual_seq_qlen=actual_seq_qlen,
        actual_seq_kvlen=actual_seq_kvlen, pre_tokens=pre_tokens, next_tokens=next_tokens,
        keep_prob=keep_prob, inner_precise=inner_precise, softmax_out_layout=softmax_out_layout,
        q_start_idx=q_start_idx, kv_start_idx=kv_start_idx, query_rope=query_rope, key_rope=key_rope)
    text = ""
    if status == FA_SUCCESS:
        lib = _abi.load()
        text = lib.fa_executor_describe(ex).decode()
        lib.fa_executor_destroy(ex)
    return status, ws_bytes, text


def lse_merge(outs, softmax_maxes, softmax_sums, *, input_layout, head_num, sink=None, softmax_out_layout="",
              actual_seq_qlen=None, out=None, softmax_max=None, softmax_sum=None):
    """Combine fa_fwd results of the same queries over disjoint key sets
    (computed without a sink) into the result over their union, adding `sink`
    once (fa_lse_merge in include/fa_fwd.h).  Returns (out, softmax_max, softmax_sum)."""
    if not outs or not outs[0].is_cuda:
        raise ValueError("lse_merge runs on CUDA tensors only (no CPU path)")
    dev = outs[0].device
    out = torch.empty_like(outs[0]) if out is None else out
    softmax_max = torch.empty_like(softmax_maxes[0]) if softmax_max is None else softmax_max
    softmax_sum = torch.empty_like(softmax_sums[0]) if softmax_sum is None else softmax_sum
    lib = _abi.load()
    n = len(outs)
    t_outs = [_ft(t) for t in outs]
    t_max = [_ft(t) for t in softmax_maxes]
    t_sum = [_ft(t) for t in softmax_sums]
    P = ctypes.POINTER(_abi.FaTensor)
    arr = lambda ts: (P * n)(*[ctypes.pointer(t) for t in ts])  # noqa: E731
    aq, nq = _i64_array(actual_seq_qlen)
    tsink, to, tmax, tsum = _ft(sink), _ft(out), _ft(softmax_max), _ft(softmax_sum)
    stream = torch.cuda.current_stream(dev).cuda_stream
    status = lib.fa_lse_merge(arr(t_outs), arr(t_max), arr(t_sum), n, _ptr(tsink), int(head_num),
                              input_layout.encode(), softmax_out_layout.encode(), aq, nq,
                              _ptr(to), _ptr(tmax), _ptr(tsum), ctypes.c_void_p(stream))
    if status != FA_SUCCESS:
        raise FaError(status, "fa_lse_merge")
    return out, softmax_max, softmax_sum


def attention_forward(query, key, value, attn_mask=None, scale=None, fused=True, head_first=False, **kwargs):
    """[B,S,N,D] (head_first=False) or [B,N,S,D] (head_first=True) attention.

    attn_mask follows the operator's convention: nonzero / True marks a
    position that does not take part.  Only the fused path exists.
    """
    if not fused:
        raise NotImplementedError("only the fused CUDA path exists")
    layout = "BNSD" if head_first else "BSND"
    n = query.shape[1] if head_first else query.shape[2]
    out, _, _ = fa_fwd(query, key, value, input_layout=layout, head_num=n, scale=scale, atten_mask=attn_mask)
    return out


def attention_forward_varlen(q, k, v, cu_seqlens_q, cu_seqlens_k, max_seqlen_q=None, max_seqlen_k=None,
                             dropout_p=0.0, softmax_scale=None, causal=False, window_size=None, softcap=None,
                             alibi_slopes=None, deterministic=None, return_attn_probs=None, block_table=None):
    """Packed [T,N,D] attention over sequences delimited by int32 cu_seqlens (B+1,) with a leading 0.

    The cumulative lengths are read on the host (a device tensor is copied
    back).  causal sets nextTokens = 0; window_size = (left, right) sets
    preTokens / nextTokens (-1 = unbounded); alibi_slopes (fp32 [N] or [B,N])
    adds -slope * |i - j|.  dropout_p must be 0; softcap and block_table are
    not supported.
    """
    if dropout_p != 0.0:
        raise NotImplementedError("dropout is not supported (keepProb is fixed at 1)")
    if softcap is not None or block_table is not None or return_attn_probs:
        raise NotImplementedError("softcap, block_table and return_attn_probs are not supported")
    cq = [int(x) for x in (cu_seqlens_q.tolist() if torch.is_tensor(cu_seqlens_q) else cu_seqlens_q)]
    ck = [int(x) for x in (cu_seqlens_k.tolist() if torch.is_tensor(cu_seqlens_k) else cu_seqlens_k)]
    if not cq or cq[0] != 0 or not ck or ck[0] != 0:
        raise ValueError("cu_seqlens must start with 0")
    pre, nxt = INT64_MAX, INT64_MAX
    if window_size is not None:
        left, right = window_size
        pre = INT64_MAX if left < 0 else int(left)
        nxt = INT64_MAX if right < 0 else int(right)
    if causal:
        nxt = 0
    out, _, _ = fa_fwd(q, k, v, input_layout="TND", head_num=q.shape[1], scale=softmax_scale,
                       real_shift=alibi_slopes, pse_type=FA_PSE_ALIBI if alibi_slopes is not None else None,
                       actual_seq_qlen=cq[1:], actual_seq_kvlen=ck[1:], pre_tokens=pre, next_tokens=nxt)
    return out


def device_error():
    """Reads and clears the kernel error word: (status, raw word)."""
    word = ctypes.c_uint64(0)
    status = _abi.load().fa_device_error(ctypes.byref(word))
    return status, word.value
