"""Binding of fa_fwd_varlen_static: the packed-TND forward that allocates
nothing.

For callers that cannot allocate device memory (code running during stream
capture, or under a runtime that hands out all device memory up front): the
per-call scratch lives in a fixed device array of the library, and this
wrapper allocates nothing either -- the caller passes the output tensors.
Argument marshalling only."""
import ctypes

import torch

from . import _abi
from ._abi import INT64_MAX, FaError, FaTensor

_declared = False


def _lib():
    global _declared
    lib = _abi.load()
    if not _declared:
        P = ctypes.POINTER
        lib.fa_fwd_varlen_static.restype = ctypes.c_int32
        lib.fa_fwd_varlen_static.argtypes = [
            P(FaTensor), P(FaTensor), P(FaTensor), P(FaTensor),    # query, key, value, sink
            P(ctypes.c_int64), P(ctypes.c_int64), ctypes.c_int64,  # actualSeqQLen, actualSeqKvLen, nSeq
            ctypes.c_double, ctypes.c_int64, ctypes.c_int64,       # scaleValue, preTokens, nextTokens
            ctypes.c_int64, ctypes.c_char_p,                       # headNum, softmaxOutLayout
            P(FaTensor), P(FaTensor), P(FaTensor),                 # softmaxMax, softmaxSum, attentionOut
            ctypes.c_void_p,                                       # stream
        ]
        _declared = True
    return lib


def fa_fwd_varlen_static(query, key, value, actual_seq_qlen, actual_seq_kvlen, out, softmax_max, softmax_sum, *,
                         head_num, scale=None, sink=None, pre_tokens=INT64_MAX, next_tokens=INT64_MAX,
                         softmax_out_layout="", stream=None):
    """Enqueues the forward into the caller's `out`, `softmax_max`, `softmax_sum`.

    actual_seq_* are host sequences of cumulative lengths without a leading
    zero.  `stream` is a raw cudaStream_t (default: the current torch stream).
    Returns the status (0); raises FaError otherwise.
    """
    from . import _ft
    if scale is None:
        scale = query.shape[-1] ** -0.5
    q_lens = [int(x) for x in actual_seq_qlen]
    kv_lens = [int(x) for x in actual_seq_kvlen]
    aq = (ctypes.c_int64 * max(1, len(q_lens)))(*q_lens)
    akv = (ctypes.c_int64 * max(1, len(kv_lens)))(*kv_lens)
    if stream is None:
        stream = torch.cuda.current_stream(query.device).cuda_stream if query.is_cuda else 0
    ts = [_ft(t) for t in (query, key, value, sink, softmax_max, softmax_sum, out)]
    ref = lambda t: ctypes.byref(t) if t is not None else None  # noqa: E731
    status = _lib().fa_fwd_varlen_static(
        ref(ts[0]), ref(ts[1]), ref(ts[2]), ref(ts[3]), aq, akv, len(q_lens), float(scale), int(pre_tokens),
        int(next_tokens), int(head_num), softmax_out_layout.encode(), ref(ts[4]), ref(ts[5]), ref(ts[6]),
        ctypes.c_void_p(stream))
    if status != 0:
        raise FaError(status, "fa_fwd_varlen_static")
    return status
