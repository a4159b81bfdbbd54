"""ctypes view of include/fa_fwd.h: the fa_tensor struct, status codes and
the exported functions of libfa_fwd.so.  Argument marshalling only."""
import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libfa_fwd.so")

FA_SUCCESS = 0
FA_ERR_PARAM_NULLPTR = 161001
FA_ERR_PARAM_INVALID = 161002
FA_ERR_INNER_NULLPTR = 561103
FA_ERR_CUDA = 561200
FA_ERR_WORKSPACE = 561201
FA_ERR_DEVICE_TIMEOUT = 561202

FA_F32, FA_F16, FA_BF16, FA_U8, FA_BOOL = 0, 1, 2, 3, 4
FA_PSE_NONE, FA_PSE_DENSE, FA_PSE_ALIBI = 0, 1, 2
FA_MASK_TENSOR, FA_MASK_BAND = 0, 1

INT64_MAX = 2**63 - 1

EXPORTS = ("fa_fwd_get_workspace_size", "fa_fwd_get_workspace_size_v5", "fa_lse_merge", "fa_fwd", "fa_executor_destroy",
           "fa_executor_describe", "fa_device_error", "fa_status_string", "fa_fwd_varlen_static")


class FaTensor(ctypes.Structure):
    _fields_ = [
        ("data", ctypes.c_void_p),
        ("dtype", ctypes.c_int32),
        ("ndim", ctypes.c_int32),
        ("shape", ctypes.c_int64 * 8),
        ("strides", ctypes.c_int64 * 8),
    ]


class FaError(RuntimeError):
    def __init__(self, status, where):
        self.status = status
        super().__init__(f"{where}: {status_string(status)}")


_lib = None


def load():
    """Load libfa_fwd.so from this package (raises if it was never built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(
            f"{LIB_PATH} is missing: build it with `python -m attention_forward_20_b200.build` "
            "(there is no fallback implementation)")
    lib = ctypes.CDLL(LIB_PATH)
    P = ctypes.POINTER
    lib.fa_fwd_get_workspace_size.restype = ctypes.c_int32
    lib.fa_fwd_get_workspace_size.argtypes = [
        P(FaTensor), P(FaTensor), P(FaTensor),                  # query, key, value
        P(FaTensor), P(FaTensor), P(FaTensor),                  # realShift, attenMask, sink
        P(ctypes.c_int64), ctypes.c_int64,                      # actualSeqQLen, nSeqQ
        P(ctypes.c_int64), ctypes.c_int64,                      # actualSeqKvLen, nSeqKv
        ctypes.c_double, ctypes.c_double, ctypes.c_int64, ctypes.c_int64,  # scale, keepProb, pre, next
        ctypes.c_int64, ctypes.c_char_p, ctypes.c_int64,        # headNum, inputLayout, innerPrecise
        ctypes.c_int64, ctypes.c_int64, ctypes.c_char_p,        # maskMode, pseType, softmaxOutLayout
        P(FaTensor), P(FaTensor), P(FaTensor),                  # softmaxMax, softmaxSum, attentionOut
        P(ctypes.c_uint64), P(ctypes.c_void_p),                 # workspaceSize, executor
    ]
    lib.fa_fwd_get_workspace_size_v5.restype = ctypes.c_int32
    lib.fa_fwd_get_workspace_size_v5.argtypes = [
        P(FaTensor), P(FaTensor), P(FaTensor), P(FaTensor),     # query, queryRope, key, keyRope
        P(FaTensor),                                            # value
        P(FaTensor), P(FaTensor), P(FaTensor),                  # realShift, attenMask, sink
        P(ctypes.c_int64), ctypes.c_int64,                      # actualSeqQLen, nSeqQ
        P(ctypes.c_int64), ctypes.c_int64,                      # actualSeqKvLen, nSeqKv
        P(ctypes.c_int64), ctypes.c_int64,                      # qStartIdx, nQStartIdx
        P(ctypes.c_int64), ctypes.c_int64,                      # kvStartIdx, nKvStartIdx
        ctypes.c_double, ctypes.c_double, ctypes.c_int64, ctypes.c_int64,  # scale, keepProb, pre, next
        ctypes.c_int64, ctypes.c_char_p, ctypes.c_int64,        # headNum, inputLayout, innerPrecise
        ctypes.c_int64, ctypes.c_int64, ctypes.c_char_p,        # maskMode, pseType, softmaxOutLayout
        P(FaTensor), P(FaTensor), P(FaTensor),                  # softmaxMax, softmaxSum, attentionOut
        P(ctypes.c_uint64), P(ctypes.c_void_p),                 # workspaceSize, executor
    ]
    lib.fa_lse_merge.restype = ctypes.c_int32
    lib.fa_lse_merge.argtypes = [
        P(P(FaTensor)), P(P(FaTensor)), P(P(FaTensor)), ctypes.c_int64,  # outs, maxes, sums, count
        P(FaTensor), ctypes.c_int64, ctypes.c_char_p, ctypes.c_char_p,   # sink, headNum, inputLayout, statsLayout
        P(ctypes.c_int64), ctypes.c_int64,                               # actualSeqQLen, nSeq
        P(FaTensor), P(FaTensor), P(FaTensor),                           # attentionOut, softmaxMax, softmaxSum
        ctypes.c_void_p,                                                 # stream
    ]
    lib.fa_fwd.restype = ctypes.c_int32
    lib.fa_fwd.argtypes = [ctypes.c_void_p, ctypes.c_uint64, ctypes.c_void_p, ctypes.c_void_p]
    lib.fa_executor_destroy.restype = None
    lib.fa_executor_destroy.argtypes = [ctypes.c_void_p]
    lib.fa_executor_describe.restype = ctypes.c_char_p
    lib.fa_executor_describe.argtypes = [ctypes.c_void_p]
    lib.fa_device_error.restype = ctypes.c_int32
    lib.fa_device_error.argtypes = [P(ctypes.c_uint64)]
    lib.fa_status_string.restype = ctypes.c_char_p
    lib.fa_status_string.argtypes = [ctypes.c_int32]
    _lib = lib
    return lib


def status_string(status):
    return load().fa_status_string(int(status)).decode()


_Dims = ctypes.c_int64 * 8


def make_tensor(data_ptr, dtype_code, shape, strides):
    """fa_tensor from a raw device address, dtype code, shape and element strides."""
    return FaTensor(int(data_ptr), int(dtype_code), len(shape), _Dims(*shape), _Dims(*strides))
