"""The C ABI on the CPU: the library loads, exports every function that
include/fa_fwd.h declares, and stage 1 validates arguments with the status
codes of the aclnn operator pages (161001 / 161002 / 561103).  Stage 1 does no
device work (it only reads the SM count), so host tensors stand in for device
ones here."""
import ctypes
import os
import re

import pytest
import torch

import attention_forward_20_b200 as fa
from attention_forward_20_b200 import _abi

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "fa_fwd.h")


@pytest.fixture(scope="module", autouse=True)
def built():
    from attention_forward_20_b200 import build
    build.build()
    return _abi.load()


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(fa_[a-z0-9_]+)\s*\(", src)))


def test_header_declares_the_documented_entry_points():
    assert declared_functions() == sorted(_abi.EXPORTS)


def test_library_exports_every_declared_symbol(built):
    for name in declared_functions():
        assert hasattr(built, name), name
    out = os.popen(f"nm -D --defined-only {_abi.LIB_PATH}").read()
    exported = set(re.findall(r" T (fa_\w+)", out))
    assert set(declared_functions()) <= exported
    # nothing else leaks out of the library's own namespace
    assert {s for s in exported if s.startswith("fa_")} == set(declared_functions())


def test_status_strings():
    for code in (fa.FA_SUCCESS, fa.FA_ERR_PARAM_NULLPTR, fa.FA_ERR_PARAM_INVALID, fa.FA_ERR_INNER_NULLPTR,
                 fa.FA_ERR_CUDA, fa.FA_ERR_WORKSPACE, fa.FA_ERR_DEVICE_TIMEOUT):
        assert str(code) in _abi.status_string(code) or code == 0
    assert _abi.status_string(12345) == "unknown fa_status"


def qkv(shape, dtype=torch.float16):
    return [torch.zeros(shape, dtype=dtype) for _ in range(3)]


def plan(q, k, v, **kw):
    kw.setdefault("input_layout", "BNSD")
    kw.setdefault("head_num", q.shape[1] if kw["input_layout"] == "BNSD" else None)
    return fa.plan(q, k, v, **kw)


# ---------------------------------------------------------------------------
# Stage 1 accepts the five workloads and picks the kernel
# ---------------------------------------------------------------------------

def test_plan_tiny_fp32_uses_cuda_core_kernel():
    q, k, v = qkv((1, 2, 128, 64), torch.float32)
    st, ws, text = plan(q, k, v, scale=0.125)
    assert st == 0 and ws == 0 and "kernel=simt_fp32acc" in text


@pytest.mark.parametrize("layout,shape,n,dtype,d", [
    ("BNSD", (2, 24, 256, 128), 24, torch.float16, 128),
    ("BSND", (2, 256, 8, 128), 8, torch.bfloat16, 128),
    ("BSH", (2, 512, 1024), 16, torch.float16, 64),
    ("SBH", (300, 2, 256), 4, torch.bfloat16, 64),
])
def test_plan_half_types_use_tcgen05(layout, shape, n, dtype, d):
    q, k, v = qkv(shape, dtype)
    st, ws, text = fa.plan(q, k, v, input_layout=layout, head_num=n)
    assert st == 0, _abi.status_string(st)
    # the workspace holds the ticket counter of the dynamic schedule
    assert "kernel=sm100_tcgen05" in text and f"D={d}" in text and ws == 256


def test_plan_varlen_workspace_holds_lengths_and_table():
    lens = [400, 1069, 1344, 763, 931, 1380, 1693, 612]
    cum = [sum(lens[:i + 1]) for i in range(len(lens))]
    q, k, v = qkv((8192, 24, 128), torch.bfloat16)
    st, ws, text = fa.plan(q, k, v, input_layout="TND", head_num=24, actual_seq_qlen=cum,
                           actual_seq_kvlen=cum, next_tokens=0)
    assert st == 0
    blocks = sum((x + 255) // 256 for x in lens)
    assert "kernel=sm100_tcgen05" in text and f"items={blocks * 24}" in text
    cu_bytes = (2 * (len(lens) + 1) * 8 + 255) // 256 * 256
    assert ws == 256 + cu_bytes + blocks * 16
    assert "split_items=0" in text  # varlen items differ in cost: never split


def _field(text, name):
    return int(text.split(f"{name}=")[1].split()[0])


def test_plan_splits_a_short_last_wave_of_equal_items():
    # 149 equal items on 148 SMs: the last item is split into key pieces
    # (at most one per 128-key block), each piece's partial rows kept in the
    # workspace for the merge.
    q, k, v = qkv((1, 149, 256, 128), torch.float16)
    kk, vv = qkv((1, 149, 1024, 128), torch.float16)[1:]
    st, ws, text = fa.plan(q, kk, vv, input_layout="BNSD", head_num=149)
    assert st == 0, text
    assert _field(text, "items") == 149 and _field(text, "grid") == 148
    assert _field(text, "split_items") == 1 and _field(text, "pieces") == 8
    assert ws == 256 + 1 * 8 * 256 * (128 + 4) * 4


def test_plan_split_pieces_fill_the_grid():
    # dense 2x24 heads x 16 query blocks = 768 items: 5 full waves + 28 items,
    # split 148 // 28 = 5 ways
    q, k, v = qkv((2, 24, 4096, 128), torch.float16)
    st, ws, text = fa.plan(q, k, v, input_layout="BNSD", head_num=24)
    assert st == 0
    assert _field(text, "split_items") == 28 and _field(text, "pieces") == 5
    assert ws == 256 + 28 * 5 * 256 * 132 * 4


@pytest.mark.parametrize("kw", [dict(next_tokens=0), dict(pre_tokens=300, next_tokens=0)])
def test_plan_does_not_split_unequal_items(kw):
    # causal and banded items differ in cost (the band's first query blocks
    # see fewer keys): the dynamic schedule balances them, nothing is split
    q, k, v = qkv((1, 149, 1024, 128), torch.float16)
    st, ws, text = fa.plan(q, k, v, input_layout="BNSD", head_num=149, **kw)
    assert st == 0
    assert _field(text, "split_items") == 0 and ws == 256


def test_plan_no_split_when_items_fill_whole_waves():
    q, k, v = qkv((1, 148, 512, 128), torch.float16)
    st, ws, text = fa.plan(q, k, v, input_layout="BNSD", head_num=148)
    assert st == 0 and _field(text, "items") == 296 and _field(text, "split_items") == 0


def test_plan_unaligned_stride_falls_to_cuda_core_kernel():
    base = torch.zeros(2, 4, 100, 130, dtype=torch.float16)
    q = base[..., :128]  # row stride 130 elements = 260 bytes: not a TMA stride
    st, _, text = fa.plan(q, q, q, input_layout="BNSD", head_num=4)
    assert st == 0 and "kernel=simt_fp32acc" in text


# ---------------------------------------------------------------------------
# 161001: NULL required arguments
# ---------------------------------------------------------------------------

def raw_stage1(q, k, v, out, smax, ssum, layout=b"BNSD", head_num=2, drop=()):
    lib = _abi.load()
    ts = {name: fa._ft(t) for name, t in dict(q=q, k=k, v=v, out=out, smax=smax, ssum=ssum).items()}
    for name in drop:
        ts[name] = None
    p = lambda t: ctypes.byref(t) if t is not None else None  # noqa: E731
    ws = ctypes.c_uint64(0)
    ex = ctypes.c_void_p(None)
    st = lib.fa_fwd_get_workspace_size(p(ts["q"]), p(ts["k"]), p(ts["v"]), None, None, None, None, 0, None, 0,
                                       0.125, 1.0, _abi.INT64_MAX, _abi.INT64_MAX, head_num, layout, 0, 0, 0, b"",
                                       p(ts["smax"]), p(ts["ssum"]), p(ts["out"]), ctypes.byref(ws),
                                       ctypes.byref(ex))
    if st == 0:
        lib.fa_executor_destroy(ex)
    else:
        assert ex.value is None
    return st


def small():
    q, k, v = qkv((1, 2, 16, 64))
    out = torch.zeros_like(q)
    smax = torch.zeros(1, 2, 16, 8)
    ssum = torch.zeros(1, 2, 16, 8)
    return q, k, v, out, smax, ssum


def test_valid_raw_call_succeeds():
    assert raw_stage1(*small()) == 0


@pytest.mark.parametrize("name", ["q", "k", "v", "out", "smax", "ssum"])
def test_null_required_tensor(name):
    assert raw_stage1(*small(), drop=(name,)) == fa.FA_ERR_PARAM_NULLPTR


def test_null_out_pointers():
    lib = _abi.load()
    q, k, v, out, smax, ssum = [fa._ft(t) for t in small()]
    r = ctypes.byref
    st = lib.fa_fwd_get_workspace_size(r(q), r(k), r(v), None, None, None, None, 0, None, 0, 0.125, 1.0,
                                       _abi.INT64_MAX, _abi.INT64_MAX, 2, b"BNSD", 0, 0, 0, b"", r(smax), r(ssum),
                                       r(out), None, None)
    assert st == fa.FA_ERR_PARAM_NULLPTR


def test_fa_fwd_null_executor_and_small_workspace():
    lib = _abi.load()
    assert lib.fa_fwd(None, 0, None, None) == fa.FA_ERR_PARAM_NULLPTR
    lens = [5, 7]
    q, k, v = qkv((12, 2, 64))
    out = torch.zeros_like(q)
    smax = torch.zeros(2, 12, 8)
    ssum = torch.zeros(2, 12, 8)
    status, ws, ex = fa._stage1(q, k, v, out, smax, ssum, input_layout="TND", head_num=2, scale=0.1,
                                real_shift=None, pse_type=0, atten_mask=None, mask_mode=0, sink=None,
                                actual_seq_qlen=[5, 12], actual_seq_kvlen=[5, 12], pre_tokens=_abi.INT64_MAX,
                                next_tokens=_abi.INT64_MAX, keep_prob=1.0, inner_precise=0, softmax_out_layout="")
    assert status == 0 and ws > 0
    # too small a workspace is refused before any CUDA call, and the executor is consumed
    assert lib.fa_fwd(ctypes.c_void_p(16), ctypes.c_uint64(ws - 1), ex, None) == fa.FA_ERR_WORKSPACE
    del lens


# ---------------------------------------------------------------------------
# 161002: dtypes and format strings
# ---------------------------------------------------------------------------

def test_bad_layout_string():
    assert raw_stage1(*small(), layout=b"NSD") == fa.FA_ERR_PARAM_INVALID


def test_mixed_qkv_dtypes():
    q, k, v, out, smax, ssum = small()
    assert raw_stage1(q, k.to(torch.bfloat16), v, out, smax, ssum) == fa.FA_ERR_PARAM_INVALID


def test_out_dtype_and_stats_dtype():
    q, k, v, out, smax, ssum = small()
    assert raw_stage1(q, k, v, out.float(), smax, ssum) == fa.FA_ERR_PARAM_INVALID
    assert raw_stage1(q, k, v, out, smax.half(), ssum) == fa.FA_ERR_PARAM_INVALID


def test_integer_inputs_rejected():
    q, k, v, out, smax, ssum = small()
    i8 = [t.to(torch.uint8) for t in (q, k, v, out)]
    assert raw_stage1(*i8, smax, ssum) == fa.FA_ERR_PARAM_INVALID


def test_bad_mask_and_sink_dtypes():
    q, k, v = qkv((1, 2, 16, 64))
    st, _, _ = plan(q, k, v, atten_mask=torch.zeros(16, 16, dtype=torch.float16))
    assert st == fa.FA_ERR_PARAM_INVALID
    st, _, _ = plan(q, k, v, sink=torch.zeros(2, dtype=torch.float16))
    assert st == fa.FA_ERR_PARAM_INVALID


def test_bad_softmax_out_layout():
    q, k, v = qkv((1, 2, 16, 64))
    assert plan(q, k, v, softmax_out_layout="NTD")[0] == fa.FA_ERR_PARAM_INVALID
    out = torch.zeros_like(q)
    s = torch.zeros(1, 2, 16, 8)
    status, _, _ = fa._stage1(q, k, v, out, s, s.clone(), input_layout="BNSD", head_num=2, scale=0.1,
                              real_shift=None, pse_type=0, atten_mask=None, mask_mode=0, sink=None,
                              actual_seq_qlen=None, actual_seq_kvlen=None, pre_tokens=_abi.INT64_MAX,
                              next_tokens=_abi.INT64_MAX, keep_prob=1.0, inner_precise=0, softmax_out_layout="NTD")
    assert status == fa.FA_ERR_PARAM_INVALID


# ---------------------------------------------------------------------------
# 561103: shapes and attributes
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("kw", [
    dict(keep_prob=0.9),
    dict(scale=0.0),
    dict(scale=float("inf")),
    dict(inner_precise=3),
    dict(mask_mode=2),
    dict(pre_tokens=3, next_tokens=-4),
    dict(pse_type=2),  # ALiBi without slopes
])
def test_bad_attributes(kw):
    q, k, v = qkv((1, 2, 16, 64))
    st, _, _ = plan(q, k, v, **kw)
    assert st == fa.FA_ERR_INNER_NULLPTR


def test_head_num_range_and_mismatch():
    q, k, v = qkv((1, 2, 16, 64))
    assert plan(q, k, v, head_num=3)[0] == fa.FA_ERR_INNER_NULLPTR
    q, k, v = qkv((1, 257, 4, 64))
    assert plan(q, k, v, head_num=257)[0] == fa.FA_ERR_INNER_NULLPTR


def test_gqa_ratio():
    q = torch.zeros(1, 6, 16, 64, dtype=torch.float16)
    kv = torch.zeros(1, 4, 16, 64, dtype=torch.float16)
    assert plan(q, kv, kv)[0] == fa.FA_ERR_INNER_NULLPTR
    kv = torch.zeros(1, 3, 16, 64, dtype=torch.float16)
    st, _, text = plan(q, kv, kv)
    assert st == 0 and "Nkv=3" in text


def test_head_dim_limits():
    q, k, v = qkv((1, 2, 16, 320))
    assert plan(q, k, v)[0] == fa.FA_ERR_INNER_NULLPTR
    q, k, _ = qkv((1, 2, 16, 64))
    v = torch.zeros(1, 2, 16, 96, dtype=torch.float16)  # value head dim above key's
    assert plan(q, k, v)[0] == fa.FA_ERR_INNER_NULLPTR
    v = torch.zeros(1, 2, 16, 32, dtype=torch.float16)  # below is allowed
    st, _, text = plan(q, k, v)
    assert st == 0 and "sm100_tcgen05" in text and "Dv=32" in text


@pytest.mark.parametrize("d,dv,kernel", [(96, 96, "sm100_tcgen05"), (128, 64, "sm100_tcgen05"),
                                         (32, 32, "sm100_tcgen05"), (80, 48, "sm100_tcgen05"),
                                         (100, 100, "simt"), (64, 36, "simt"), (160, 160, "sm100_tcgen05"),
                                         (256, 256, "sm100_tcgen05"), (192, 128, "sm100_tcgen05"),
                                         (264, 264, "simt")])
def test_plan_head_dims_route(d, dv, kernel):
    # half types with D <= 256 and D, Dv multiples of 8 run zero-padded on the
    # tensor cores; the rest on the CUDA-core kernel (up to 256; 264 is rejected)
    if d > 256:
        q, k, v = qkv((1, 2, 300, d))
        assert plan(q, k, v)[0] == fa.FA_ERR_INNER_NULLPTR
        return
    q, k, _ = qkv((1, 2, 300, d))
    v = torch.zeros(1, 2, 300, dv, dtype=torch.float16)
    st, _, text = plan(q, k, v)
    assert st == 0 and kernel in text


def test_batch_and_seq_mismatch():
    q = torch.zeros(2, 2, 16, 64, dtype=torch.float16)
    k = torch.zeros(1, 2, 16, 64, dtype=torch.float16)
    assert plan(q, k, k)[0] == fa.FA_ERR_INNER_NULLPTR
    k = torch.zeros(2, 2, 16, 64, dtype=torch.float16)
    v = torch.zeros(2, 2, 17, 64, dtype=torch.float16)
    assert plan(q, k, v)[0] == fa.FA_ERR_INNER_NULLPTR


def test_varlen_arguments():
    q, k, v = qkv((12, 2, 64))
    base = dict(input_layout="TND", head_num=2)
    assert plan(q, k, v, **base)[0] == fa.FA_ERR_PARAM_NULLPTR               # TND needs lengths
    assert plan(q, k, v, **base, actual_seq_qlen=[5, 12], actual_seq_kvlen=[12])[0] == fa.FA_ERR_INNER_NULLPTR
    assert plan(q, k, v, **base, actual_seq_qlen=[7, 5, 12], actual_seq_kvlen=[7, 5, 12])[0] == \
        fa.FA_ERR_INNER_NULLPTR                                                # not cumulative
    assert plan(q, k, v, **base, actual_seq_qlen=[5, 11], actual_seq_kvlen=[5, 11])[0] == \
        fa.FA_ERR_INNER_NULLPTR                                                # last != T
    st, _, _ = plan(q, k, v, **base, actual_seq_qlen=[5, 5, 12], actual_seq_kvlen=[0, 6, 12])
    assert st == 0                                                             # empty sequences allowed
    q4, k4, v4 = qkv((1, 2, 16, 64))
    assert plan(q4, k4, v4, actual_seq_qlen=[16], actual_seq_kvlen=[16])[0] == fa.FA_ERR_INNER_NULLPTR


def test_stats_shapes():
    q, k, v = qkv((12, 2, 64))
    base = dict(input_layout="TND", head_num=2, actual_seq_qlen=[12], actual_seq_kvlen=[12])
    st, _, _ = plan(q, k, v, **base, softmax_max=torch.zeros(12, 2, 8), softmax_sum=torch.zeros(12, 2, 8))
    assert st == fa.FA_ERR_INNER_NULLPTR   # "" wants [N, T, 8]
    st, _, _ = plan(q, k, v, **base, softmax_out_layout="same_as_input",
                    softmax_max=torch.zeros(12, 2, 8), softmax_sum=torch.zeros(12, 2, 8))
    assert st == 0


def test_sink_pse_and_mask_shapes():
    q, k, v = qkv((2, 2, 16, 64))
    assert plan(q, k, v, sink=torch.zeros(3))[0] == fa.FA_ERR_INNER_NULLPTR
    assert plan(q, k, v, sink=torch.zeros(2))[0] == 0
    assert plan(q, k, v, real_shift=torch.zeros(2, 2, 16, 15, dtype=torch.float16))[0] == fa.FA_ERR_INNER_NULLPTR
    assert plan(q, k, v, real_shift=torch.zeros(1, 2, 16, 16, dtype=torch.float16))[0] == 0
    assert plan(q, k, v, real_shift=torch.zeros(3), pse_type=2)[0] == fa.FA_ERR_INNER_NULLPTR
    assert plan(q, k, v, real_shift=torch.zeros(2, 2), pse_type=2)[0] == 0
    for shape in [(2, 2, 16, 16), (2, 1, 16, 16), (1, 1, 16, 16), (16, 16)]:
        assert plan(q, k, v, atten_mask=torch.zeros(shape, dtype=torch.uint8))[0] == 0, shape
    assert plan(q, k, v, atten_mask=torch.zeros(1, 2, 16, 16, dtype=torch.uint8))[0] == 0
    for shape in [(16, 15), (3, 1, 16, 16), (2, 3, 16, 16), (16,)]:
        assert plan(q, k, v, atten_mask=torch.zeros(shape, dtype=torch.bool))[0] == fa.FA_ERR_INNER_NULLPTR, shape


# ---------------------------------------------------------------------------
# Dense bias layouts besides [B|1, N|1, Sq, Skv]
# ---------------------------------------------------------------------------

def test_plan_compressed_bias_rows():
    q, k, v = qkv((1, 2, 1100, 64), torch.float16)
    pse = torch.zeros(1, 2, 1024, 1100, dtype=torch.float16)
    st, _, _ = plan(q, k, v, real_shift=pse, pse_type=1, next_tokens=0)
    assert st == 0
    # only for a lower-triangular band (keys at or left of the diagonal)
    st, _, _ = plan(q, k, v, real_shift=pse, pse_type=1)
    assert st == _abi.FA_ERR_INNER_NULLPTR
    # only when Sq > 1024 and Sq = Skv
    q2, k2, v2 = qkv((1, 2, 1000, 64), torch.float16)
    st, _, _ = plan(q2, k2, v2, real_shift=torch.zeros(1, 2, 1024, 1000, dtype=torch.float16), pse_type=1,
                    next_tokens=0)
    assert st == _abi.FA_ERR_INNER_NULLPTR


def test_plan_tnd_flat_bias_length_and_workspace():
    lens = [300, 129, 700]
    cum = [sum(lens[:i + 1]) for i in range(len(lens))]
    q, k, v = qkv((sum(lens), 2, 128), torch.bfloat16)
    total = sum(2 * x * x for x in lens)
    st, ws, _ = plan(q, k, v, input_layout="TND", head_num=2, actual_seq_qlen=cum, actual_seq_kvlen=cum,
                     real_shift=torch.zeros(total, dtype=torch.bfloat16), pse_type=1)
    assert st == 0
    st2, ws0, _ = plan(q, k, v, input_layout="TND", head_num=2, actual_seq_qlen=cum, actual_seq_kvlen=cum)
    # the per-sequence bias offsets travel with the cumulative lengths
    assert ws >= ws0 and ws - ws0 <= 256
    st, _, _ = plan(q, k, v, input_layout="TND", head_num=2, actual_seq_qlen=cum, actual_seq_kvlen=cum,
                    real_shift=torch.zeros(total - 1, dtype=torch.bfloat16), pse_type=1)
    assert st == _abi.FA_ERR_INNER_NULLPTR


# ---------------------------------------------------------------------------
# Global positions and the merge entry point (validation only on the CPU)
# ---------------------------------------------------------------------------

def test_plan_start_indices_shift_must_be_common():
    lens = [300, 200]
    cum = [300, 500]
    q, k, v = qkv((500, 2, 128), torch.bfloat16)
    base = dict(input_layout="TND", head_num=2, actual_seq_qlen=cum, actual_seq_kvlen=cum, next_tokens=0)
    assert plan(q, k, v, q_start_idx=[64, 64], kv_start_idx=[0, 0], **base)[0] == 0
    assert plan(q, k, v, q_start_idx=64, kv_start_idx=[0, 0], **base)[0] == 0
    # different kvStart - qStart per sequence
    assert plan(q, k, v, q_start_idx=[0, 0], kv_start_idx=[0, 5], **base)[0] == _abi.FA_ERR_INNER_NULLPTR
    # one value per sequence or a single value only
    assert plan(q, k, v, q_start_idx=[0, 0, 0], **base)[0] == _abi.FA_ERR_INNER_NULLPTR
    assert plan(q, k, v, kv_start_idx=-1, **base)[0] == _abi.FA_ERR_INNER_NULLPTR


def test_plan_rope_routes_and_validates():
    """queryRope / keyRope (aclnnFlashAttentionVarLenScoreV5 parameter list):
    bf16 only, both together, no realShift, the query's / key's sizes with a
    head dim of their own."""
    cum = [300, 500]
    base = dict(input_layout="TND", head_num=4, actual_seq_qlen=cum, actual_seq_kvlen=cum, next_tokens=0)
    q = torch.zeros(500, 4, 128, dtype=torch.bfloat16)
    k = v = torch.zeros(500, 2, 128, dtype=torch.bfloat16)
    qr = torch.zeros(500, 4, 64, dtype=torch.bfloat16)
    kr = torch.zeros(500, 2, 64, dtype=torch.bfloat16)
    st, _, text = plan(q, k, v, query_rope=qr, key_rope=kr, **base)
    assert st == 0 and "kernel=sm100_tcgen05" in text and "Dr=64" in text
    # another rope head dim: CUDA-core kernel
    st, _, text = plan(q, k, v, query_rope=qr[..., :32], key_rope=kr[..., :32].contiguous(), **base)
    assert st == 0 and "kernel=simt" in text and "Dr=32" in text
    # one without the other, a realShift with it, wrong sizes or head counts
    assert plan(q, k, v, query_rope=qr, **base)[0] == _abi.FA_ERR_INNER_NULLPTR
    assert plan(q, k, v, key_rope=kr, **base)[0] == _abi.FA_ERR_INNER_NULLPTR
    slopes = torch.ones(4)
    assert plan(q, k, v, query_rope=qr, key_rope=kr, real_shift=slopes, pse_type=2,
                **base)[0] == _abi.FA_ERR_INNER_NULLPTR
    assert plan(q, k, v, query_rope=qr, key_rope=kr[..., :32].contiguous(), **base)[0] == _abi.FA_ERR_INNER_NULLPTR
    assert plan(q, k, v, query_rope=qr[:499], key_rope=kr, **base)[0] == _abi.FA_ERR_INNER_NULLPTR
    assert plan(q, k, v, query_rope=kr, key_rope=kr, **base)[0] == _abi.FA_ERR_INNER_NULLPTR
    big = torch.zeros(500, 4, 192, dtype=torch.bfloat16)
    bigk = torch.zeros(500, 2, 192, dtype=torch.bfloat16)
    assert plan(q, k, v, query_rope=big, key_rope=bigk, **base)[0] == _abi.FA_ERR_INNER_NULLPTR  # D + Dr > 256
    # dtypes: rope bf16 and query bf16
    assert plan(q, k, v, query_rope=qr.half(), key_rope=kr.half(), **base)[0] == _abi.FA_ERR_PARAM_INVALID
    qh, kh = q.half(), k.half()
    assert plan(qh, kh, kh, query_rope=qr, key_rope=kr, **base)[0] == _abi.FA_ERR_PARAM_INVALID
    # dense layouts: BSH rope has H = heads * Dr
    qb = torch.zeros(2, 100, 4 * 64, dtype=torch.bfloat16)
    kb = torch.zeros(2, 100, 2 * 64, dtype=torch.bfloat16)
    st, _, text = plan(qb, kb, kb, input_layout="BSH", head_num=4, query_rope=torch.zeros(2, 100, 4 * 64,
                       dtype=torch.bfloat16), key_rope=torch.zeros(2, 100, 2 * 64, dtype=torch.bfloat16))
    assert st == 0 and "Dr=64" in text and "kernel=sm100_tcgen05" in text


def _merge_status(outs, maxes, sums, out, smax, ssum, layout="BNSD", heads=2):
    lib = _abi.load()
    n = len(outs)
    P = ctypes.POINTER(_abi.FaTensor)
    ft = lambda t: _abi.make_tensor(t.data_ptr(), 1 if t.dtype == torch.float16 else 0, t.shape, t.stride())  # noqa: E731
    keep = [ft(t) for t in outs + maxes + sums]
    arr = lambda ts: (P * max(1, len(ts)))(*[ctypes.pointer(t) for t in ts])  # noqa: E731
    o, m, s_ = ft(out), ft(smax), ft(ssum)
    return lib.fa_lse_merge(arr(keep[:n]), arr(keep[n:2 * n]), arr(keep[2 * n:]), n, None, heads, layout.encode(),
                            b"", None, 0, ctypes.byref(o), ctypes.byref(m), ctypes.byref(s_), None)


def test_merge_validation():
    out = torch.zeros(1, 2, 40, 64, dtype=torch.float16)
    st = torch.zeros(1, 2, 40, 8)
    assert _merge_status([], [], [], out, st, st) == _abi.FA_ERR_INNER_NULLPTR  # no part
    bad = torch.zeros(1, 2, 41, 64, dtype=torch.float16)
    assert _merge_status([bad], [st], [st], out, st, st) == _abi.FA_ERR_INNER_NULLPTR  # shape
    assert _merge_status([out], [torch.zeros(1, 2, 40, 4)], [st], out, st, st) == _abi.FA_ERR_INNER_NULLPTR


def test_limits_rejected_one_past():
    # S and T up to 1M, heads up to 256 (aclnnFlashAttentionVarLenScoreV5, 约束说明)
    q = torch.zeros(1, 1, (1 << 20) + 1, 8, dtype=torch.float16)
    assert plan(q, q, q)[0] == fa.FA_ERR_INNER_NULLPTR
    q = torch.zeros(1, 1, 1 << 20, 8, dtype=torch.float16)
    assert plan(q, q, q)[0] == 0
    q = torch.zeros(1, 257, 4, 8, dtype=torch.float16)
    assert plan(q, q, q)[0] == fa.FA_ERR_INNER_NULLPTR
    # B up to 20000 sequences
    t = torch.zeros(20001, 1, 8, dtype=torch.float16)
    cum = list(range(1, 20002))
    assert plan(t, t, t, input_layout="TND", head_num=1, actual_seq_qlen=cum,
                actual_seq_kvlen=cum)[0] == fa.FA_ERR_INNER_NULLPTR
    t = torch.zeros(20000, 1, 8, dtype=torch.float16)
    cum = list(range(1, 20001))
    assert plan(t, t, t, input_layout="TND", head_num=1, actual_seq_qlen=cum, actual_seq_kvlen=cum)[0] == 0


def test_header_is_plain_c_and_stage_one_runs_from_c(built, tmp_path):
    """A C99 program compiles against include/fa_fwd.h (no C++ or torch types
    in the interface), links libfa_fwd.so, plans a dense BNSD call and a bad
    layout, and frees the plan; stage 1 touches no device memory."""
    import shutil
    import subprocess
    if shutil.which("gcc") is None:
        pytest.skip("no C compiler")
    src = tmp_path / "stage1.c"
    src.write_text(r'''
#include <stdio.h>
#include <string.h>
#include "fa_fwd.h"

static fa_tensor bnsd(int32_t dtype, int64_t b, int64_t n, int64_t s, int64_t d, void* data) {
    fa_tensor t;
    memset(&t, 0, sizeof t);
    t.data = data; t.dtype = dtype; t.ndim = 4;
    t.shape[0] = b; t.shape[1] = n; t.shape[2] = s; t.shape[3] = d;
    t.strides[3] = 1; t.strides[2] = d; t.strides[1] = s * d; t.strides[0] = n * s * d;
    return t;
}

int main(void) {
    void* fake = (void*)(uintptr_t)0x100000; /* never dereferenced by stage 1 */
    fa_tensor q = bnsd(FA_F16, 2, 4, 1000, 128, fake), o = q;
    fa_tensor st = bnsd(FA_F32, 2, 4, 1000, 8, fake);
    uint64_t ws = 0;
    fa_executor* ex = NULL;
    fa_status s = fa_fwd_get_workspace_size(&q, &q, &q, NULL, NULL, NULL, NULL, 0, NULL, 0, 0.088, 1.0,
                                            INT64_MAX, 0, 4, "BNSD", 0, 0, 0, "", &st, &st, &o, &ws, &ex);
    if (s != FA_SUCCESS || ex == NULL) return 1;
    printf("%s\n", fa_executor_describe(ex));
    fa_executor_destroy(ex);
    s = fa_fwd_get_workspace_size(&q, &q, &q, NULL, NULL, NULL, NULL, 0, NULL, 0, 0.088, 1.0,
                                  INT64_MAX, 0, 4, "XYZ", 0, 0, 0, "", &st, &st, &o, &ws, &ex);
    if (s != FA_ERR_PARAM_INVALID || ex != NULL) return 2;
    printf("%s\n", fa_status_string(s));
    return 0;
}
''')
    lib = os.path.join(ROOT, "attention_forward_20_b200", "libfa_fwd.so")
    exe = tmp_path / "stage1"
    cc = subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"),
                         str(src), lib, "-o", str(exe), f"-Wl,-rpath,{os.path.dirname(lib)}"],
                        capture_output=True, text=True)
    assert cc.returncode == 0, cc.stderr
    run = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert run.returncode == 0, (run.returncode, run.stdout, run.stderr)
    assert "kernel=sm100_tcgen05" in run.stdout and "FA_ERR_PARAM_INVALID" in run.stdout
