"""CUDA path vs the float64 oracle through the C ABI, on the same seeded
inputs.  Small cases compare every output element and span several 128-row
tiles with a ragged tail; the five workloads at full size compare sampled rows
(oracle row by row) in the launch configuration the bench times."""
import numpy as np
import pytest
import torch

import attention_forward_20_b200 as fa
from workloads import normal, causal_mask_u8, alibi_slopes, cumulative, build, Workload
from tests.parity import run_gpu, compare_full, compare_rows, sample_rows, f64

pytestmark = pytest.mark.gpu
INT64_MAX = 2**63 - 1


@pytest.fixture(scope="module", autouse=True)
def lib():
    from attention_forward_20_b200 import build as b
    b.build()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    yield
    status, word = fa.device_error()
    assert status == 0 and word == 0, f"kernel error word {word:#x}"


def W(layout, dtype, shape, heads, seed, **kw):
    """Workload from q/k/v drawn N(0,1) with consecutive seeds."""
    kshape = kw.pop("kshape", shape)
    vshape = kw.pop("vshape", kshape)
    return Workload("case", 0, layout, dtype, heads, normal(shape, dtype, seed), normal(kshape, dtype, seed + 1),
                    normal(vshape, dtype, seed + 2), scale=kw.pop("scale", None) or
                    (shape[-1] if layout not in ("BSH", "SBH") else shape[-1] // heads) ** -0.5, **kw)


def plan_text(w):
    q, k, v = w.q.cuda(), w.k.cuda(), w.v.cuda()
    return fa.plan(q, k, v, input_layout=w.layout, head_num=w.head_num, scale=w.scale,
                   actual_seq_qlen=w.actual_seq_q, actual_seq_kvlen=w.actual_seq_kv)[2]


# ---------------------------------------------------------------------------
# tcgen05 kernel, dense layouts
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("dtype", ["f16", "bf16"])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("s", [128, 300, 513])
def test_dense_bnsd(dtype, d, s):
    w = W("BNSD", dtype, (2, 3, s, d), 3, 100 + s)
    assert "sm100_tcgen05" in plan_text(w)
    compare_full(w)


def test_workload_2_shape_reduced():
    w = build(2, seq_scale=8)   # [2,24,512,128] fp16
    compare_full(w)


@pytest.mark.parametrize("dtype", ["f16", "bf16"])
def test_causal_band_and_sink(dtype):
    w = W("BSND", dtype, (2, 333, 4, 128), 4, 200, next_tokens=0, sink=normal((4,), "f32", 204))
    compare_full(w)


@pytest.mark.parametrize("mask_mode", [0, 1])
def test_causal_mask_tensor_with_sink(mask_mode):
    w = build(3, seq_scale=16)  # [4,512,32,128] bf16, mask [512,512]
    w.mask_mode = mask_mode
    compare_full(w)


def test_mask_tensor_random_with_band():
    s = 300
    w = W("BNSD", "f16", (1, 2, s, 64), 2, 300, pre_tokens=200, next_tokens=40)
    g = torch.Generator().manual_seed(301)
    w.atten_mask = (torch.rand(1, 2, s, s, generator=g) < 0.3).to(torch.uint8)
    compare_full(w)


def test_band_alibi_bsh_d64():
    w = build(5, seq_scale=32)   # [2,512,1024] N=16 D=64, pre=64, next=0, slopes
    compare_full(w)


def test_band_alibi_two_sided():
    w = W("BNSD", "bf16", (1, 4, 400, 128), 4, 400, pre_tokens=150, next_tokens=70,
          pse=alibi_slopes(4), pse_type=2)
    compare_full(w)


@pytest.mark.parametrize("dtype,d,pre,nxt", [("f16", 64, 0, 200), ("bf16", 128, -3, 150), ("f16", 256, 0, 90),
                                             ("bf16", 64, 260, -2), ("f16", 128, 300, 0)])
def test_band_alibi_one_side_of_diagonal(dtype, d, pre, nxt):
    """Bands that keep keys on one side of the diagonal only (preTokens <= 0:
    at or right of it; nextTokens <= 0: at or left of it), so that the ALiBi
    distance |i - j| is linear in j over every kept key of every block, the
    diagonal block included (V5 page: preTokens/nextTokens, pseType 2)."""
    w = W("BNSD", dtype, (2, 3, 330, d), 3, 610 + d, pre_tokens=pre, next_tokens=nxt,
          pse=alibi_slopes(3), pse_type=2)
    compare_full(w)


def _per_batch_slopes(n_batch, n_heads):
    """fp32 [B, N] ALiBi slopes, different along both axes and not symmetric."""
    b = torch.arange(n_batch, dtype=torch.float64)[:, None]
    n = torch.arange(n_heads, dtype=torch.float64)[None, :]
    return (2.0 ** -(n + 1) * (1 + 0.37 * b) + 0.05 * n * b).to(torch.float32)


@pytest.mark.parametrize("case", ["two_tile_bsnd_d64", "two_tile_tnd_d128", "wide_bnsd_d256", "cuda_core_f32"])
def test_alibi_per_batch_slopes(case):
    """Slope-only pse of shape [B, N] (aclnnFlashAttentionVarLenScoreV5,
    realShiftOptional notes): batch row (TND: sequence) b of head n uses
    slope[b, n], on each of the three kernels."""
    if case == "two_tile_bsnd_d64":
        w = W("BSND", "f16", (3, 300, 3, 64), 3, 460, pre_tokens=150, next_tokens=0)
        kernel = "sm100_tcgen05"
    elif case == "two_tile_tnd_d128":
        lens = [23, 400, 170]
        cum = cumulative(lens, False)
        w = W("TND", "bf16", (sum(lens), 2, 128), 2, 470, actual_seq_q=cum, actual_seq_kv=list(cum),
              pre_tokens=200, next_tokens=30)
        kernel = "sm100_tcgen05"
    elif case == "wide_bnsd_d256":
        w = W("BNSD", "bf16", (2, 2, 260, 256), 2, 480, pre_tokens=100, next_tokens=0)
        kernel = "sm100_tcgen05"
    else:
        w = W("BNSD", "f32", (2, 3, 150, 64), 3, 490, pre_tokens=60, next_tokens=5)
        kernel = "simt"
    n_batch = len(w.actual_seq_q) if w.layout == "TND" else w.q.shape[0]
    w.pse, w.pse_type = _per_batch_slopes(n_batch, w.head_num), 2
    assert kernel in plan_text(w)
    compare_full(w)
    # every batch row given row 0's slopes: the same bits as the [N] form
    rows_equal = w.pse[:1].expand(n_batch, -1).contiguous()
    a = run_gpu(w, real_shift=rows_equal.cuda())
    b = run_gpu(w, real_shift=w.pse[0].contiguous().cuda())
    for x, y in zip(a, b):
        assert torch.equal(x, y)


@pytest.mark.parametrize("dtype", ["f16", "bf16"])
def test_dense_pse_tensor(dtype):
    s = 260
    w = W("BNSD", dtype, (2, 2, s, 64), 2, 500, next_tokens=0)
    w.pse = normal((2, 2, s, s), dtype, 505)
    w.pse_type = 1
    compare_full(w)
    w.pse = normal((1, 2, s, s), dtype, 506)  # broadcast over the batch
    compare_full(w)


@pytest.mark.parametrize("dtype", ["f16", "bf16"])
def test_dense_pse_tensor_staged_by_tma(dtype):
    """Head dim 64 with a dense bias whose rows are 16-byte multiples: the
    bias blocks come into shared memory by TMA (two buffers per query tile).
    Ragged query and key tails, a band, bias broadcast over batch or heads,
    and fewer queries than keys."""
    s = 392  # 3 blocks + 8 rows
    w = W("BNSD", dtype, (2, 2, s, 64), 2, 520, pre_tokens=200, next_tokens=30)
    w.pse, w.pse_type = normal((2, 2, s, s), dtype, 525), 1
    compare_full(w)
    w.pse = normal((1, 2, s, s), dtype, 526)   # broadcast over the batch
    compare_full(w)
    w.pse = normal((2, 1, s, s), dtype, 527)   # broadcast over the heads
    w.next_tokens = 0
    compare_full(w)
    w = W("BSND", dtype, (1, 300, 2, 64), 2, 530, kshape=(1, 392, 2, 64), sink=normal((2,), "f32", 534))
    w.pse, w.pse_type = normal((1, 2, 300, 392), dtype, 535), 1
    compare_full(w)


def test_sq_differs_from_skv():
    w = W("BNSD", "f16", (2, 2, 200, 128), 2, 600, kshape=(2, 2, 333, 128))
    compare_full(w)
    w = W("BSND", "bf16", (1, 390, 2, 64), 2, 610, kshape=(1, 150, 2, 64), pre_tokens=100, next_tokens=5)
    compare_full(w)


def test_gqa():
    w = W("BNSD", "bf16", (1, 8, 256, 128), 8, 700, kshape=(1, 2, 256, 128), next_tokens=0)
    compare_full(w)


def test_sbh_layout():
    w = W("SBH", "f16", (270, 2, 4 * 64), 4, 800, next_tokens=0)
    compare_full(w)


def test_negative_scale():
    w = W("BNSD", "f16", (1, 2, 200, 64), 2, 900, scale=-0.1)
    compare_full(w)


def test_empty_rows_band_and_sink():
    # nextTokens = -3: rows 0..2 keep nothing; with a sink they get (0, sink, 1)
    w = W("BNSD", "bf16", (1, 2, 140, 64), 2, 1000, pre_tokens=10, next_tokens=-3)
    compare_full(w)
    w.sink = normal((2,), "f32", 1004)
    compare_full(w)


def test_kv_shorter_than_a_tile_and_single_row():
    compare_full(W("BNSD", "f16", (1, 1, 1, 128), 1, 1100))
    compare_full(W("BNSD", "f16", (1, 1, 300, 128), 1, 1110, kshape=(1, 1, 5, 128)))


def test_permuted_strides_tma():
    base = normal((2, 3, 200, 128), "bf16", 1200)
    w = W("BSND", "bf16", (2, 200, 3, 128), 3, 1210)
    w.q = base.permute(0, 2, 1, 3)          # BSND view of a BNSD buffer
    assert not w.q.is_contiguous()
    compare_full(w)


# ---------------------------------------------------------------------------
# varlen TND
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("stats_layout", ["", "same_as_input"])
def test_varlen_causal(stats_layout):
    lens = [300, 0, 129, 1, 513, 64]
    t = sum(lens)
    cum = cumulative(lens, leading_zero=False)
    w = W("TND", "bf16", (t, 3, 128), 3, 1300, next_tokens=0, actual_seq_q=cum, actual_seq_kv=list(cum),
          softmax_out_layout=stats_layout)
    compare_full(w)


def test_varlen_kv_lengths_differ_with_sink_and_alibi():
    lq, lk = [100, 260, 0, 7], [300, 10, 5, 129]
    wq = normal((sum(lq), 2, 64), "f16", 1400)
    w = W("TND", "f16", (sum(lk), 2, 64), 2, 1401, actual_seq_q=cumulative(lq, False),
          actual_seq_kv=cumulative(lk, False), pre_tokens=50, next_tokens=20,
          sink=normal((2,), "f32", 1405), pse=alibi_slopes(2), pse_type=2)
    w.q = wq
    compare_full(w)


def test_varlen_mask_tensor():
    lens = [200, 77]
    cum = cumulative(lens, False)
    w = W("TND", "bf16", (277, 2, 128), 2, 1500, actual_seq_q=cum, actual_seq_kv=list(cum))
    w.atten_mask = causal_mask_u8(256, 256)
    compare_full(w)


def test_varlen_workload_4_reduced():
    compare_full(build(4, seq_scale=4))


def test_attention_forward_varlen_api():
    lens = [128, 300]
    cu = torch.tensor(cumulative(lens, True), dtype=torch.int32)
    q, k, v = (normal((428, 2, 128), "bf16", 1600 + i).cuda() for i in range(3))
    out = fa.attention_forward_varlen(q, k, v, cu, cu, causal=True)
    w = W("TND", "bf16", (428, 2, 128), 2, 1600, next_tokens=0, actual_seq_q=cumulative(lens, False),
          actual_seq_kv=cumulative(lens, False))
    ref_out, _, _ = run_gpu(w)
    assert torch.equal(out, ref_out)


def test_attention_forward_api_layouts():
    q, k, v = (normal((2, 200, 4, 64), "f16", 1700 + i).cuda() for i in range(3))
    out_bsnd = fa.attention_forward(q, k, v)
    out_bnsd = fa.attention_forward(q.transpose(1, 2).contiguous(), k.transpose(1, 2).contiguous(),
                                    v.transpose(1, 2).contiguous(), head_first=True)
    assert torch.equal(out_bsnd, out_bnsd.transpose(1, 2))


# ---------------------------------------------------------------------------
# CUDA-core kernel (fp32 and head dims the tensor-core kernel does not take)
# ---------------------------------------------------------------------------

def test_workload_1_tiny_fp32():
    w = build(1)
    assert "simt" in plan_text(w)
    compare_full(w)


@pytest.mark.parametrize("layout", ["BNSD", "BSH", "TND"])
def test_fp32_features(layout):
    if layout == "TND":
        lens = [70, 0, 33]
        cum = cumulative(lens, False)
        w = W("TND", "f32", (103, 2, 64), 2, 1800, actual_seq_q=cum, actual_seq_kv=list(cum), next_tokens=0,
              sink=normal((2,), "f32", 1805), pse=alibi_slopes(2), pse_type=2)
    elif layout == "BSH":
        w = W("BSH", "f32", (2, 90, 3 * 32), 3, 1810, pre_tokens=20, next_tokens=3)
        w.atten_mask = (torch.rand(90, 90, generator=torch.Generator().manual_seed(1811)) < 0.2).to(torch.bool)
    else:
        w = W("BNSD", "f32", (1, 2, 77, 96), 2, 1820)
        w.pse = normal((1, 2, 77, 77), "f32", 1821)
        w.pse_type = 1
    compare_full(w)


@pytest.mark.parametrize("d,kernel", [(32, "sm100_tcgen05"), (96, "sm100_tcgen05"), (100, "simt"),
                                      (256, "sm100_tcgen05"), (204, "simt")])
def test_half_types_other_head_dims(d, kernel):
    w = W("BNSD", "bf16", (1, 2, 150, d), 2, 1900 + d, next_tokens=0)
    assert kernel in plan_text(w)
    compare_full(w)


def test_value_head_dim_smaller():
    w = W("BNSD", "f16", (1, 2, 100, 128), 2, 2000, vshape=(1, 2, 100, 64))
    assert "sm100_tcgen05" in plan_text(w)
    compare_full(w)


# Head dims below the kernel's 64 / 128 columns (zero-padded by the loads):
# dense with a split last wave (the merge kernel writes Dv columns), varlen
# causal with a sink, BSH band with GQA, a value head dim that is not a
# multiple of 32, and rope on top of D = 96.
@pytest.mark.parametrize("dtype,d,dv", [("f16", 96, 96), ("bf16", 128, 64), ("bf16", 80, 48), ("f16", 48, 40),
                                        ("bf16", 120, 88)])
def test_padded_head_dims_split_dense(dtype, d, dv):
    n = 19  # 152 items of 256 rows: on 148 SMs the last wave is split
    w = W("BNSD", dtype, (1, n, 2048, d), n, 4000 + d + dv, vshape=(1, n, 2048, dv))
    text = plan_text(w)
    assert "sm100_tcgen05" in text
    if _sms() == 148:
        assert _split_of(w)[0] > 0
    compare_full(w)


@pytest.mark.parametrize("d,dv", [(96, 96), (128, 72), (40, 40)])
def test_padded_head_dims_varlen_causal_sink(d, dv):
    lens = [300, 0, 513, 129, 1]
    t = sum(lens)
    w = W("TND", "bf16", (t, 4, d), 4, 4100 + d, kshape=(t, 2, d), vshape=(t, 2, dv),
          actual_seq_q=cumulative(lens, False), actual_seq_kv=cumulative(lens, False), next_tokens=0,
          sink=normal((4,), "f32", 4150))
    assert "sm100_tcgen05" in plan_text(w)
    compare_full(w)


# Head dims 129..256: the wide kernel (one query tile at a time, S
# double-buffered, K/V in 128-column halves).
@pytest.mark.parametrize("dtype,d,dv", [("bf16", 256, 256), ("f16", 192, 128), ("bf16", 160, 96)])
def test_wide_head_dims_split_dense(dtype, d, dv):
    n = 19  # 152 items: the last wave is split and merged
    w = W("BNSD", dtype, (1, n, 2048, d), n, 4300 + d + dv, vshape=(1, n, 2048, dv))
    assert "sm100_tcgen05" in plan_text(w)
    if _sms() == 148:
        assert _split_of(w)[0] > 0
    compare_full(w)


@pytest.mark.parametrize("d,dv", [(256, 256), (224, 136)])
def test_wide_head_dims_varlen_causal_sink_gqa(d, dv):
    lens = [300, 0, 513, 129, 1, 640]
    t = sum(lens)
    w = W("TND", "bf16", (t, 4, d), 4, 4400 + d, kshape=(t, 2, d), vshape=(t, 2, dv),
          actual_seq_q=cumulative(lens, False), actual_seq_kv=cumulative(lens, False), next_tokens=0,
          sink=normal((4,), "f32", 4450))
    assert "sm100_tcgen05" in plan_text(w)
    compare_full(w)


def test_wide_head_dims_band_alibi_and_dense_bias_and_mask():
    w = W("BSH", "f16", (2, 420, 2 * 256), 2, 4500, pre_tokens=150, next_tokens=40)
    w.pse, w.pse_type = alibi_slopes(2), 2
    compare_full(w)
    w2 = W("BNSD", "bf16", (1, 2, 333, 256), 2, 4510, kshape=(1, 2, 400, 256), sink=normal((2,), "f32", 4520))
    w2.pse, w2.pse_type = normal((1, 2, 333, 400), "bf16", 4530), 1
    w2.atten_mask = (torch.rand(333, 400, generator=torch.Generator().manual_seed(4540)) < 0.2).to(torch.uint8)
    compare_full(w2)


def test_wide_head_dims_negative_scale_and_single_rows():
    w = W("BNSD", "f16", (1, 2, 1, 256), 2, 4600, kshape=(1, 2, 5, 256), scale=-0.05)
    compare_full(w)
    w = W("BNSD", "bf16", (2, 2, 129, 256), 2, 4610, kshape=(2, 2, 1, 256))
    compare_full(w)


def test_padded_head_dims_bsh_band_alibi():
    w = W("BSH", "f16", (2, 300, 4 * 96), 4, 4200, kshape=(2, 300, 2 * 96), vshape=(2, 300, 2 * 56),
          pre_tokens=90, next_tokens=30)
    w.pse, w.pse_type = alibi_slopes(4), 2
    assert "sm100_tcgen05" in plan_text(w)
    compare_full(w)


# ---------------------------------------------------------------------------
# invariants
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("number", [2, 3])
def test_deterministic_reruns(number):
    w = build(number, seq_scale=8)
    a = run_gpu(w)
    b = run_gpu(w)
    for x, y in zip(a, b):
        assert torch.equal(x, y)


def test_outputs_fully_written():
    """NaN-prefilled outputs: every element is overwritten (no gaps)."""
    w = W("BNSD", "f16", (2, 3, 333, 128), 3, 2100, next_tokens=0)
    q, k, v = w.q.cuda(), w.k.cuda(), w.v.cuda()
    out = torch.full_like(q, float("nan"))
    sm = torch.full((2, 3, 333, 8), float("nan"), device="cuda")
    ss = torch.full((2, 3, 333, 8), float("nan"), device="cuda")
    fa.fa_fwd(q, k, v, input_layout="BNSD", head_num=3, next_tokens=0, out=out, softmax_max=sm, softmax_sum=ss)
    torch.cuda.synchronize()
    assert not out.isnan().any() and not sm.isnan().any() and not ss.isnan().any()


# ---------------------------------------------------------------------------
# the five workloads at full size, as the bench launches them: sampled rows
# ---------------------------------------------------------------------------

def _split_item_rows(w, text):
    """(b, n, i) rows of every split work item of a dense-layout launch: the
    first, a middle and the last row of each of its two 128-row tiles.

    Work item u of the dense layouts is (head bn, query block qb) with the
    heads in groups of `head_group`; inside a group the query blocks run from
    the last to the first, heads fastest.  The split items are the last
    `split_items` of that order."""
    n_split = int(text.split("split_items=")[1].split()[0])
    if n_split == 0:
        return []
    sq = {"BNSD": w.q.shape[2], "BSND": w.q.shape[1], "BSH": w.q.shape[1], "SBH": w.q.shape[0]}[w.layout]
    bsz = w.q.shape[1] if w.layout == "SBH" else w.q.shape[0]
    d = w.q.shape[-1] if w.layout not in ("BSH", "SBH") else w.q.shape[-1] // w.head_num
    hg = 4 if d > 128 else 16
    n_qb = (sq + 255) // 256
    bn_total = bsz * w.head_num
    n_items = n_qb * bn_total
    assert f"items={n_items} " in text
    rows = []
    for u in range(n_items - n_split, n_items):
        g, within = divmod(u, hg * n_qb)
        g_heads = min(hg, bn_total - g * hg)
        level, h = divmod(within, g_heads)
        b, n = divmod(g * hg + h, w.head_num)
        qb = n_qb - 1 - level
        for r in (0, 63, 127, 128, 200, 255):
            if qb * 256 + r < sq:
                rows.append((b, n, qb * 256 + r))
    return rows


@pytest.mark.parametrize("number", [1, 2, 3, 4, 5])
def test_full_size_workloads_sampled(number):
    w = build(number)
    res = run_gpu(w)
    for t in res:
        assert not torch.isnan(t).any()
    rows = sample_rows(w, 24, seed=number)
    if w.layout != "TND" and w.dtype != "f32":
        split_rows = _split_item_rows(w, plan_text(w))
        if number == 2:  # the headline launch splits its short last wave
            assert len(split_rows) >= 2 * 6, "expected split items in the headline launch"
        rows += split_rows
    compare_rows(w, res, rows)


# ---------------------------------------------------------------------------
# Dynamic schedule: equal work items whose last wave is split into key pieces
# and merged (the describe string says how many items were split)
# ---------------------------------------------------------------------------

def _split_of(w):
    text = plan_text(w)
    return int(text.split("split_items=")[1].split()[0]), int(text.split("pieces=")[1].split()[0])


def _sms():
    return torch.cuda.get_device_properties(0).multi_processor_count


@pytest.mark.parametrize("dtype", ["f16", "bf16"])
def test_split_last_wave_dense(dtype):
    n = _sms() + 1  # one item past a full wave: that item is split into 8 key pieces
    w = W("BNSD", dtype, (1, n, 256, 128), n, 3000, kshape=(1, n, 1024, 128))
    assert _split_of(w) == (1, 8)
    res = run_gpu(w)
    compare_full(w, res)
    again = run_gpu(w)
    for a, b in zip(res, again):  # the merge order is fixed: bitwise reruns
        assert torch.equal(a, b)


def test_split_with_sink_gqa_and_ragged_keys():
    n = _sms() + 2
    nkv = n // 2 if n % 2 == 0 else n
    w = W("BNSD", "bf16", (1, n, 256, 64), n, 3100, kshape=(1, nkv, 1000, 64), sink=normal((n,), "f32", 3104))
    items, pieces = _split_of(w)
    assert items == 2 and pieces == 8  # 1000 keys: 8 blocks, the last one ragged
    compare_full(w)


def test_split_random_mask_with_rows_empty_in_some_pieces():
    n = _sms() + 1
    sq, skv = 256, 1024
    w = W("BNSD", "f16", (1, n, sq, 128), n, 3200, kshape=(1, n, skv, 128))
    g = torch.Generator().manual_seed(3205)
    mask = (torch.rand(1, 1, sq, skv, generator=g) < 0.4).to(torch.uint8)
    mask[:, :, :10, : skv // 2] = 1   # rows 0-9: no key in the pieces over the first half
    mask[:, :, 20, :] = 1             # row 20: no key at all (o = 0, m = -inf, l = 0)
    w.atten_mask = mask
    assert _split_of(w) == (1, 8)
    compare_full(w)


# ---------------------------------------------------------------------------
# Dense bias layouts besides [B|1, N|1, Sq, Skv]: the compressed last 1024
# rows of a lower-triangular bias, and the flattened TND bias
# ---------------------------------------------------------------------------

def _alibi_rows(slopes, sq, skv, first_row, dtype):
    i = torch.arange(first_row, sq, dtype=torch.float64)[:, None]
    j = torch.arange(skv, dtype=torch.float64)[None, :]
    return torch.stack([-s * (i - j).abs() for s in slopes])[None].to(DT[dtype])


DT = {"f16": torch.float16, "bf16": torch.bfloat16, "f32": torch.float32}


@pytest.mark.parametrize("dtype,d", [("f16", 64), ("bf16", 128), ("f32", 64)])
def test_compressed_alibi_bias(dtype, d):
    s, n = 1100, 2
    w = W("BNSD", dtype, (1, n, s, d), n, 3300, next_tokens=0, pre_tokens=600)
    w.pse = _alibi_rows([0.5, 0.0625], s, s, s - 1024, dtype)  # [1, N, 1024, S]
    w.pse_type = 1
    compare_full(w)


@pytest.mark.parametrize("dtype,d,s", [("bf16", 128, 1090), ("f16", 64, 1300), ("bf16", 64, 1091)])
def test_compressed_bias_not_translation_invariant(dtype, d, s):
    # arbitrary stored values: the kernel must read them as the oracle's reading
    # says (head dim 64: rows above the stored ones through the per-warp
    # windows, including a warp that straddles the first stored row)
    n = 2
    w = W("BSND", dtype, (2, s, n, d), n, 3310, next_tokens=0, pre_tokens=700)
    w.pse = normal((2, n, 1024, s), dtype, 3315)
    w.pse_type = 1
    compare_full(w)


@pytest.mark.parametrize("dtype,d", [("bf16", 128), ("f16", 64), ("f32", 128)])
def test_tnd_flat_bias(dtype, d):
    lq, lk, n = [300, 129, 700], [260, 400, 700], 2
    w = W("TND", dtype, (sum(lq), n, d), n, 3400, kshape=(sum(lk), n, d),
          actual_seq_q=cumulative(lq, False), actual_seq_kv=cumulative(lk, False))
    w.pse = torch.cat([normal((n, a, b), dtype, 3405 + i).reshape(-1) for i, (a, b) in enumerate(zip(lq, lk))])
    w.pse_type = 1
    compare_full(w)


def test_full_size_band_with_compressed_bias_sampled():
    # the band + ALiBi workload at full size with the bias given as its last
    # 1024 rows (the layout `bench.py --workload 5 --pse compressed` times)
    w = build(5)
    s = w.q.shape[1]
    slopes = w.pse.double().tolist()
    w.pse = _alibi_rows(slopes, s, s, s - 1024, w.dtype)  # [1, 16, 1024, 16384]
    w.pse_type = 1
    res = run_gpu(w)
    for t in res:
        assert not torch.isnan(t).any()
    compare_rows(w, res, sample_rows(w, 16, seed=55))


# ---------------------------------------------------------------------------
# Global positions and the merge of partial results (a forward split along the
# keys: each key chunk run at its kvStartIdx, then fa_lse_merge with the sink)
# ---------------------------------------------------------------------------

from tests.parity import check_out, check_stats, oracle_full  # noqa: E402


def _kv_chunks_merged(w, bounds):
    q = w.q.cuda()
    kw = dict(input_layout=w.layout, head_num=w.head_num, scale=w.scale, pre_tokens=w.pre_tokens,
              next_tokens=w.next_tokens)
    if w.pse is not None:
        kw.update(real_shift=w.pse.cuda(), pse_type=w.pse_type)
    parts = []
    for a, b in bounds:
        kc = w.k[:, :, a:b].contiguous().cuda()
        vc = w.v[:, :, a:b].contiguous().cuda()
        parts.append(fa.fa_fwd(q, kc, vc, kv_start_idx=a, **kw))
    sink = None if w.sink is None else w.sink.cuda()
    res = fa.lse_merge([p_[0] for p_ in parts], [p_[1] for p_ in parts], [p_[2] for p_ in parts],
                       input_layout=w.layout, head_num=w.head_num, sink=sink)
    torch.cuda.synchronize()
    return res


@pytest.mark.parametrize("dtype,d,kw", [
    ("f16", 128, dict(pre_tokens=300, next_tokens=0)),
    ("bf16", 64, dict(pre_tokens=120, next_tokens=40)),
    ("f32", 64, dict(next_tokens=0)),
])
def test_key_chunks_at_their_start_merged(dtype, d, kw):
    n, s = 2, 700
    w = W("BNSD", dtype, (1, n, s, d), n, 3500, sink=normal((n,), "f32", 3504), **kw)
    if dtype == "f16":
        w.pse, w.pse_type = alibi_slopes(n), 2
    out, smax, ssum = _kv_chunks_merged(w, [(0, 256), (256, 500), (500, 700)])
    want = oracle_full(w)
    check_out(f64(out), want["out"], dtype)
    check_stats(f64(smax), want["softmax_max"], "softmaxMax")
    check_stats(f64(ssum), want["softmax_sum"], "softmaxSum")


@pytest.mark.parametrize("dtype,d", [("bf16", 128), ("f32", 64)])
def test_query_chunk_at_its_start(dtype, d):
    n, s, a, b = 2, 640, 200, 530
    w = W("BNSD", dtype, (1, n, s, d), n, 3600, pre_tokens=150, next_tokens=0)
    w.pse, w.pse_type = alibi_slopes(n), 2
    out, smax, ssum = fa.fa_fwd(w.q[:, :, a:b].contiguous().cuda(), w.k.cuda(), w.v.cuda(), input_layout="BNSD",
                                head_num=n, scale=w.scale, pre_tokens=150, next_tokens=0,
                                real_shift=w.pse.cuda(), pse_type=2, q_start_idx=a)
    torch.cuda.synchronize()
    want = oracle_full(w)
    check_out(f64(out), want["out"][:, :, a:b], dtype)
    check_stats(f64(smax), want["softmax_max"][:, :, a:b], "softmaxMax")
    check_stats(f64(ssum), want["softmax_sum"][:, :, a:b], "softmaxSum")


# ---------------------------------------------------------------------------
# queryRope / keyRope: S = scale * (Q K^T + Qr Kr^T) (the V5 page's formula)
# ---------------------------------------------------------------------------

def _rope_case(layout, shape_q, shape_k, dr_shape_q, dr_shape_k, heads, seed, **kw):
    w = W(layout, "bf16", shape_q, heads, seed, kshape=shape_k, **kw)
    qr = normal(dr_shape_q, "bf16", seed + 10)
    kr = normal(dr_shape_k, "bf16", seed + 11)
    return w, qr, kr


def _rope_compare(w, qr, kr, kernel):
    q, k, v, pse, mask, sink = (None if t is None else t.cuda()
                                for t in (w.q, w.k, w.v, w.pse, w.atten_mask, w.sink))
    kw = dict(input_layout=w.layout, head_num=w.head_num, scale=w.scale, atten_mask=mask, sink=sink,
              actual_seq_qlen=w.actual_seq_q, actual_seq_kvlen=w.actual_seq_kv, pre_tokens=w.pre_tokens,
              next_tokens=w.next_tokens, query_rope=qr.cuda(), key_rope=kr.cuda())
    assert kernel in fa.plan(q, k, v, **kw)[2]
    out, smax, ssum = fa.fa_fwd(q, k, v, **kw)
    torch.cuda.synchronize()
    want = ref.forward(f64(w.q), f64(w.k), f64(w.v), layout=w.layout, head_num=w.head_num, scale=w.scale,
                       atten_mask=f64(w.atten_mask), pre_tokens=w.pre_tokens, next_tokens=w.next_tokens,
                       sink=f64(w.sink), actual_seq_q=w.actual_seq_q, actual_seq_kv=w.actual_seq_kv,
                       query_rope=f64(qr), key_rope=f64(kr))
    check_out(f64(out), want["out"], "bf16")
    check_stats(f64(smax), want["softmax_max"], "softmaxMax")
    check_stats(f64(ssum), want["softmax_sum"], "softmaxSum")


from oracle import ref  # noqa: E402


def test_rope_worked_example():
    """The V5 page's call example, rope tensors included: T=256, N=1, D=128,
    Dr=64, everything 1, uint8 mask of zeros, sink 3.0, scale 0.088388."""
    t = 256
    one = torch.ones(t, 1, 128, dtype=torch.bfloat16, device="cuda")
    rope = torch.ones(t, 1, 64, dtype=torch.bfloat16, device="cuda")
    out, smax, ssum = fa.fa_fwd(one, one, one, input_layout="TND", head_num=1, scale=0.088388,
                                atten_mask=torch.zeros(t, t, dtype=torch.uint8, device="cuda"),
                                sink=torch.tensor([3.0], device="cuda"), actual_seq_qlen=[t], actual_seq_kvlen=[t],
                                pre_tokens=65536, next_tokens=65536, softmax_out_layout="same_as_input",
                                query_rope=rope, key_rope=rope)
    torch.cuda.synchronize()
    m = 0.088388 * 192
    assert out.float().eq(1.0).all()
    assert smax.shape == (t, 1, 8)
    check_stats(f64(smax), np.full((t, 1, 8), m), "softmaxMax")
    check_stats(f64(ssum), np.full((t, 1, 8), t + np.exp(3.0 - m)), "softmaxSum")


@pytest.mark.parametrize("case", ["tnd_gqa_causal_sink", "bnsd_d64", "bsh_band", "tnd_d96"])
def test_rope_tcgen05(case):
    if case == "tnd_gqa_causal_sink":
        lens = [300, 0, 513, 129]
        t = sum(lens)
        w, qr, kr = _rope_case("TND", (t, 4, 128), (t, 2, 128), (t, 4, 64), (t, 2, 64), 4, 3700,
                               actual_seq_q=cumulative(lens, False), actual_seq_kv=cumulative(lens, False),
                               next_tokens=0, sink=normal((4,), "f32", 3720))
    elif case == "bnsd_d64":
        w, qr, kr = _rope_case("BNSD", (2, 3, 300, 64), (2, 3, 333, 64), (2, 3, 300, 64), (2, 3, 333, 64), 3, 3730)
    elif case == "bsh_band":
        w, qr, kr = _rope_case("BSH", (2, 260, 2 * 128), (2, 260, 2 * 128), (2, 260, 2 * 64), (2, 260, 2 * 64), 2,
                               3740, pre_tokens=100, next_tokens=20)
    else:
        lens = [200, 333]
        t = sum(lens)
        w, qr, kr = _rope_case("TND", (t, 2, 96), (t, 2, 96), (t, 2, 64), (t, 2, 64), 2, 3760,
                               actual_seq_q=cumulative(lens, False), actual_seq_kv=cumulative(lens, False),
                               next_tokens=0)
    _rope_compare(w, qr, kr, "sm100_tcgen05")


@pytest.mark.parametrize("d,dr", [(96, 32), (64, 128)])
def test_rope_cuda_core_kernel(d, dr):
    lens = [77, 190]
    t = sum(lens)
    w, qr, kr = _rope_case("TND", (t, 2, d), (t, 2, d), (t, 2, dr), (t, 2, dr), 2, 3750 + d,
                           actual_seq_q=cumulative(lens, False), actual_seq_kv=cumulative(lens, False),
                           next_tokens=0)
    _rope_compare(w, qr, kr, "simt")


def test_full_size_varlen_with_rope_sampled():
    """The varlen causal bf16 workload at full size with Dr = 64 rope tensors,
    in the bench's configuration (`bench.py --workload 4 --rope`); sampled rows."""
    w = build(4)
    t, nq = w.q.shape[0], w.head_num
    nkv = w.k.shape[1]
    qr, kr = normal((t, nq, 64), "bf16", 3800), normal((t, nkv, 64), "bf16", 3801)
    q, k, v = w.q.cuda(), w.k.cuda(), w.v.cuda()
    kw = dict(input_layout="TND", head_num=nq, scale=w.scale, actual_seq_qlen=w.actual_seq_q,
              actual_seq_kvlen=w.actual_seq_kv, pre_tokens=w.pre_tokens, next_tokens=w.next_tokens,
              softmax_out_layout=w.softmax_out_layout, query_rope=qr.cuda(), key_rope=kr.cuda())
    assert "sm100_tcgen05" in fa.plan(q, k, v, **kw)[2]
    res = fa.fa_fwd(q, k, v, **kw)
    torch.cuda.synchronize()
    rows = sample_rows(w, 48, seed=7)
    from tests.parity import gather_rows
    o, m, l = gather_rows(w, *res, rows)
    wo, wm, wl = ref.forward_rows(f64(w.q), f64(w.k), f64(w.v), rows, layout="TND", head_num=nq, scale=w.scale,
                                  pre_tokens=w.pre_tokens, next_tokens=w.next_tokens,
                                  actual_seq_q=w.actual_seq_q, actual_seq_kv=w.actual_seq_kv,
                                  query_rope=f64(qr), key_rope=f64(kr))
    check_out(o, wo, "bf16", "sampled attentionOut rows")
    check_stats(m, wm, "sampled softmaxMax")
    check_stats(l, wl, "sampled softmaxSum")


# ---------------------------------------------------------------------------
# The operator's limits (aclnnFlashAttentionVarLenScoreV5, 约束说明: S and T up
# to 1M, B up to 20000, N up to 256), sampled rows against the oracle
# ---------------------------------------------------------------------------

def test_max_sequence_length_band_alibi_sampled():
    s = 1 << 20
    w = W("BNSD", "bf16", (1, 1, s, 64), 1, 5000, pre_tokens=4096, next_tokens=0)
    w.pse, w.pse_type = alibi_slopes(1), 2
    res = run_gpu(w)
    rows = sample_rows(w, 24, seed=1) + [(0, 0, s - 4097), (0, 0, 4095)]
    compare_rows(w, res, rows)


def test_max_tokens_varlen_causal_sampled():
    lens = [262144, 131072, 393216, 262144]  # T = 1M
    t = sum(lens)
    w = W("TND", "bf16", (t, 1, 128), 1, 5100, actual_seq_q=cumulative(lens, False),
          actual_seq_kv=cumulative(lens, False), next_tokens=0, sink=normal((1,), "f32", 5150))
    res = run_gpu(w)
    compare_rows(w, res, sample_rows(w, 12, seed=2))


def test_max_sequences_varlen_sampled():
    rng = np.random.default_rng(5200)
    lens = [int(x) for x in rng.integers(0, 100, size=20000)]  # B = 20000, zero lengths included
    t = sum(lens)
    w = W("TND", "f16", (t, 2, 64), 2, 5210, actual_seq_q=cumulative(lens, False),
          actual_seq_kv=cumulative(lens, False), next_tokens=0, sink=normal((2,), "f32", 5220))
    assert "sm100_tcgen05" in plan_text(w)
    res = run_gpu(w)
    compare_rows(w, res, sample_rows(w, 48, seed=3))
    # every row finite and written (zero-length sequences contribute no rows)
    assert torch.isfinite(res[0].float()).all()


def test_max_heads_gqa():
    w = W("BNSD", "bf16", (1, 256, 200, 64), 256, 5300, kshape=(1, 8, 200, 64), next_tokens=0)
    compare_full(w)


# ---------------------------------------------------------------------------
# Guard bands: outputs and statistics as views into larger buffers filled with
# a sentinel (a guard zone before and after, padding columns in every row);
# nothing outside the logical tensors may change.
# ---------------------------------------------------------------------------

def _guarded(shape, pad, dtype, sentinel=-7777.0, guard=4096):
    padded = tuple(shape[:-1]) + (shape[-1] + pad,)
    n = int(np.prod(padded))
    base = torch.full((guard + n + guard,), sentinel, dtype=dtype, device="cuda")
    view = base[guard:guard + n].view(padded)[..., :shape[-1]]
    return base, view, (guard, n, padded)


def _guards_intact(base, meta, width, sentinel=-7777.0):
    guard, n, padded = meta
    s = torch.tensor(sentinel, dtype=base.dtype, device="cuda")
    assert torch.equal(base[:guard], s.expand(guard)), "write before the tensor"
    assert torch.equal(base[guard + n:], s.expand(base.numel() - guard - n)), "write after the tensor"
    pad_cols = base[guard:guard + n].view(padded)[..., width:]
    assert torch.equal(pad_cols, s.expand_as(pad_cols)), "write into a row's padding"


@pytest.mark.parametrize("case", ["dense_split_dv40", "varlen_ragged", "wide_dv136", "sbh_band"])
def test_outputs_stay_inside_their_tensors(case):
    dtype = torch.bfloat16
    if case == "dense_split_dv40":
        w = W("BNSD", "bf16", (1, 19, 2048, 48), 19, 5500, vshape=(1, 19, 2048, 40))
        out_shape, st_shape = (1, 19, 2048, 40), (1, 19, 2048, 8)
    elif case == "varlen_ragged":
        lens = [129, 0, 300, 1, 255]
        t = sum(lens)
        w = W("TND", "bf16", (t, 3, 128), 3, 5510, actual_seq_q=cumulative(lens, False),
              actual_seq_kv=cumulative(lens, False), next_tokens=0, sink=normal((3,), "f32", 5515))
        out_shape, st_shape = (t, 3, 128), (3, t, 8)
    elif case == "wide_dv136":
        w = W("BNSD", "f16", (1, 2, 333, 256), 2, 5520, vshape=(1, 2, 333, 136), next_tokens=0)
        out_shape, st_shape, dtype = (1, 2, 333, 136), (1, 2, 333, 8), torch.float16
    else:
        w = W("SBH", "bf16", (300, 2, 2 * 64), 2, 5530, pre_tokens=90, next_tokens=7)
        out_shape, st_shape = (300, 2, 2 * 64), (2, 2, 300, 8)
    ob, ov, om = _guarded(out_shape, 16, dtype)
    mb, mv, mm = _guarded(st_shape, 8, torch.float32)
    lb, lv, lm = _guarded(st_shape, 8, torch.float32)
    res = run_gpu(w, out=ov, softmax_max=mv, softmax_sum=lv)
    _guards_intact(ob, om, out_shape[-1])
    _guards_intact(mb, mm, 8)
    _guards_intact(lb, lm, 8)
    compare_full(w, res=res)
