"""Pins for the float64 oracle: each check comes from something other than the
oracle itself — the pages' worked example, a closed form, a library routine
that computes the same definition, a brute-force twin, or an invariant.
CPU only."""
import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import ref, brute
from workloads import normal, causal_mask_u8, alibi_slopes, cumulative

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
INT64_MAX = ref.INT64_MAX


def f64(t):
    return t.double().numpy()


def rand(shape, seed):
    return f64(normal(shape, "f32", seed))


# ---------------------------------------------------------------------------
# The pages' worked example (aclnnFlashAttentionVarLenScoreV5, call example).
# ---------------------------------------------------------------------------

def test_worked_example_sink_closed_form():
    g = json.load(open(os.path.join(GOLDEN, "sink_example_tnd.json")))
    t, n, d = g["T"], g["N"], g["D"]
    one = torch.ones(t, n, d, dtype=torch.bfloat16)
    res = ref.forward(f64(one), f64(one), f64(one), layout="TND", head_num=n,
                      scale=g["scale"], atten_mask=np.zeros((t, t), np.uint8),
                      pre_tokens=g["pre_tokens"], next_tokens=g["next_tokens"],
                      sink=np.array([g["host_fill"]["sink"]]),
                      actual_seq_q=g["actual_seq_q"], actual_seq_kv=g["actual_seq_kv"],
                      softmax_out_layout=g["softmax_out_layout"])
    exp = g["expected_without_rope"]
    assert res["softmax_max"].shape == tuple(g["stats_shape"])
    assert res["out"].shape == tuple(g["out_shape"])
    np.testing.assert_allclose(res["softmax_max"], exp["softmax_max"], rtol=1e-12)
    np.testing.assert_allclose(res["softmax_sum"], exp["softmax_sum"], rtol=1e-12)
    np.testing.assert_allclose(res["out"], exp["out"], rtol=1e-12)
    # the stored values are the closed form of the fixture's notes
    s = g["scale"] * d
    m = max(3.0, s)
    l = t * math.exp(s - m) + math.exp(3.0 - m)
    assert abs(exp["softmax_sum"] - l) < 1e-9 and abs(exp["out"] - t * math.exp(s - m) / l) < 1e-12
    # rounded to bf16 the output is exactly 1.0
    assert torch.tensor(res["out"]).to(torch.bfloat16).float().eq(1.0).all()


def test_worked_example_with_rope_closed_form():
    """The page's exact call, queryRope/keyRope [256, 1, 64] of ones included:
    every score is scale * (128 + 64)."""
    g = json.load(open(os.path.join(GOLDEN, "sink_example_tnd.json")))
    t, n, d, dr = g["T"], g["N"], g["D"], g["rope_dim"]
    one = f64(torch.ones(t, n, d, dtype=torch.bfloat16))
    rope = f64(torch.ones(t, n, dr, dtype=torch.bfloat16))
    res = ref.forward(one, one, one, layout="TND", head_num=n, scale=g["scale"],
                      atten_mask=np.zeros((t, t), np.uint8),
                      pre_tokens=g["pre_tokens"], next_tokens=g["next_tokens"],
                      sink=np.array([g["host_fill"]["sink"]]),
                      actual_seq_q=g["actual_seq_q"], actual_seq_kv=g["actual_seq_kv"],
                      softmax_out_layout=g["softmax_out_layout"], query_rope=rope, key_rope=rope)
    exp = g["expected_with_rope"]
    np.testing.assert_allclose(res["softmax_max"], exp["softmax_max"], rtol=1e-12)
    np.testing.assert_allclose(res["softmax_sum"], exp["softmax_sum"], rtol=1e-12)
    np.testing.assert_allclose(res["out"], exp["out"], rtol=1e-12)
    s = g["scale"] * (d + dr)
    assert abs(exp["softmax_max"] - s) < 1e-9
    assert abs(exp["softmax_sum"] - (t + math.exp(3.0 - s))) < 1e-9


# ---------------------------------------------------------------------------
# Reduction to a library routine: torch scaled_dot_product_attention (float64).
# ---------------------------------------------------------------------------

def _sdpa(q, k, v, scale, bias):
    """torch SDPA on one head with an additive float bias (-inf = excluded)."""
    qt, kt, vt = (torch.from_numpy(x)[None, None] for x in (q, k, v))
    b = torch.from_numpy(bias)[None, None]
    out = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=b, scale=scale)
    scores = scale * (torch.from_numpy(q) @ torch.from_numpy(k).T) + torch.from_numpy(bias)
    return out[0, 0].numpy(), torch.logsumexp(scores, dim=-1).numpy()


@pytest.mark.parametrize("sq,skv,d,dv,pre,nxt", [
    (37, 53, 16, 16, INT64_MAX, INT64_MAX),
    (64, 64, 32, 24, 10, 0),
    (50, 70, 8, 8, 5, 30),
])
def test_head_matches_sdpa(sq, skv, d, dv, pre, nxt):
    q, k, v = rand((sq, d), 1), rand((skv, d), 2), rand((skv, dv), 3)
    pse = rand((sq, skv), 4)
    rng = np.random.default_rng(5)
    excluded = rng.random((sq, skv)) < 0.2
    scale = 0.37
    o, m, l = ref.head_forward(q, k, v, scale, pse=pse, excluded=excluded,
                               pre_tokens=pre, next_tokens=nxt)
    # the bias the test hands to SDPA: pse where kept, -inf where excluded by
    # the mask or outside the band
    i = np.arange(sq)[:, None]
    j = np.arange(skv)[None, :]
    outside = (j - i < -pre) | (j - i > nxt) | excluded
    bias = np.where(outside, -np.inf, pse)
    live = ~outside.all(axis=1)
    o_ref, lse = _sdpa(q, k, v, scale, bias)
    np.testing.assert_allclose(o[live], o_ref[live], rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose((m + np.log(l))[live], lse[live], rtol=1e-12, atol=1e-12)


def test_sink_matches_sdpa_with_extra_key():
    """A sink is an extra key column with logit sink_n and a zero value row."""
    sq, skv, d = 40, 33, 16
    q, k, v = rand((sq, d), 11), rand((skv, d), 12), rand((skv, d), 13)
    sink, scale = 1.7, 0.25
    o, m, l = ref.head_forward(q, k, v, scale, sink=sink, next_tokens=0)
    # extra key j = -1 placed first: q . 0 = 0, bias = sink, value 0
    k2 = np.vstack([np.zeros((1, d)), k])
    v2 = np.vstack([np.zeros((1, d)), v])
    i = np.arange(sq)[:, None]
    j = np.arange(skv)[None, :]
    bias = np.hstack([np.full((sq, 1), sink), np.where(j - i > 0, -np.inf, 0.0)])
    o_ref, lse = _sdpa(q, k2, v2, scale, bias)
    np.testing.assert_allclose(o, o_ref, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(m + np.log(l), lse, rtol=1e-12)
    assert (m >= sink).all()


# ---------------------------------------------------------------------------
# Brute force: the sink formula typed out with Python scalars.
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("with_sink,with_pse,with_mask,pre,nxt", [
    (False, False, False, INT64_MAX, INT64_MAX),
    (True, False, False, INT64_MAX, 0),
    (True, True, True, 2, 1),
    (False, True, False, 1, -1),
])
def test_ref_matches_brute(with_sink, with_pse, with_mask, pre, nxt):
    sq, skv, d, dv = 5, 4, 3, 2
    q, k, v = rand((sq, d), 21), rand((skv, d), 22), rand((skv, dv), 23)
    pse = rand((sq, skv), 24) if with_pse else None
    excl = (np.random.default_rng(25).random((sq, skv)) < 0.3) if with_mask else None
    sink = 0.4 if with_sink else None
    o, m, l = ref.head_forward(q, k, v, 0.6, pse=pse, excluded=excl,
                               pre_tokens=pre, next_tokens=nxt, sink=sink)
    ob, mb, lb = brute.head_forward(q.tolist(), k.tolist(), v.tolist(), 0.6,
                                    pse=None if pse is None else pse.tolist(),
                                    excluded=None if excl is None else excl.tolist(),
                                    pre_tokens=pre, next_tokens=nxt, sink=sink)
    np.testing.assert_allclose(o, np.array(ob), rtol=1e-12, atol=1e-14)
    np.testing.assert_array_equal(np.isinf(m), np.isinf(np.array(mb)))
    fin = np.isfinite(m)
    np.testing.assert_allclose(m[fin], np.array(mb)[fin], rtol=1e-13)
    np.testing.assert_allclose(l, np.array(lb), rtol=1e-12)


@pytest.mark.parametrize("with_sink,pre,nxt", [(False, INT64_MAX, INT64_MAX), (True, 2, 0)])
def test_rope_matches_brute(with_sink, pre, nxt):
    sq, skv, d, dr, dv = 5, 6, 3, 2, 2
    q, k, v = rand((sq, d), 31), rand((skv, d), 32), rand((skv, dv), 33)
    qr, kr = rand((sq, dr), 34), rand((skv, dr), 35)
    sink = -0.3 if with_sink else None
    o, m, l = ref.head_forward(q, k, v, 0.7, pre_tokens=pre, next_tokens=nxt, sink=sink, q_rope=qr, k_rope=kr)
    ob, mb, lb = brute.head_forward(q.tolist(), k.tolist(), v.tolist(), 0.7, pre_tokens=pre, next_tokens=nxt,
                                    sink=sink, q_rope=qr.tolist(), k_rope=kr.tolist())
    np.testing.assert_allclose(o, np.array(ob), rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(m, np.array(mb), rtol=1e-13)
    np.testing.assert_allclose(l, np.array(lb), rtol=1e-12)


# ---------------------------------------------------------------------------
# Closed forms.
# ---------------------------------------------------------------------------

def test_constant_value_returns_constant():
    q, k = rand((30, 8), 31), rand((45, 8), 32)
    v = np.full((45, 5), 2.5)
    o, _, _ = ref.head_forward(q, k, v, 0.3, next_tokens=3, pre_tokens=10)
    np.testing.assert_allclose(o, 2.5, rtol=1e-13)


def test_constant_value_with_sink():
    q, k = rand((20, 8), 33), rand((20, 8), 34)
    v = np.full((20, 3), -1.5)
    o, m, l = ref.head_forward(q, k, v, 0.3, sink=0.8)
    np.testing.assert_allclose(o, np.broadcast_to(-1.5 * (1.0 - np.exp(0.8 - m) / l)[:, None], o.shape), rtol=1e-12)


def test_causal_first_row_is_v0():
    q, k, v = rand((16, 8), 41), rand((16, 8), 42), rand((16, 8), 43)
    o, m, l = ref.head_forward(q, k, v, 0.5, next_tokens=0)
    np.testing.assert_allclose(o[0], v[0], rtol=1e-14)
    assert l[0] == 1.0
    np.testing.assert_allclose(m[0], 0.5 * q[0] @ k[0], rtol=1e-14)


@pytest.mark.parametrize("sq,skv,pre,nxt", [
    (40, 40, INT64_MAX, 0), (40, 40, 7, 0), (33, 50, 4, 9), (50, 20, 0, 0), (25, 25, 3, -2)])
def test_zero_query_band_counts(sq, skv, pre, nxt):
    """With Q = 0 and no pse every kept score is 0: m = 0, l = number of kept
    keys = min(Skv-1, i+next) - max(0, i-pre) + 1 (inclusive band, top-left
    aligned), and o = mean of the kept value rows."""
    q = np.zeros((sq, 4))
    k, v = rand((skv, 4), 51), rand((skv, 3), 52)
    o, m, l = ref.head_forward(q, k, v, 1.0, pre_tokens=pre, next_tokens=nxt)
    for i in range(sq):
        lo = max(0, i - pre) if pre < INT64_MAX else 0
        hi = min(skv - 1, i + nxt)
        count = max(0, hi - lo + 1)
        if count == 0:
            assert m[i] == -np.inf and l[i] == 0 and (o[i] == 0).all()
            continue
        assert m[i] == 0.0 and l[i] == count
        np.testing.assert_allclose(o[i], v[lo:hi + 1].mean(axis=0), rtol=1e-12, atol=1e-14)


def test_alibi_geometric_series():
    """Q = 0, ALiBi slope s, causal band of width pre: the kept weights are
    r^0..r^K with r = e^-s and K = min(i, pre), so l = (1 - r^(K+1))/(1 - r)."""
    sq, n_heads, pre = 64, 4, 9
    slopes = f64(alibi_slopes(n_heads))
    q = np.zeros((1, sq, n_heads, 8))
    k, v = rand((1, sq, n_heads, 8), 61), rand((1, sq, n_heads, 8), 62)
    res = ref.forward(q, k, v, layout="BSND", head_num=n_heads, scale=1.0,
                      pse=slopes, pse_type=2, pre_tokens=pre, next_tokens=0)
    for n in range(n_heads):
        r = math.exp(-slopes[n])
        for i in range(sq):
            kk = min(i, pre)
            l_exact = (1 - r ** (kk + 1)) / (1 - r)
            assert res["softmax_max"][0, n, i, 0] == 0.0
            np.testing.assert_allclose(res["softmax_sum"][0, n, i], l_exact, rtol=1e-13)


def per_batch_slopes(n_batch, n_heads):
    """fp32 [B, N] ALiBi slopes that differ along both axes and are not
    symmetric: slope[b, n] = 2^(-(n+1)) * (1 + 0.37 b) + 0.05 n b."""
    b = np.arange(n_batch, dtype=np.float64)[:, None]
    n = np.arange(n_heads, dtype=np.float64)[None, :]
    return (2.0 ** -(n + 1) * (1 + 0.37 * b) + 0.05 * n * b).astype(np.float32)


@pytest.mark.parametrize("layout", ["BSND", "TND"])
def test_alibi_geometric_series_per_batch_slopes(layout):
    """The [B, N] slope form (aclnnFlashAttentionVarLenScoreV5, realShiftOptional
    notes: a slope-only pse of shape [B, N] or [N]): batch row b, head n use
    slope[b, n].  Q = 0, causal band of width pre: l = (1 - r^(K+1))/(1 - r)
    with r = e^-slope[b, n] and K = min(i, pre), as for [N] slopes, but with a
    different r for every (b, n); for TND, b is the sequence."""
    n_batch, n_heads, pre = 3, 3, 9
    slopes = per_batch_slopes(n_batch, n_heads).astype(np.float64)
    assert not np.allclose(slopes, slopes.T)
    if layout == "BSND":
        lens = [40] * n_batch
        q = np.zeros((n_batch, 40, n_heads, 8))
        k, v = rand((n_batch, 40, n_heads, 8), 65), rand((n_batch, 40, n_heads, 8), 66)
        res = ref.forward(q, k, v, layout="BSND", head_num=n_heads, scale=1.0,
                          pse=slopes, pse_type=2, pre_tokens=pre, next_tokens=0)
        lsum = lambda b, n, i: res["softmax_sum"][b, n, i]  # noqa: E731
        lmax = lambda b, n, i: res["softmax_max"][b, n, i]  # noqa: E731
    else:
        lens = [23, 40, 17]
        t = sum(lens)
        q = np.zeros((t, n_heads, 8))
        k, v = rand((t, n_heads, 8), 67), rand((t, n_heads, 8), 68)
        cu = cumulative(lens, False)
        res = ref.forward(q, k, v, layout="TND", head_num=n_heads, scale=1.0, pse=slopes, pse_type=2,
                          pre_tokens=pre, next_tokens=0, actual_seq_q=cu, actual_seq_kv=cu)
        starts = [0] + cu[:-1]
        lsum = lambda b, n, i: res["softmax_sum"][n, starts[b] + i]  # noqa: E731
        lmax = lambda b, n, i: res["softmax_max"][n, starts[b] + i]  # noqa: E731
    for b in range(n_batch):
        for n in range(n_heads):
            r = math.exp(-slopes[b, n])
            for i in range(lens[b]):
                kk = min(i, pre)
                assert np.all(lmax(b, n, i) == 0.0)
                np.testing.assert_allclose(lsum(b, n, i), (1 - r ** (kk + 1)) / (1 - r), rtol=1e-13)


def test_alibi_symmetric_band():
    """Q = 0, ALiBi slope s, band [i - pre, i + next]: the kept weights are
    r^|i-j|, so l = sum over the two one-sided geometric series
    (1 - r^(a+1))/(1 - r) + r (1 - r^b)/(1 - r), a = min(i, pre),
    b = min(S-1-i, next)."""
    s, n_heads, pre, nxt = 40, 2, 6, 11
    slopes = f64(alibi_slopes(n_heads))
    q = np.zeros((1, n_heads, s, 8))
    k, v = rand((1, n_heads, s, 8), 63), rand((1, n_heads, s, 8), 64)
    res = ref.forward(q, k, v, layout="BNSD", head_num=n_heads, scale=1.0,
                      pse=slopes, pse_type=2, pre_tokens=pre, next_tokens=nxt)
    for n in range(n_heads):
        r = math.exp(-slopes[n])
        for i in range(s):
            a, b = min(i, pre), min(s - 1 - i, nxt)
            l_exact = (1 - r ** (a + 1)) / (1 - r) + r * (1 - r ** b) / (1 - r)
            np.testing.assert_allclose(res["softmax_sum"][0, n, i], l_exact, rtol=1e-13)


def test_empty_rows():
    q, k, v = rand((6, 4), 71), rand((6, 4), 72), rand((6, 4), 73)
    excl = np.zeros((6, 6), bool)
    excl[2, :] = True
    o, m, l = ref.head_forward(q, k, v, 1.0, excluded=excl)
    assert (o[2] == 0).all() and m[2] == -np.inf and l[2] == 0
    o, m, l = ref.head_forward(q, k, v, 1.0, excluded=excl, sink=-0.3)
    assert (o[2] == 0).all() and m[2] == -0.3 and l[2] == 1.0
    # a band that leaves row 0 empty (nextTokens < 0)
    o, m, l = ref.head_forward(q, k, v, 1.0, pre_tokens=3, next_tokens=-1)
    assert m[0] == -np.inf and l[0] == 0 and (o[0] == 0).all()


def test_identity_value_exposes_probability_rows():
    """With V = I the output row is the softmax row itself: it sums to 1, and
    to 1 - e^(sink-m)/l with a sink."""
    s = 24
    q, k = rand((s, 8), 81), rand((s, 8), 82)
    eye = np.eye(s)
    o, m, l = ref.head_forward(q, k, eye, 0.4, next_tokens=0)
    np.testing.assert_allclose(o.sum(axis=1), 1.0, rtol=1e-13)
    assert (np.triu(o, 1) == 0).all()
    assert (o >= 0).all() and ((l >= 1) & (l <= np.arange(1, s + 1))).all()
    o, m, l = ref.head_forward(q, k, eye, 0.4, sink=0.9)
    np.testing.assert_allclose(o.sum(axis=1), 1.0 - np.exp(0.9 - m) / l, rtol=1e-13)


# ---------------------------------------------------------------------------
# Invariants across layouts, varlen, heads.
# ---------------------------------------------------------------------------

def _bnsd_to(x, layout):
    if layout == "BNSD":
        return x
    if layout == "BSND":
        return x.transpose(0, 2, 1, 3)
    b, n, s, d = x.shape
    if layout == "BSH":
        return x.transpose(0, 2, 1, 3).reshape(b, s, n * d)
    if layout == "SBH":
        return x.transpose(2, 0, 1, 3).reshape(s, b, n * d)
    raise ValueError(layout)


def test_layouts_agree():
    b, n, s, d = 2, 3, 21, 8
    q, k, v = rand((b, n, s, d), 91), rand((b, n, s, d), 92), rand((b, n, s, d), 93)
    sink = rand((n,), 94)
    base = ref.forward(q, k, v, layout="BNSD", head_num=n, scale=0.3, next_tokens=0, sink=sink)
    for layout in ("BSND", "BSH", "SBH"):
        res = ref.forward(_bnsd_to(q, layout), _bnsd_to(k, layout), _bnsd_to(v, layout),
                          layout=layout, head_num=n, scale=0.3, next_tokens=0, sink=sink)
        np.testing.assert_array_equal(res["out"], _bnsd_to(base["out"], layout))
        np.testing.assert_array_equal(res["softmax_max"], base["softmax_max"])
        np.testing.assert_array_equal(res["softmax_sum"], base["softmax_sum"])


def test_varlen_equals_each_sequence_alone():
    lens, n, d = [5, 0, 17, 9], 2, 8
    t = sum(lens)
    q, k, v = rand((t, n, d), 101), rand((t, n, d), 102), rand((t, n, d), 103)
    cum = cumulative(lens, leading_zero=False)
    res = ref.forward(q, k, v, layout="TND", head_num=n, scale=0.5, next_tokens=0,
                      actual_seq_q=cum, actual_seq_kv=cum, softmax_out_layout="same_as_input")
    res_ntd = ref.forward(q, k, v, layout="TND", head_num=n, scale=0.5, next_tokens=0,
                          actual_seq_q=cum, actual_seq_kv=cum)
    np.testing.assert_array_equal(res_ntd["softmax_max"], res["softmax_max"].transpose(1, 0, 2))
    start = 0
    for length in lens:
        if length:
            sl = slice(start, start + length)
            one = ref.forward(q[sl].transpose(1, 0, 2)[None], k[sl].transpose(1, 0, 2)[None],
                              v[sl].transpose(1, 0, 2)[None], layout="BNSD", head_num=n,
                              scale=0.5, next_tokens=0)
            np.testing.assert_array_equal(res["out"][sl], one["out"][0].transpose(1, 0, 2))
            np.testing.assert_array_equal(res["softmax_sum"][sl], one["softmax_sum"][0].transpose(1, 0, 2))
        start += length


def test_permuting_keys_leaves_output_unchanged():
    q, k, v = rand((12, 8), 111), rand((19, 8), 112), rand((19, 6), 113)
    perm = np.random.default_rng(114).permutation(19)
    o1, m1, l1 = ref.head_forward(q, k, v, 0.7)
    o2, m2, l2 = ref.head_forward(q, k[perm], v[perm], 0.7)
    np.testing.assert_allclose(o1, o2, rtol=1e-12)
    np.testing.assert_allclose(m1, m2, rtol=1e-15)
    np.testing.assert_allclose(l1, l2, rtol=1e-13)


def test_gqa_equals_repeated_kv_heads():
    b, nq, nkv, s, d = 1, 4, 2, 10, 8
    q = rand((b, nq, s, d), 121)
    k, v = rand((b, nkv, s, d), 122), rand((b, nkv, s, d), 123)
    res = ref.forward(q, k, v, layout="BNSD", head_num=nq, scale=0.4)
    rep = ref.forward(q, np.repeat(k, 2, axis=1), np.repeat(v, 2, axis=1), layout="BNSD",
                      head_num=nq, scale=0.4)
    np.testing.assert_array_equal(res["out"], rep["out"])


def test_mask_tensor_broadcast_forms_agree():
    b, n, s, d = 2, 2, 9, 4
    q, k, v = rand((b, n, s, d), 131), rand((b, n, s, d), 132), rand((b, n, s, d), 133)
    m2 = causal_mask_u8(s, s).numpy()
    outs = []
    for mask in (m2, m2[None, None], np.broadcast_to(m2, (b, 1, s, s)), np.broadcast_to(m2, (b, n, s, s))):
        outs.append(ref.forward(q, k, v, layout="BNSD", head_num=n, scale=0.5, atten_mask=mask)["out"])
    band = ref.forward(q, k, v, layout="BNSD", head_num=n, scale=0.5, next_tokens=0)["out"]
    for o in outs:
        np.testing.assert_array_equal(o, band)


def test_forward_rows_matches_forward():
    b, n, s, d = 2, 3, 30, 8
    q, k, v = rand((b, s, n, d), 141), rand((b, s, n, d), 142), rand((b, s, n, d), 143)
    sink = rand((n,), 144)
    full = ref.forward(q, k, v, layout="BSND", head_num=n, scale=0.3, pre_tokens=6,
                       next_tokens=0, sink=sink)
    rows = [(0, 0, 0), (1, 2, 29), (0, 1, 17)]
    o, m, l = ref.forward_rows(q, k, v, rows, layout="BSND", head_num=n, scale=0.3,
                               pre_tokens=6, next_tokens=0, sink=sink)
    for r, (bb, nn, i) in enumerate(rows):
        # a one-row product may round differently from the blocked one
        np.testing.assert_allclose(o[r], full["out"][bb, i, nn], rtol=1e-13, atol=1e-15)
        np.testing.assert_allclose(m[r], full["softmax_max"][bb, nn, i, 0], rtol=1e-14)
        np.testing.assert_allclose(l[r], full["softmax_sum"][bb, nn, i, 0], rtol=1e-13)


# ---------------------------------------------------------------------------
# Dense bias layouts besides [B|1, N|1, Sq, Skv]
# (aclnnFlashAttentionVarLenScoreV5, realShiftOptional and its notes).
# ---------------------------------------------------------------------------

def _alibi_full(slopes, sq, skv):
    i = np.arange(sq, dtype=np.float64)[:, None]
    j = np.arange(skv, dtype=np.float64)[None, :]
    return np.stack([-s * np.abs(i - j) for s in slopes])[None]  # [1, N, Sq, Skv]


@pytest.mark.parametrize("nxt", [0, -3])
def test_compressed_alibi_bias_equals_slopes(nxt):
    # The last 1024 rows of an ALiBi bias (alibi_compress = pse[:, :, -1024:, :])
    # under a lower-triangular band reproduce the slope-generated bias, which
    # the oracle computes from -slope * |i - j| on its own path (pse type 2).
    s, n, d = 1100, 2, 8
    q, k, v = rand((1, n, s, d), 901), rand((1, n, s, d), 902), rand((1, n, s, d), 903)
    slopes = np.array([0.5, 0.03125])
    full = _alibi_full(slopes, s, s)
    kw = dict(layout="BNSD", head_num=n, scale=d ** -0.5, pre_tokens=300, next_tokens=nxt)
    want = ref.forward(q, k, v, pse=slopes, pse_type=2, **kw)
    got_full = ref.forward(q, k, v, pse=full, pse_type=1, **kw)
    got_c = ref.forward(q, k, v, pse=full[:, :, -1024:, :].copy(), pse_type=1, **kw)
    for got in (got_full, got_c):
        np.testing.assert_allclose(got["out"], want["out"], rtol=0, atol=1e-12)
        np.testing.assert_allclose(got["softmax_max"], want["softmax_max"], rtol=1e-13)
        np.testing.assert_allclose(got["softmax_sum"], want["softmax_sum"], rtol=1e-12)


def test_compressed_bias_rows_are_read_along_the_diagonal():
    # a bias that is not a function of i - j tells apart which stored entry
    # each full-bias position reads: rows at or below Sq - 1024 read their own
    # stored row; a row above reads stored row 0 shifted by (Sq - 1024 - i)
    s, n = 1030, 1
    stored = rand((1, n, 1024, s), 904)
    rows = np.array([0, 3, 5, 6, 700, 1029])
    got = ref._pse_rows(stored, 1, 0, 0, rows, s, seqs=[(0, s, 0, s)], n_heads=n)
    first = s - 1024
    for r_, i in enumerate(rows):
        for j in (0, 1, i - 1, i):
            if j < 0:
                continue
            want = stored[0, 0, i - first, j] if i >= first else stored[0, 0, 0, j + first - i]
            assert got[r_, j] == want


def test_tnd_flat_bias_equals_each_sequence_with_its_own_bias():
    lq, lk, n, d = [5, 9, 3], [7, 4, 6], 2, 8
    q = rand((sum(lq), n, d), 911)
    k = rand((sum(lk), n, d), 912)
    v = rand((sum(lk), n, d), 913)
    blocks = [rand((n, a, b), 914 + i) for i, (a, b) in enumerate(zip(lq, lk))]
    flat = np.concatenate([x.reshape(-1) for x in blocks])
    res = ref.forward(q, k, v, layout="TND", head_num=n, scale=0.3, pse=flat, pse_type=1,
                      actual_seq_q=cumulative(lq, False), actual_seq_kv=cumulative(lk, False))
    cq, ck = [0] + cumulative(lq, False), [0] + cumulative(lk, False)
    for b in range(len(lq)):
        one = ref.forward(q[None, cq[b]:cq[b + 1]].transpose(0, 2, 1, 3), k[None, ck[b]:ck[b + 1]].transpose(0, 2, 1, 3),
                          v[None, ck[b]:ck[b + 1]].transpose(0, 2, 1, 3), layout="BNSD", head_num=n, scale=0.3,
                          pse=blocks[b][None], pse_type=1)
        np.testing.assert_allclose(res["out"][cq[b]:cq[b + 1]], one["out"][0].transpose(1, 0, 2), atol=1e-13)
        np.testing.assert_allclose(res["softmax_max"][:, cq[b]:cq[b + 1], 0], one["softmax_max"][0, :, :, 0],
                                   rtol=1e-13)


# ---------------------------------------------------------------------------
# Global positions (qStartIdx / kvStartIdx) and the merge of partial results
# ---------------------------------------------------------------------------

def _chunked_forward(q, k, v, n, bounds, **kw):
    sink = kw.pop("sink", None)
    parts = [ref.forward(q, k[:, :, a:b], v[:, :, a:b], layout="BNSD", head_num=n, kv_start=a, **kw)
             for a, b in bounds]
    o, m, l = ref.merge([p_["out"] for p_ in parts], [p_["softmax_max"][..., 0] for p_ in parts],
                        [p_["softmax_sum"][..., 0] for p_ in parts],
                        sink=None if sink is None else np.asarray(sink)[None, :, None])
    return o, m, l


@pytest.mark.parametrize("kw", [dict(pre_tokens=90, next_tokens=0),
                                dict(pre_tokens=40, next_tokens=25),
                                dict(next_tokens=0, pse_type=2)])
def test_key_chunks_at_their_start_merge_to_the_whole(kw):
    # the whole forward regrouped by key chunk: each chunk sees its keys at
    # global positions (kv_start) and the merge combines the chunks' rows
    n, s, d = 2, 200, 16
    q, k, v = rand((1, n, s, d), 931), rand((1, n, s, d), 932), rand((1, n, s, d), 933)
    sink = np.array([0.7, -1.3])
    kw = dict(kw)
    if kw.get("pse_type") == 2:
        kw["pse"] = np.array([0.25, 0.0625])
    whole = ref.forward(q, k, v, layout="BNSD", head_num=n, scale=0.3, sink=sink, **kw)
    o, m, l = _chunked_forward(q, k, v, n, [(0, 70), (70, 130), (130, 200)], scale=0.3, sink=sink, **kw)
    np.testing.assert_allclose(o, whole["out"], rtol=0, atol=1e-12)
    np.testing.assert_allclose(m, whole["softmax_max"][..., 0], rtol=1e-13)
    np.testing.assert_allclose(l, whole["softmax_sum"][..., 0], rtol=1e-12)


def test_query_chunk_at_its_start_equals_rows_of_the_whole():
    n, s, d = 2, 160, 8
    q, k, v = rand((1, n, s, d), 941), rand((1, n, s, d), 942), rand((1, n, s, d), 943)
    kw = dict(layout="BNSD", head_num=n, scale=0.4, pre_tokens=50, next_tokens=3, pse=np.array([0.5, 0.125]),
              pse_type=2)
    whole = ref.forward(q, k, v, **kw)
    part = ref.forward(q[:, :, 100:140], k, v, q_start=100, **kw)
    np.testing.assert_allclose(part["out"], whole["out"][:, :, 100:140], atol=1e-13)
    np.testing.assert_allclose(part["softmax_sum"], whole["softmax_sum"][:, :, 100:140], rtol=1e-13)


def test_merge_of_empty_parts():
    # rows with no key in any part: o = 0, m = -inf, l = 0; with a sink m = sink, l = 1
    o, m, l = ref.merge([np.zeros((3, 4))] * 2, [np.full(3, -np.inf)] * 2, [np.zeros(3)] * 2)
    assert (o == 0).all() and np.isneginf(m).all() and (l == 0).all()
    o, m, l = ref.merge([np.zeros((3, 4))], [np.full(3, -np.inf)], [np.zeros(3)], sink=np.full(3, 2.0))
    assert (o == 0).all() and (m == 2.0).all() and (l == 1.0).all()


# ---------------------------------------------------------------------------
# queryRope / keyRope (aclnnFlashAttentionVarLenScoreV5 formula): the sum of
# the two dot products is one dot product over the joined head dims.
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("layout", ["BSH", "TND"])
def test_rope_equals_joined_head_dim(layout):
    n_q, n_kv, d, dr, dv = 4, 2, 8, 4, 6
    kw = dict(pre_tokens=9, next_tokens=0, sink=np.array([0.2, -1.0, 0.5, 1.5]))
    if layout == "TND":
        lens_q, lens_kv = [7, 0, 12], [9, 3, 12]
        tq, tkv = sum(lens_q), sum(lens_kv)
        q, qr = rand((tq, n_q, d), 41), rand((tq, n_q, dr), 42)
        k, kr = rand((tkv, n_kv, d), 43), rand((tkv, n_kv, dr), 44)
        v = rand((tkv, n_kv, dv), 45)
        kw.update(actual_seq_q=cumulative(lens_q, False), actual_seq_kv=cumulative(lens_kv, False))
        qj, kj = np.concatenate([q, qr], axis=-1), np.concatenate([k, kr], axis=-1)
    else:
        bsz, sq, skv = 2, 11, 13
        q, qr = rand((bsz, sq, n_q * d), 41), rand((bsz, sq, n_q * dr), 42)
        k, kr = rand((bsz, skv, n_kv * d), 43), rand((bsz, skv, n_kv * dr), 44)
        v = rand((bsz, skv, n_kv * dv), 45)

        def join(a, b, n):  # per head: the head's D columns, then its Dr columns
            return np.concatenate([a.reshape(bsz, -1, n, d), b.reshape(bsz, -1, n, dr)],
                                  axis=-1).reshape(bsz, -1, n * (d + dr))
        qj, kj = join(q, qr, n_q), join(k, kr, n_kv)
    with_rope = ref.forward(q, k, v, layout=layout, head_num=n_q, scale=0.3, query_rope=qr, key_rope=kr, **kw)
    joined = ref.forward(qj, kj, v, layout=layout, head_num=n_q, scale=0.3, **kw)
    for key in ("out", "softmax_max", "softmax_sum"):
        np.testing.assert_allclose(with_rope[key], joined[key], rtol=1e-12, atol=1e-14)
