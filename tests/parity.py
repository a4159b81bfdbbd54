"""Shared helpers of the GPU parity tests: run a workload through the C ABI,
run the float64 oracle on the same inputs, compare within the stated
tolerances."""
import numpy as np
import torch

import attention_forward_20_b200 as fa
from oracle import ref

# attentionOut max-abs error (fp32 accumulation): bf16 2e-2, fp16 5e-3, fp32 1e-4;
# softmaxMax / softmaxSum relative error 1e-3 (absolute below magnitude 1).
OUT_TOL = {"bf16": 2e-2, "f16": 5e-3, "f32": 1e-4}
STAT_RTOL = 1e-3


def f64(t):
    return None if t is None else t.detach().cpu().double().numpy()


def to_cuda(w):
    c = lambda t: None if t is None else t.cuda()  # noqa: E731
    return c(w.q), c(w.k), c(w.v), c(w.pse), c(w.atten_mask), c(w.sink)


def run_gpu(w, **overrides):
    q, k, v, pse, mask, sink = to_cuda(w)
    kw = dict(input_layout=w.layout, head_num=w.head_num, scale=w.scale, real_shift=pse,
              pse_type=w.pse_type if pse is not None else None, atten_mask=mask, mask_mode=w.mask_mode,
              sink=sink, actual_seq_qlen=w.actual_seq_q, actual_seq_kvlen=w.actual_seq_kv,
              pre_tokens=w.pre_tokens, next_tokens=w.next_tokens, softmax_out_layout=w.softmax_out_layout)
    kw.update(overrides)
    out, smax, ssum = fa.fa_fwd(q, k, v, **kw)
    torch.cuda.synchronize()
    return out, smax, ssum


def oracle_full(w):
    return ref.forward(f64(w.q), f64(w.k), f64(w.v), layout=w.layout, head_num=w.head_num, scale=w.scale,
                       pse=f64(w.pse), pse_type=w.pse_type, atten_mask=f64(w.atten_mask),
                       pre_tokens=w.pre_tokens, next_tokens=w.next_tokens, sink=f64(w.sink),
                       actual_seq_q=w.actual_seq_q, actual_seq_kv=w.actual_seq_kv,
                       softmax_out_layout=w.softmax_out_layout)


def check_stats(got, want, what):
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    assert got.shape == want.shape, (what, got.shape, want.shape)
    inf_w = np.isinf(want)
    assert np.array_equal(np.isinf(got) & inf_w, inf_w) and np.array_equal(got[inf_w], want[inf_w]), \
        f"{what}: infinities differ"
    fin = ~inf_w
    assert np.isfinite(got[fin]).all(), f"{what}: non-finite values"
    err = np.abs(got[fin] - want[fin]) / np.maximum(np.abs(want[fin]), 1.0)
    assert err.size == 0 or err.max() <= STAT_RTOL, f"{what}: rel err {err.max():.3e}"


def check_out(got, want, dtype, what="attentionOut"):
    got = np.asarray(got, dtype=np.float64)
    assert got.shape == want.shape, (what, got.shape, want.shape)
    assert np.isfinite(got).all(), f"{what}: non-finite values"
    err = np.abs(got - want).max() if got.size else 0.0
    assert err <= OUT_TOL[dtype], f"{what}: max-abs err {err:.3e} > {OUT_TOL[dtype]}"
    return err


def compare_full(w, res=None, **overrides):
    out, smax, ssum = res if res is not None else run_gpu(w, **overrides)
    want = oracle_full(w)
    err = check_out(f64(out), want["out"], w.dtype)
    check_stats(f64(smax), want["softmax_max"], "softmaxMax")
    check_stats(f64(ssum), want["softmax_sum"], "softmaxSum")
    return err


def sample_rows(w, count, seed=0):
    """(b, n, i) triples spread over the workload, including first and last rows."""
    rng = np.random.default_rng(seed)
    if w.layout == "TND":
        lens = np.diff([0] + list(w.actual_seq_q))
        nonempty = [b for b, L in enumerate(lens) if L > 0]
        rows = [(nonempty[0], 0, 0), (nonempty[-1], w.head_num - 1, int(lens[nonempty[-1]]) - 1)]
        while len(rows) < count:
            b = int(rng.choice(nonempty))
            rows.append((b, int(rng.integers(w.head_num)), int(rng.integers(lens[b]))))
        return rows
    sq = {"BNSD": w.q.shape[2], "BSND": w.q.shape[1], "BSH": w.q.shape[1], "SBH": w.q.shape[0]}[w.layout]
    bsz = w.q.shape[1] if w.layout == "SBH" else w.q.shape[0]
    rows = [(0, 0, 0), (bsz - 1, w.head_num - 1, sq - 1)]
    while len(rows) < count:
        rows.append((int(rng.integers(bsz)), int(rng.integers(w.head_num)), int(rng.integers(sq))))
    return rows


def gather_rows(w, out, smax, ssum, rows):
    """GPU outputs of the sampled rows: o [R, Dv], m [R], l [R]."""
    o_list, m_list, l_list = [], [], []
    out = out.float()
    n_heads = w.head_num
    for (b, n, i) in rows:
        if w.layout == "TND":
            t = ([0] + list(w.actual_seq_q))[b] + i
            o = out[t, n]
            st = (t, n) if w.softmax_out_layout == "same_as_input" else (n, t)
            m, l = smax[st][0], ssum[st][0]
        else:
            if w.layout == "BNSD":
                o = out[b, n, i]
            elif w.layout == "BSND":
                o = out[b, i, n]
            elif w.layout == "BSH":
                o = out[b, i].view(n_heads, -1)[n]
            else:
                o = out[i, b].view(n_heads, -1)[n]
            m, l = smax[b, n, i, 0], ssum[b, n, i, 0]
        o_list.append(o.double().cpu().numpy())
        m_list.append(float(m))
        l_list.append(float(l))
    return np.array(o_list), np.array(m_list), np.array(l_list)


def compare_rows(w, res, rows):
    out, smax, ssum = res
    o, m, l = gather_rows(w, out, smax, ssum, rows)
    wo, wm, wl = ref.forward_rows(f64(w.q), f64(w.k), f64(w.v), rows, layout=w.layout, head_num=w.head_num,
                                  scale=w.scale, pse=f64(w.pse), pse_type=w.pse_type,
                                  atten_mask=f64(w.atten_mask), pre_tokens=w.pre_tokens,
                                  next_tokens=w.next_tokens, sink=f64(w.sink), actual_seq_q=w.actual_seq_q,
                                  actual_seq_kv=w.actual_seq_kv)
    err = check_out(o, wo, w.dtype, "sampled attentionOut rows")
    check_stats(m, wm, "sampled softmaxMax")
    check_stats(l, wl, "sampled softmaxSum")
    return err
