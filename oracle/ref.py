"""Float64 CPU oracle for the FlashAttention self-attention forward.

TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and bench.py's
cpu_baseline / reference leg may import this module.  It shares no code with
the CUDA path and imports nothing from it.

What it computes is the plain definition that the FlashAttention operator
pages describe and that the tiled kernel reaches up to rounding order
(aclnnFlashAttentionVarLenScoreV5, "计算公式" — the forward formula and the
sink formula; aclnnFlashAttentionScore, parameter list for attenMask,
scaleValue, preTockens/nextTockens, softmaxMax/softmaxSum):

    s_ij    = scale * (sum_d q_id k_jd + sum_e qr_ie kr_je) + pse_ij
              (pse_ij = 0 without pse; the rope term only with queryRope/keyRope)
    keep_ij = (-preTokens <= j - i <= nextTokens) and not attenMask_ij
    m_i     = max({s_ij : keep_ij} U {sink_n if a sink is given})
    l_i     = sum_{keep} exp(s_ij - m_i) + [sink] exp(sink_n - m_i)
    o_i     = sum_{keep} exp(s_ij - m_i) v_j / l_i

Readings where the pages are silent:
  * pse is added after scaling, as the printed formula writes it;
  * the sink formula's S is this full transformed, masked score; the sink
    itself is neither scaled nor masked;
  * masked positions are excluded exactly (weight 0), not given a large
    finite negative value;
  * the band is inclusive and top-left aligned within each sequence (i and j
    both count from 0 in the sequence);
  * a row with nothing kept and no sink gives o = 0, m = -inf, l = 0; with a
    sink it gives o = 0, m = sink, l = 1;
  * softmaxMax / softmaxSum are m_i (natural-log units) and l_i, written to
    all 8 lanes of the trailing axis;
  * ALiBi slopes (pse type 2) give pse_ij = -slope_n * |i - j|;
  * queryRope / keyRope (aclnnFlashAttentionVarLenScoreV5 formula,
    scale*(query key^T + queryRope keyRope^T)) add a second dot product over
    their own head dim inside the scaling.

Inputs are taken exactly as the kernel sees them: arrays already rounded to
their storage dtype, then widened to float64 here.
"""
import numpy as np

INT64_MAX = 2**63 - 1
ROW_BLOCK = 512

LAYOUTS = ("BSH", "SBH", "BSND", "BNSD", "TND")


# ---------------------------------------------------------------------------
# Layouts (aclnnFlashAttentionScore, inputLayout: BSH, SBH, BSND, BNSD with
# H = N*D; aclnnFlashAttentionVarLenScoreV5, TND with T the packed B*S axis).
# ---------------------------------------------------------------------------

def heads_view(x, layout, head_dim):
    """Logical [B, N, S, D] view of a dense-layout tensor, or [T, N, D] for TND."""
    x = np.asarray(x, dtype=np.float64)
    if layout == "BNSD":
        return x
    if layout == "BSND":
        return x.transpose(0, 2, 1, 3)
    if layout == "BSH":
        b, s, h = x.shape
        return x.reshape(b, s, h // head_dim, head_dim).transpose(0, 2, 1, 3)
    if layout == "SBH":
        s, b, h = x.shape
        return x.reshape(s, b, h // head_dim, head_dim).transpose(1, 2, 0, 3)
    if layout == "TND":
        return x
    raise ValueError(f"unknown layout {layout}")


def from_heads(o, layout):
    """Inverse of heads_view for the output: [B, N, S, Dv] (or [T, N, Dv]) to `layout`."""
    if layout in ("BNSD", "TND"):
        return o
    if layout == "BSND":
        return o.transpose(0, 2, 1, 3)
    if layout == "BSH":
        b, n, s, d = o.shape
        return o.transpose(0, 2, 1, 3).reshape(b, s, n * d)
    if layout == "SBH":
        b, n, s, d = o.shape
        return o.transpose(2, 0, 1, 3).reshape(s, b, n * d)
    raise ValueError(f"unknown layout {layout}")


# ---------------------------------------------------------------------------
# One (batch, head): the definition above, row block by row block.
# ---------------------------------------------------------------------------

def head_forward(q, k, v, scale, rows=None, pse=None, excluded=None,
                 pre_tokens=INT64_MAX, next_tokens=INT64_MAX, sink=None, delta=0,
                 q_rope=None, k_rope=None):
    """Attention of one (batch, head).

    q: [R, D] query rows whose in-sequence indices are `rows` (default 0..R-1);
    k: [Skv, D]; v: [Skv, Dv]; pse: [R, Skv] additive bias or None;
    excluded: bool [R, Skv] (True = does not take part) or None;
    sink: float or None; delta: kvStartIdx - qStartIdx, the band compares the
    global positions (kvStart + j) - (qStart + i) = j - i + delta;
    q_rope [R, Dr], k_rope [Skv, Dr]: the rope parts of query and key, or None.
    Returns o [R, Dv], m [R], l [R] in float64.
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    n_rows, skv = q.shape[0], k.shape[0]
    if rows is None:
        rows = np.arange(n_rows, dtype=np.int64)
    rows = np.asarray(rows, dtype=np.int64)
    o = np.zeros((n_rows, v.shape[1]))
    m = np.full(n_rows, -np.inf)
    l = np.zeros(n_rows)
    j = np.arange(skv, dtype=np.int64)
    for r0 in range(0, n_rows, ROW_BLOCK):
        r1 = min(n_rows, r0 + ROW_BLOCK)
        i = rows[r0:r1]
        qk = q[r0:r1] @ k.T
        if q_rope is not None:
            qk = qk + np.asarray(q_rope[r0:r1], dtype=np.float64) @ np.asarray(k_rope, dtype=np.float64).T
        s = scale * qk
        if pse is not None:
            s = s + np.asarray(pse[r0:r1], dtype=np.float64)
        diff = j[None, :] - i[:, None] + delta
        keep = (diff >= -pre_tokens) & (diff <= next_tokens)
        if excluded is not None:
            keep &= ~np.asarray(excluded[r0:r1], dtype=bool)
        s_kept = np.where(keep, s, -np.inf)
        mi = s_kept.max(axis=1) if skv > 0 else np.full(r1 - r0, -np.inf)
        if sink is not None:
            mi = np.maximum(mi, float(sink))
        finite = np.isfinite(mi)
        shift = np.where(finite, mi, 0.0)
        p = np.where(keep, np.exp(s_kept - shift[:, None]), 0.0)
        li = p.sum(axis=1)
        if sink is not None:
            li = li + np.exp(float(sink) - shift)
        safe_l = np.where(li > 0, li, 1.0)
        o[r0:r1] = (p @ v) / safe_l[:, None]
        m[r0:r1] = mi
        l[r0:r1] = li
    return o, m, l


# ---------------------------------------------------------------------------
# Whole call: layouts, varlen (actualSeqQLen / actualSeqKvLen cumulative
# without a leading 0), GQA head mapping, pse, attenMask broadcast, sink,
# statistics layouts.
# ---------------------------------------------------------------------------

def _sequences(layout, qh, kh, actual_seq_q, actual_seq_kv):
    """List of (q_start, q_len, kv_start, kv_len) per batch."""
    if layout == "TND":
        cq = [0] + [int(x) for x in actual_seq_q]
        ck = [0] + [int(x) for x in actual_seq_kv]
        return [(cq[b], cq[b + 1] - cq[b], ck[b], ck[b + 1] - ck[b]) for b in range(len(cq) - 1)]
    b = qh.shape[0]
    return [(0, qh.shape[2], 0, kh.shape[2]) for _ in range(b)]


def _head_inputs(layout, qh, kh, vh, b, n, n_kv, seq):
    q0, ql, k0, kl = seq
    if layout == "TND":
        return qh[q0:q0 + ql, n, :], kh[k0:k0 + kl, n_kv, :], vh[k0:k0 + kl, n_kv, :]
    return qh[b, n, :ql, :], kh[b, n_kv, :kl, :], vh[b, n_kv, :kl, :]


def _rope_views(query_rope, key_rope, layout, head_num):
    """Logical views of queryRope / keyRope (the query's / key's layout, own head dim), or Nones."""
    if query_rope is None and key_rope is None:
        return None, None
    if query_rope is None or key_rope is None:
        raise ValueError("queryRope and keyRope go together")
    dr = _head_dim(query_rope, layout, head_num)
    return heads_view(query_rope, layout, dr), heads_view(key_rope, layout, dr)


def _rope_inputs(layout, qrh, krh, b, n, n_kv, seq):
    if qrh is None:
        return None, None
    q0, ql, k0, kl = seq
    if layout == "TND":
        return qrh[q0:q0 + ql, n, :], krh[k0:k0 + kl, n_kv, :]
    return qrh[b, n, :ql, :], krh[b, n_kv, :kl, :]


def _pse_rows(pse, pse_type, b, n, rows, kv_len, seqs=None, n_heads=None, delta=0):
    """Additive bias rows [len(rows), kv_len] for (b, n), or None.

    Dense bias layouts (aclnnFlashAttentionVarLenScoreV5, realShiftOptional
    and its notes on alibi compression and TND):
      [B or 1, N or 1, Sq, Skv]  the bias itself;
      [B or 1, N or 1, 1024, Skv] with Sq > 1024 (the compressed form): the last
          1024 rows of the full bias, alibi_compress = pse[:, :, -1024:, :].  A
          row i above them is read along its diagonal from the first stored
          row: bias[i][j] = stored[0][j + (Sq - 1024 - i)] (reading: for a bias
          that depends on i - j only this is the full bias; columns past the
          stored row, which the lower-triangular mask excludes, read 0);
      [sum_b N * Sq_b * Skv_b] (TND): sequence b's [N, Sq_b, Skv_b] block,
          flattened, after the blocks of sequences 0 .. b-1.
    """
    if pse is None or pse_type in (0, None):
        return None
    pse = np.asarray(pse, dtype=np.float64)
    rows = np.asarray(rows)
    if pse_type == 1 and pse.ndim == 1:
        off = sum(n_heads * s[1] * s[3] for s in seqs[:b])
        q_len = seqs[b][1]
        block = pse[off:off + n_heads * q_len * kv_len].reshape(n_heads, q_len, kv_len)
        return block[n][rows]
    if pse_type == 1:  # dense tensor [B or 1, N or 1, Sq or 1024, Skv]
        bb = b if pse.shape[0] > 1 else 0
        nn = n if pse.shape[1] > 1 else 0
        q_len = seqs[b][1] if seqs is not None else pse.shape[2]
        if pse.shape[2] == 1024 and q_len > 1024:
            first = q_len - 1024
            out = np.zeros((len(rows), kv_len))
            for k, i in enumerate(rows):
                if i >= first:
                    out[k] = pse[bb, nn, i - first, :kv_len]
                else:
                    shift = first - i
                    out[k, :kv_len - shift] = pse[bb, nn, 0, shift:kv_len]
            return out
        return pse[bb, nn][rows][:, :kv_len]
    if pse_type == 2:  # slopes [N] or [B, N]: pse_ij = -slope * |i - j| at global positions
        slope = pse[b, n] if pse.ndim == 2 else pse[n]
        j = np.arange(kv_len, dtype=np.float64) + delta
        return -slope * np.abs(np.asarray(rows, dtype=np.float64)[:, None] - j[None, :])
    raise ValueError(f"unknown pse_type {pse_type}")


def _mask_rows(mask, b, n, rows, kv_len):
    """Excluded-flag rows [len(rows), kv_len] for (b, n), or None."""
    if mask is None:
        return None
    mk = np.asarray(mask) != 0
    if mk.ndim == 2:
        return mk[rows][:, :kv_len]
    bb = b if mk.shape[0] > 1 else 0
    nn = n if mk.shape[1] > 1 else 0
    return mk[bb, nn][rows][:, :kv_len]


def _deltas(q_start, kv_start, n_seqs):
    """kvStartIdx - qStartIdx per sequence (each None, one value or one per sequence)."""
    def at(x, b):
        if x is None:
            return 0
        x = np.atleast_1d(np.asarray(x, dtype=np.int64))
        return int(x[0] if x.size == 1 else x[b])
    return [at(kv_start, b) - at(q_start, b) for b in range(n_seqs)]


def forward(query, key, value, *, layout, head_num, scale, pse=None, pse_type=None,
            atten_mask=None, pre_tokens=INT64_MAX, next_tokens=INT64_MAX, sink=None,
            actual_seq_q=None, actual_seq_kv=None, softmax_out_layout="", q_start=None, kv_start=None,
            query_rope=None, key_rope=None):
    """Full forward.  Returns dict(out, softmax_max, softmax_sum) in float64.

    out has the query layout (value head dim); the statistics are
    [B, N, Sq, 8] for BSH/SBH/BSND/BNSD, and for TND [N, T, 8]
    (softmax_out_layout "") or [T, N, 8] ("same_as_input").
    """
    head_dim = _head_dim(query, layout, head_num)
    qh = heads_view(query, layout, head_dim)
    kh = heads_view(key, layout, head_dim)
    vh = heads_view(value, layout, _value_head_dim(value, key, layout, head_dim))
    qrh, krh = _rope_views(query_rope, key_rope, layout, head_num)
    n_q = head_num
    n_kv = kh.shape[1]
    group = n_q // n_kv
    seqs = _sequences(layout, qh, kh, actual_seq_q, actual_seq_kv)
    deltas = _deltas(q_start, kv_start, len(seqs))
    dv = vh.shape[-1]
    sink_arr = None if sink is None else np.asarray(sink, dtype=np.float64)
    if layout == "TND":
        t = qh.shape[0]
        out = np.zeros((t, n_q, dv))
        smax = np.zeros((t, n_q))
        ssum = np.zeros((t, n_q))
    else:
        bsz, _, sq, _ = qh.shape
        out = np.zeros((bsz, n_q, sq, dv))
        smax = np.zeros((bsz, n_q, sq))
        ssum = np.zeros((bsz, n_q, sq))
    for b, seq in enumerate(seqs):
        q_len, kv_len = seq[1], seq[3]
        if q_len == 0:
            continue
        rows = np.arange(q_len)
        for n in range(n_q):
            qs, ks, vs = _head_inputs(layout, qh, kh, vh, b, n, n // group, seq)
            qr, kr = _rope_inputs(layout, qrh, krh, b, n, n // group, seq)
            o, m, l = head_forward(
                qs, ks, vs, scale, rows=rows, q_rope=qr, k_rope=kr,
                pse=_pse_rows(pse, pse_type, b, n, rows, kv_len, seqs, n_q, deltas[b]),
                excluded=_mask_rows(atten_mask, b, n, rows, kv_len),
                pre_tokens=pre_tokens, next_tokens=next_tokens,
                sink=None if sink_arr is None else sink_arr[n], delta=deltas[b])
            if layout == "TND":
                out[seq[0]:seq[0] + q_len, n] = o
                smax[seq[0]:seq[0] + q_len, n] = m
                ssum[seq[0]:seq[0] + q_len, n] = l
            else:
                out[b, n, :q_len] = o
                smax[b, n, :q_len] = m
                ssum[b, n, :q_len] = l
    if layout == "TND" and softmax_out_layout != "same_as_input":
        smax, ssum = smax.T, ssum.T  # [N, T]
    return {
        "out": from_heads(out, layout),
        "softmax_max": np.repeat(smax[..., None], 8, axis=-1),
        "softmax_sum": np.repeat(ssum[..., None], 8, axis=-1),
    }


def forward_rows(query, key, value, rows, *, layout, head_num, scale, pse=None, pse_type=None,
                 atten_mask=None, pre_tokens=INT64_MAX, next_tokens=INT64_MAX, sink=None,
                 actual_seq_q=None, actual_seq_kv=None, q_start=None, kv_start=None,
                 query_rope=None, key_rope=None):
    """Selected output rows only: `rows` is a list of (b, n, i), i the in-sequence index.

    Returns o [R, Dv], m [R], l [R]; used to check full-size runs row by row.
    """
    head_dim = _head_dim(query, layout, head_num)
    qh = heads_view(query, layout, head_dim)
    kh = heads_view(key, layout, head_dim)
    vh = heads_view(value, layout, _value_head_dim(value, key, layout, head_dim))
    qrh, krh = _rope_views(query_rope, key_rope, layout, head_num)
    group = head_num // kh.shape[1]
    seqs = _sequences(layout, qh, kh, actual_seq_q, actual_seq_kv)
    deltas = _deltas(q_start, kv_start, len(seqs))
    sink_arr = None if sink is None else np.asarray(sink, dtype=np.float64)
    outs, ms, ls = [], [], []
    for (b, n, i) in rows:
        seq = seqs[b]
        qs, ks, vs = _head_inputs(layout, qh, kh, vh, b, n, n // group, seq)
        qr, kr = _rope_inputs(layout, qrh, krh, b, n, n // group, seq)
        r = np.array([i])
        o, m, l = head_forward(
            qs[i:i + 1], ks, vs, scale, rows=r,
            q_rope=None if qr is None else qr[i:i + 1], k_rope=kr,
            pse=_pse_rows(pse, pse_type, b, n, r, seq[3], seqs, head_num, deltas[b]),
            excluded=_mask_rows(atten_mask, b, n, r, seq[3]),
            pre_tokens=pre_tokens, next_tokens=next_tokens,
            sink=None if sink_arr is None else sink_arr[n], delta=deltas[b])
        outs.append(o[0])
        ms.append(m[0])
        ls.append(l[0])
    return np.array(outs), np.array(ms), np.array(ls)


def merge(outs, maxes, sums, sink=None):
    """Result over the union of disjoint key sets from per-set results.

    outs[k] [..., Dv], maxes[k] / sums[k] [...]: normalised output, row max
    and row sum (natural log units) of the same rows over key set k, without
    a sink.  The forward formula over the union regroups its sums by set:
    with M the largest max over sets holding a key (and the sink),
      l = sum_k sums_k e^(maxes_k - M) + e^(sink - M),
      o = sum_k sums_k e^(maxes_k - M) outs_k / l;
    rows with no key and no sink give o = 0, m = -inf, l = 0.
    `sink` broadcasts against the rows (e.g. shape [N, 1] for [N, T] rows).
    """
    ms = [np.asarray(x, dtype=np.float64) for x in maxes]
    ls = [np.asarray(x, dtype=np.float64) for x in sums]
    os_ = [np.asarray(x, dtype=np.float64) for x in outs]
    big = np.full(ms[0].shape, -np.inf)
    for m_k, l_k in zip(ms, ls):
        big = np.maximum(big, np.where(l_k > 0, m_k, -np.inf))
    if sink is not None:
        big = np.maximum(big, np.asarray(sink, dtype=np.float64))
    shift = np.where(np.isfinite(big), big, 0.0)
    l = np.zeros(big.shape)
    o = np.zeros(os_[0].shape)
    for o_k, m_k, l_k in zip(os_, ms, ls):
        w = np.where(l_k > 0, l_k * np.exp(np.where(l_k > 0, m_k, 0.0) - shift), 0.0)
        l = l + w
        o = o + w[..., None] * o_k
    if sink is not None:
        l = l + np.exp(np.asarray(sink, dtype=np.float64) - shift)
    safe = np.where(l > 0, l, 1.0)
    o = np.where((l > 0)[..., None], o / safe[..., None], 0.0)
    m = np.where(l > 0, big, -np.inf)
    return o, m, l


def _head_dim(query, layout, head_num):
    shape = np.shape(query)
    if layout in ("BSH", "SBH"):
        return shape[2] // head_num
    return shape[-1]


def _value_head_dim(value, key, layout, head_dim):
    if layout not in ("BSH", "SBH"):
        return np.shape(value)[-1]
    # with H = N * D, value's H over key's head count gives the value head dim
    n_kv = np.shape(key)[2] // head_dim
    return np.shape(value)[2] // n_kv
