"""Pure-Python, loop-by-loop twin of the oracle for tiny shapes.

TEST INFRASTRUCTURE ONLY (same import rule as oracle/ref.py).

It types out the sink formula of the aclnnFlashAttentionVarLenScoreV5 page
("计算公式", after "增加sink之后"): m = max(sink, max(S)) and
Attention = e^{S-m} V / (sum e^{S-m} + e^{sink-m}), with S the scaled,
biased, masked score of one query row.  Scalars only: Python floats, math.exp
and math.fsum, no NumPy, so that it shares no arithmetic routine with ref.py.
"""
import math

INT64_MAX = 2**63 - 1


def head_forward(q, k, v, scale, pse=None, excluded=None,
                 pre_tokens=INT64_MAX, next_tokens=INT64_MAX, sink=None, q_rope=None, k_rope=None):
    """q: Sq lists of D floats; k: Skv lists of D; v: Skv lists of Dv.

    pse: Sq lists of Skv floats or None; excluded: Sq lists of Skv bools or
    None; q_rope / k_rope: Sq / Skv lists of Dr floats or None (the page's
    forward formula scales queryRope keyRope^T together with query key^T).
    Returns (o, m, l) as nested Python lists / floats.
    """
    sq, skv, dv = len(q), len(k), (len(v[0]) if v else 0)
    outs, maxes, sums = [], [], []
    for i in range(sq):
        scores = []  # (S_ij, j) for the keys row i attends to
        for j in range(skv):
            if j - i < -pre_tokens or j - i > next_tokens:
                continue
            if excluded is not None and excluded[i][j]:
                continue
            terms = [q[i][d] * k[j][d] for d in range(len(q[i]))]
            if q_rope is not None:
                terms += [q_rope[i][e] * k_rope[j][e] for e in range(len(q_rope[i]))]
            dot = math.fsum(terms)
            s = scale * dot + (pse[i][j] if pse is not None else 0.0)
            scores.append((s, j))
        candidates = [s for s, _ in scores] + ([sink] if sink is not None else [])
        if not candidates:
            outs.append([0.0] * dv)
            maxes.append(-math.inf)
            sums.append(0.0)
            continue
        m = max(candidates)
        weights = [(math.exp(s - m), j) for s, j in scores]
        denom = math.fsum(w for w, _ in weights) + (math.exp(sink - m) if sink is not None else 0.0)
        row = [math.fsum(w * v[j][d] for w, j in weights) / denom for d in range(dv)]
        outs.append(row)
        maxes.append(m)
        sums.append(denom)
    return outs, maxes, sums
