"""Plant plausible mistakes in a copy of the oracle and check that the pins in
test_oracle.py catch each one.  The mutants are built from oracle/ref.py's
source text on the CPU; nothing here touches the real module."""
import sys
import types

import pytest

import tests.test_oracle as pins
from oracle import ref

INT64_MAX = ref.INT64_MAX

# (name, exact text in oracle/ref.py, replacement)
MUTATIONS = [
    ("band left bound exclusive", "(diff >= -pre_tokens)", "(diff > -pre_tokens)"),
    ("band right bound exclusive", "(diff <= next_tokens)", "(diff < next_tokens)"),
    ("band direction swapped", "diff = j[None, :] - i[:, None]", "diff = i[:, None] - j[None, :]"),
    ("scale dropped", "s = scale * qk", "s = qk"),
    ("rope term dropped", "qk = qk + np.asarray(q_rope[r0:r1], dtype=np.float64) @ np.asarray(k_rope, dtype=np.float64).T",
     "qk = qk"),
    ("rope term outside the scale",
     "qk = qk + np.asarray(q_rope[r0:r1], dtype=np.float64) @ np.asarray(k_rope, dtype=np.float64).T",
     "qk = qk + np.asarray(q_rope[r0:r1], dtype=np.float64) @ np.asarray(k_rope, dtype=np.float64).T / scale"),
    ("rope key rows from the query", "np.asarray(k_rope, dtype=np.float64).T", "np.asarray(q_rope, dtype=np.float64).T"),
    ("rope key head map by query head", "return qrh[b, n, :ql, :], krh[b, n_kv, :kl, :]",
     "return qrh[b, n, :ql, :], krh[b, n % krh.shape[1], :kl, :]"),
    ("scale applied to pse too", "s = s + np.asarray(pse[r0:r1], dtype=np.float64)",
     "s = s + scale * np.asarray(pse[r0:r1], dtype=np.float64)"),
    ("pse sign flipped", "s = s + np.asarray(pse[r0:r1], dtype=np.float64)",
     "s = s - np.asarray(pse[r0:r1], dtype=np.float64)"),
    ("sink left out of the max", "mi = np.maximum(mi, float(sink))", "mi = mi"),
    ("sink left out of the denominator", "li = li + np.exp(float(sink) - shift)", "li = li"),
    ("sink scaled like a score", "mi = np.maximum(mi, float(sink))", "mi = np.maximum(mi, scale * float(sink))"),
    ("no normalisation", "o[r0:r1] = (p @ v) / safe_l[:, None]", "o[r0:r1] = (p @ v)"),
    ("mask polarity inverted", "keep &= ~np.asarray(excluded[r0:r1], dtype=bool)",
     "keep &= np.asarray(excluded[r0:r1], dtype=bool)"),
    ("ALiBi sign flipped", "return -slope * np.abs(", "return slope * np.abs("),
    ("ALiBi [B, N] slopes indexed [n, b]", "slope = pse[b, n] if pse.ndim == 2 else pse[n]",
     "slope = pse[n, b] if pse.ndim == 2 else pse[n]"),
    ("ALiBi [B, N] slopes ignore the batch row", "slope = pse[b, n] if pse.ndim == 2 else pse[n]",
     "slope = pse[0, n] if pse.ndim == 2 else pse[n]"),
    ("ALiBi without abs", "np.abs(np.asarray(rows, dtype=np.float64)[:, None] - j[None, :])",
     "(np.asarray(rows, dtype=np.float64)[:, None] - j[None, :])"),
    ("BSH split order", "x.reshape(b, s, h // head_dim, head_dim).transpose(0, 2, 1, 3)",
     "x.reshape(b, s, head_dim, h // head_dim).transpose(0, 3, 1, 2)"),
    ("SBH axes swapped", "x.reshape(s, b, h // head_dim, head_dim).transpose(1, 2, 0, 3)",
     "x.reshape(s, b, h // head_dim, head_dim).transpose(0, 2, 1, 3)"),
    ("TND stats not transposed", "smax, ssum = smax.T, ssum.T  # [N, T]", "pass"),
    ("GQA head map modulo", "qs, ks, vs = _head_inputs(layout, qh, kh, vh, b, n, n // group, seq)",
     "qs, ks, vs = _head_inputs(layout, qh, kh, vh, b, n, n % n_kv, seq)"),
    ("query row index off by one", "rows = np.arange(q_len)", "rows = np.arange(1, q_len + 1)"),
    ("stats in log2 units", "m[r0:r1] = mi", "m[r0:r1] = mi / np.log(2.0)"),
    ("compressed bias row shift off by one", "out[k, :kv_len - shift] = pse[bb, nn, 0, shift:kv_len]",
     "out[k, :kv_len - shift - 1] = pse[bb, nn, 0, shift + 1:kv_len]"),
    ("compressed bias read from the first full rows", "out[k] = pse[bb, nn, i - first, :kv_len]",
     "out[k] = pse[bb, nn, min(i, 1023), :kv_len]"),
    ("flat bias sequence offset skips the heads", "off = sum(n_heads * s[1] * s[3] for s in seqs[:b])",
     "off = sum(s[1] * s[3] for s in seqs[:b])"),
    ("global position shift with the wrong sign", "diff = j[None, :] - i[:, None] + delta",
     "diff = j[None, :] - i[:, None] - delta"),
    ("ALiBi ignores the global positions", "j = np.arange(kv_len, dtype=np.float64) + delta",
     "j = np.arange(kv_len, dtype=np.float64)"),
    ("merge weights without the partial sums", "w = np.where(l_k > 0, l_k * np.exp(", "w = np.where(l_k > 0, 1.0 * np.exp("),
]


def _mutant(src, old, new, tag):
    assert src.count(old) >= 1, f"mutation target not found: {old!r}"
    mod = types.ModuleType(f"oracle_mutant_{tag}")
    exec(compile(src.replace(old, new), f"<mutant {tag}>", "exec"), mod.__dict__)
    return mod


def _run_pins():
    """Every pin of test_oracle.py, with fixed arguments; raises on the first failure."""
    pins.test_worked_example_sink_closed_form()
    pins.test_worked_example_with_rope_closed_form()
    for args in [(False, INT64_MAX, INT64_MAX), (True, 2, 0)]:
        pins.test_rope_matches_brute(*args)
    for layout in ("BSH", "TND"):
        pins.test_rope_equals_joined_head_dim(layout)
    for args in [(37, 53, 16, 16, INT64_MAX, INT64_MAX), (64, 64, 32, 24, 10, 0), (50, 70, 8, 8, 5, 30)]:
        pins.test_head_matches_sdpa(*args)
    pins.test_sink_matches_sdpa_with_extra_key()
    for args in [(False, False, False, INT64_MAX, INT64_MAX), (True, False, False, INT64_MAX, 0),
                 (True, True, True, 2, 1), (False, True, False, 1, -1)]:
        pins.test_ref_matches_brute(*args)
    pins.test_constant_value_returns_constant()
    pins.test_constant_value_with_sink()
    pins.test_causal_first_row_is_v0()
    for args in [(40, 40, INT64_MAX, 0), (40, 40, 7, 0), (33, 50, 4, 9), (50, 20, 0, 0), (25, 25, 3, -2)]:
        pins.test_zero_query_band_counts(*args)
    pins.test_alibi_geometric_series()
    for layout in ("BSND", "TND"):
        pins.test_alibi_geometric_series_per_batch_slopes(layout)
    pins.test_alibi_symmetric_band()
    pins.test_empty_rows()
    pins.test_identity_value_exposes_probability_rows()
    pins.test_layouts_agree()
    pins.test_varlen_equals_each_sequence_alone()
    pins.test_gqa_equals_repeated_kv_heads()
    pins.test_mask_tensor_broadcast_forms_agree()
    for nxt in (0, -3):
        pins.test_compressed_alibi_bias_equals_slopes(nxt)
    pins.test_compressed_bias_rows_are_read_along_the_diagonal()
    pins.test_tnd_flat_bias_equals_each_sequence_with_its_own_bias()
    for kw in (dict(pre_tokens=90, next_tokens=0), dict(pre_tokens=40, next_tokens=25),
               dict(next_tokens=0, pse_type=2)):
        pins.test_key_chunks_at_their_start_merge_to_the_whole(kw)
    pins.test_query_chunk_at_its_start_equals_rows_of_the_whole()
    pins.test_merge_of_empty_parts()


def _with_ref(mod):
    saved = pins.ref
    pins.ref = mod
    try:
        _run_pins()
        return True
    except (AssertionError, ValueError, IndexError, FloatingPointError):
        return False
    finally:
        pins.ref = saved


def test_unmutated_copy_passes_every_pin():
    src = open(ref.__file__).read()
    assert _with_ref(_mutant(src, "ROW_BLOCK = 512", "ROW_BLOCK = 512", "identity"))


@pytest.mark.parametrize("name,old,new", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_pins_catch_planted_mistake(name, old, new):
    src = open(ref.__file__).read()
    tag = "".join(c if c.isalnum() else "_" for c in name)
    mutant = _mutant(src, old, new, tag)
    assert not _with_ref(mutant), f"no pin caught: {name}"
    sys.modules.pop(mutant.__name__, None)
