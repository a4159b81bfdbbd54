"""The bench's host logic on CPU: the FLOP counts it divides by (closed forms
and brute-force tile counts), the inputs it builds for other head dims and for
rope, and the reference arm's JSON line."""
import contextlib
import io
import json

import numpy as np

import bench
from workloads import build, cumulative, Workload, normal

INT64_MAX = 2**63 - 1


def _brute_tiles(sq, skv, pre, nxt):
    """128x128 tiles holding at least one kept pair, and the kept pairs."""
    tiles = pairs = 0
    for i0 in range(0, sq, 128):
        for j0 in range(0, skv, 128):
            kept = sum(1 for i in range(i0, min(sq, i0 + 128)) for j in range(j0, min(skv, j0 + 128))
                       if -pre <= j - i <= nxt)
            tiles += 1 if kept else 0
            pairs += kept
    return tiles, pairs


def test_dense_flops_closed_form():
    w = build(2)
    tiles, exact = bench.tile_flops(w)
    assert tiles == exact == 4.0 * 128 * 4096 * 4096 * 2 * 24


def test_band_and_causal_tiles_match_brute_force():
    for sq, skv, pre, nxt in [(300, 300, INT64_MAX, 0), (333, 200, 50, 7), (257, 513, 100, -3)]:
        q = normal((1, 2, sq, 64), "f16", 1)
        k = normal((1, 2, skv, 64), "f16", 2)
        w = Workload("t", 0, "BNSD", "f16", 2, q, k, k, scale=0.125, pre_tokens=pre, next_tokens=nxt)
        tiles, exact = bench.tile_flops(w)
        bt, bp = _brute_tiles(sq, skv, min(pre, 10**6), nxt)
        assert tiles == 4.0 * 64 * bt * 128 * 128 * 2
        assert exact == 4.0 * 64 * bp * 2


def test_value_head_dim_enters_the_flops():
    w = bench.with_head_dims(build(2, seq_scale=16), 128, 64)
    d, dv = bench.head_dims(w)
    assert (d, dv) == (128, 64)
    tiles, exact = bench.tile_flops(w)
    s = 4096 // 16
    assert exact == (2.0 * 128 + 2.0 * 64) * s * s * 2 * 24


def test_with_head_dims_every_layout():
    for number in (2, 3, 4, 5):
        w0 = build(number, seq_scale=32)
        w = bench.with_head_dims(build(number, seq_scale=32), 96, 64)
        assert bench.head_dims(w) == (96, 64)
        assert abs(w.scale - 96 ** -0.5) < 1e-15
        assert w.q.shape[:-1] == w0.q.shape[:-1] and w.k.shape[:-1] == w0.k.shape[:-1]
        if w.layout in ("BSH", "SBH"):
            assert w.q.shape[-1] == w.head_num * 96
        assert w.name.endswith("_d96_dv64")
        # masks, band and sink carried over
        assert (w.pre_tokens, w.next_tokens) == (w0.pre_tokens, w0.next_tokens)


def test_rope_tensors_follow_the_layout():
    w = build(4, seq_scale=16)
    qr, kr = bench.rope_tensors(w, 64, seed=1)
    assert qr.shape == (w.q.shape[0], w.head_num, 64) and kr.shape == (w.k.shape[0], w.k.shape[1], 64)
    w = build(5, seq_scale=64)  # BSH, 16 heads of 64
    qr, kr = bench.rope_tensors(w, 32, seed=1)
    assert qr.shape == w.q.shape[:2] + (16 * 32,) and kr.shape == w.k.shape[:2] + (16 * 32,)
    assert str(qr.dtype) == "torch.bfloat16"


def test_reference_arm_line():
    args = bench.parse_args(["--workload", "1", "--steps", "2", "--warmup", "3", "--impl", "reference"])
    buf = io.StringIO()
    with contextlib.redirect_stdout(buf):
        bench.run_reference(args, rank=0)
    line = json.loads(buf.getvalue().strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["unit"] == bench.UNIT and line["metric"] == bench.METRIC
    assert line["value"] > 0 and line["higher_is_better"] is True
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["d2h_bytes_per_step"] == 0
    # the other ranks print nothing
    buf = io.StringIO()
    with contextlib.redirect_stdout(buf):
        bench.run_reference(args, rank=1)
    assert buf.getvalue() == ""


def test_varlen_flops_sum_over_sequences():
    lens = [300, 0, 129]
    t = sum(lens)
    q = normal((t, 2, 64), "bf16", 3)
    w = Workload("v", 0, "TND", "bf16", 2, q, q, q, scale=0.125, next_tokens=0,
                 actual_seq_q=cumulative(lens, False), actual_seq_kv=cumulative(lens, False))
    tiles, exact = bench.tile_flops(w)
    want_pairs = sum(n * (n + 1) // 2 for n in lens)
    assert exact == 4.0 * 64 * want_pairs * 2
    want_tiles = sum(_brute_tiles(n, n, 10**6, 0)[0] for n in lens if n)
    assert tiles == 4.0 * 64 * want_tiles * 128 * 128 * 2
    assert np.isfinite(tiles)


def test_step_stats():
    st = bench.step_stats([1.0, 2.0, 3.0, 4.0, 10.0])
    assert st["median"] == 3.0 and st["min"] == 1.0 and st["mean"] == 4.0
    assert 4.0 <= st["p90"] <= 10.0


def test_with_lengths_rebuilds_the_varlen_workload():
    w = bench.with_lengths(build(4), ["2048", "2048", "2048", "2048"])
    assert w.q.shape == (8192, 24, 128) and w.actual_seq_q == [2048, 4096, 6144, 8192]
    assert w.extra["cu_seqlens"] == [0, 2048, 4096, 6144, 8192] and w.name.endswith("_2048_2048_2048_2048")
    assert w.actual_seq_kv == w.actual_seq_q
    # the default lengths' inputs come from the same seeds
    w0 = build(4)
    assert bench.with_lengths(build(4), w0.extra["lengths"]).q.float().sum() == w0.q.float().sum()


def test_single_thread_oracle_time():
    value, secs = bench.time_oracle_single_thread(build(1))
    assert value > 0 and secs > 0
