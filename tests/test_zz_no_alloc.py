"""fa_fwd_varlen_static, the varlen forward that allocates nothing.

Some callers cannot allocate device memory (code that runs while a stream is
captured, or a runtime that owns all device memory up front), so they cannot
hand the ordinary varlen call its workspace.  This entry point keeps that
scratch in a fixed device array of the library.  These tests call it through
the C ABI and check every output element against the float64 oracle, and
against the ordinary two-stage call on the same inputs, within the parity
tolerances, over consecutive calls that rewrite the shared scratch.  The file
is named to be collected last."""
import ctypes

import pytest
import torch

import attention_forward_20_b200 as fa
from attention_forward_20_b200 import _abi
from attention_forward_20_b200.static_scratch import fa_fwd_varlen_static, _lib
from oracle import ref
from workloads import normal, cumulative
from tests.parity import OUT_TOL, check_out, check_stats

pytestmark = pytest.mark.gpu

MAX_SEQS = 2048  # the entry point's documented limit


@pytest.fixture(scope="module", autouse=True)
def built():
    from attention_forward_20_b200 import build
    build.build()
    _lib()


def case(dtype, d, lens_q, lens_kv, heads, seed, kv_heads=None, dv=None, **kw):
    tq, tk = sum(lens_q), sum(lens_kv)
    kv_heads = kv_heads or heads
    q = normal((tq, heads, d), dtype, seed)
    k = normal((tk, kv_heads, d), dtype, seed + 1)
    v = normal((tk, kv_heads, dv or d), dtype, seed + 2)
    return dict(q=q, k=k, v=v, cq=cumulative(lens_q, False), ck=cumulative(lens_kv, False), heads=heads,
                dtype=dtype, **kw)


def run_static(c):
    """The allocation-free call into fresh output tensors."""
    q, k, v = c["q"].cuda(), c["k"].cuda(), c["v"].cuda()
    sink = c.get("sink")
    sink = sink.cuda() if sink is not None else None
    sol = c.get("sol", "")
    tq, heads, dv = q.shape[0], c["heads"], v.shape[-1]
    out = torch.empty(tq, heads, dv, dtype=q.dtype, device="cuda")
    stats_shape = (tq, heads, 8) if sol == "same_as_input" else (heads, tq, 8)
    smax = torch.empty(stats_shape, dtype=torch.float32, device="cuda")
    ssum = torch.empty(stats_shape, dtype=torch.float32, device="cuda")
    fa_fwd_varlen_static(q, k, v, c["cq"], c["ck"], out, smax, ssum, head_num=heads, sink=sink,
                         softmax_out_layout=sol, pre_tokens=c.get("pre", fa.INT64_MAX),
                         next_tokens=c.get("next", fa.INT64_MAX))
    torch.cuda.synchronize()
    return out, smax, ssum


def run_workspace_call(c):
    """The ordinary two-stage call (caller-allocated workspace) on the same inputs."""
    sink = c.get("sink")
    res = fa.fa_fwd(c["q"].cuda(), c["k"].cuda(), c["v"].cuda(), input_layout="TND", head_num=c["heads"],
                    sink=None if sink is None else sink.cuda(), actual_seq_qlen=c["cq"], actual_seq_kvlen=c["ck"],
                    softmax_out_layout=c.get("sol", ""), pre_tokens=c.get("pre", fa.INT64_MAX),
                    next_tokens=c.get("next", fa.INT64_MAX))
    torch.cuda.synchronize()
    return res


def oracle(c):
    f = lambda t: None if t is None else t.double().numpy()  # noqa: E731
    d = c["q"].shape[-1]
    return ref.forward(f(c["q"]), f(c["k"]), f(c["v"]), layout="TND", head_num=c["heads"], scale=d ** -0.5,
                       sink=f(c.get("sink")), actual_seq_q=c["cq"], actual_seq_kv=c["ck"],
                       pre_tokens=c.get("pre", ref.INT64_MAX), next_tokens=c.get("next", ref.INT64_MAX),
                       softmax_out_layout=c.get("sol", ""))


def check_against_oracle(c, got):
    want = oracle(c)
    check_out(got[0].double().cpu().numpy(), want["out"], c["dtype"])
    check_stats(got[1].double().cpu().numpy(), want["softmax_max"], "softmaxMax")
    check_stats(got[2].double().cpu().numpy(), want["softmax_sum"], "softmaxSum")


def check_against_workspace_call(c, got):
    want = run_workspace_call(c)
    err = (got[0].double() - want[0].double()).abs().max().item() if got[0].numel() else 0.0
    assert err <= OUT_TOL[c["dtype"]], err
    check_stats(got[1].double().cpu().numpy(), want[1].double().cpu().numpy(), "softmaxMax")
    check_stats(got[2].double().cpu().numpy(), want[2].double().cpu().numpy(), "softmaxSum")


CASES = {
    # ragged lengths with an empty sequence, causal, per-head sink (two-tile tensor-core kernel)
    "bf16_d128_causal_sink": lambda: case("bf16", 128, [300, 0, 129, 513], [300, 0, 129, 513], 3, 31, next=0,
                                          sink=normal((3,), "f32", 35)),
    # query and key lengths differ, two-sided band, [T, N, 8] statistics
    "f16_d64_band_same_as_input": lambda: case("f16", 64, [1000, 77, 5], [900, 200, 5], 2, 41, pre=100,
                                               next=10, sol="same_as_input"),
    # GQA (4 query heads over 2 key/value heads)
    "bf16_d128_gqa": lambda: case("bf16", 128, [257, 40, 130], [257, 40, 130], 4, 61, kv_heads=2, next=0),
    # head dims above 128 (one-tile tensor-core kernel), Dv < D, an empty sequence
    "bf16_d256_dv136": lambda: case("bf16", 256, [200, 0, 300], [200, 0, 300], 2, 71, dv=136, next=0),
    # fp32: the CUDA-core kernel
    "f32_d64_causal": lambda: case("f32", 64, [70, 33], [70, 33], 2, 51, next=0),
}


@pytest.mark.parametrize("name", list(CASES))
def test_static_scratch_matches_oracle(name):
    c = CASES[name]()
    check_against_oracle(c, run_static(c))


def test_static_scratch_matches_oracle_and_workspace_call_on_consecutive_calls():
    """A, B, A: each call rewrites the shared scratch; every result matches
    the oracle and the ordinary call, and the two A calls agree bit for bit."""
    a = CASES["bf16_d128_causal_sink"]()
    b = CASES["f16_d64_band_same_as_input"]()
    results = [run_static(a), run_static(b), run_static(a)]
    for c, got in zip([a, b, a], results):
        check_against_oracle(c, got)
        check_against_workspace_call(c, got)
    for x, y in zip(results[0], results[2]):
        assert torch.equal(x, y)


def test_static_scratch_at_the_sequence_limit():
    """Exactly the documented maximum of sequences (short ones, so the
    offsets and the table both reach their largest extent for that count)."""
    lens = [1 + (i % 3) for i in range(MAX_SEQS)]
    c = case("bf16", 64, lens, lens, 1, 81, next=0, sink=normal((1,), "f32", 85))
    got = run_static(c)
    check_against_oracle(c, got)
    check_against_workspace_call(c, got)
    # a shorter call right after: it rewrites only the front of the scratch
    c2 = case("bf16", 64, [5, 300], [5, 300], 1, 91, next=0)
    check_against_oracle(c2, run_static(c2))


def test_static_scratch_rejects_too_many_sequences():
    lib = _lib()
    t = torch.zeros(4096, 1, 64, dtype=torch.float16)
    ft = fa._ft(t)
    st = fa._ft(torch.zeros(1, 4096, 8))
    n = MAX_SEQS + 1
    cum = (ctypes.c_int64 * n)(*[min(i + 1, 4096) for i in range(n)])
    r = ctypes.byref
    status = lib.fa_fwd_varlen_static(r(ft), r(ft), r(ft), None, cum, cum, n, 0.125, fa.INT64_MAX, fa.INT64_MAX,
                                      1, b"", r(st), r(st), r(ft), None)
    assert status == fa.FA_ERR_INNER_NULLPTR
    assert _abi.status_string(status).startswith("FA_ERR_INNER_NULLPTR")
