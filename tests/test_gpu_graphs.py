"""The forward captured into a CUDA graph and replayed: the per-call tables
(varlen offsets and work table, the split schedule's ticket counter) must live
in the graph, not in host memory that the call frees.  Replays with new inputs
written into the captured buffers equal eager calls bit for bit (the kernels
are deterministic)."""
import pytest
import torch

import attention_forward_20_b200 as fa
from workloads import normal, cumulative

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def built():
    from attention_forward_20_b200 import build
    build.build()
    assert torch.cuda.is_available()
    yield
    status, word = fa.device_error()
    assert status == 0 and word == 0, f"kernel error word {word:#x}"


def _capture(fn):
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        fn()  # warm-up outside the capture
    torch.cuda.current_stream().wait_stream(side)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn()
    return g


CASES = {
    # 152 items of 256 rows: the last wave is split and merged; dynamic counter for the causal one
    "dense_split": dict(layout="BNSD", shape=(1, 19, 2048, 128), dtype="f16", kw={}),
    "dense_causal_sink": dict(layout="BNSD", shape=(1, 19, 2048, 128), dtype="bf16", kw=dict(next_tokens=0),
                              sink=True),
    "varlen": dict(layout="TND", lens=[300, 0, 513, 129, 1, 777], heads=4, kv_heads=2, d=128, dtype="bf16",
                   kw=dict(next_tokens=0)),
    "wide_varlen": dict(layout="TND", lens=[200, 333, 64], heads=2, kv_heads=2, d=256, dtype="f16",
                        kw=dict(next_tokens=0)),
}


def _inputs(c, seed):
    if c["layout"] == "TND":
        t = sum(c["lens"])
        q = normal((t, c["heads"], c["d"]), c["dtype"], seed)
        k = normal((t, c["kv_heads"], c["d"]), c["dtype"], seed + 1)
        v = normal((t, c["kv_heads"], c["d"]), c["dtype"], seed + 2)
    else:
        q, k, v = (normal(c["shape"], c["dtype"], seed + i) for i in range(3))
    return q.cuda(), k.cuda(), v.cuda()


def _churn():
    # other calls with other tables between capture and replay: host memory that
    # a captured host-to-device copy pointed at would now hold other bytes
    for lens in ([5, 900, 31], [256] * 40, [1] * 300):
        t = sum(lens)
        x = normal((t, 2, 64), "f16", 6500 + len(lens)).cuda()
        cum = cumulative(lens, False)
        fa.fa_fwd(x, x, x, input_layout="TND", head_num=2, actual_seq_qlen=cum, actual_seq_kvlen=cum)
    torch.cuda.synchronize()


@pytest.mark.parametrize("name", list(CASES))
def test_graph_replay_equals_eager(name):
    c = CASES[name]
    q, k, v = _inputs(c, 6000)
    kw = dict(input_layout=c["layout"], **c["kw"])
    if c["layout"] == "TND":
        cum = cumulative(c["lens"], False)
        kw.update(head_num=c["heads"], actual_seq_qlen=cum, actual_seq_kvlen=cum)
    else:
        kw.update(head_num=c["shape"][1])
    if c.get("sink"):
        kw["sink"] = normal((kw["head_num"],), "f32", 6010).cuda()
    out, smax, ssum = fa.fa_fwd(q, k, v, **kw)
    g = _capture(lambda: fa.fa_fwd(q, k, v, out=out, softmax_max=smax, softmax_sum=ssum, **kw))
    _churn()
    for seed in (6100, 6200):
        nq, nk, nv = _inputs(c, seed)
        q.copy_(nq), k.copy_(nk), v.copy_(nv)
        out.fill_(float("nan"))
        g.replay()
        torch.cuda.synchronize()
        want = fa.fa_fwd(q, k, v, **kw)
        torch.cuda.synchronize()
        assert torch.equal(out, want[0]) and torch.equal(smax, want[1]) and torch.equal(ssum, want[2])


def test_static_entry_graph_replay_equals_eager():
    from attention_forward_20_b200.static_scratch import fa_fwd_varlen_static
    c = CASES["varlen"]
    q, k, v = _inputs(c, 6300)
    cum = cumulative(c["lens"], False)
    want = fa.fa_fwd(q, k, v, input_layout="TND", head_num=4, actual_seq_qlen=cum, actual_seq_kvlen=cum,
                     next_tokens=0)
    out, smax, ssum = (torch.empty_like(t) for t in want)
    g = _capture(lambda: fa_fwd_varlen_static(q, k, v, cum, cum, out, smax, ssum, head_num=4, next_tokens=0))
    # an eager call with another table rewrites the shared host staging buffer
    # and the device scratch; the replay must bring its own table back
    lens_b = [64, 1000, 3, 400]
    xb = normal((sum(lens_b), 4, 128), "bf16", 6450).cuda()
    cum_b = cumulative(lens_b, False)
    ob, mb, lb = (torch.empty_like(t) for t in fa.fa_fwd(xb, xb, xb, input_layout="TND", head_num=4,
                                                          actual_seq_qlen=cum_b, actual_seq_kvlen=cum_b))
    fa_fwd_varlen_static(xb, xb, xb, cum_b, cum_b, ob, mb, lb, head_num=4)
    _churn()
    nq, nk, nv = _inputs(c, 6400)
    q.copy_(nq), k.copy_(nk), v.copy_(nv)
    g.replay()
    torch.cuda.synchronize()
    want = fa.fa_fwd(q, k, v, input_layout="TND", head_num=4, actual_seq_qlen=cum, actual_seq_kvlen=cum,
                     next_tokens=0)
    torch.cuda.synchronize()
    assert torch.equal(out, want[0]) and torch.equal(smax, want[1]) and torch.equal(ssum, want[2])
