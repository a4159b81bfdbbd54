"""Failure detection on the GPU without a GPU fault: every wait of the tcgen05
kernel is bounded.  FA_DEBUG_STALL=1 makes the kernel wait on a barrier that
is never signalled; the wait runs out after about two seconds, the kernel
winds down (waits, with a bound of its own, for the copies and MMAs it has
issued, frees TMEM, returns), the host reads FA_ERR_DEVICE_TIMEOUT from the
error word, and the context stays usable.  Both tcgen05 kernels and the rope
variant."""
import pytest
import torch

import attention_forward_20_b200 as fa
from tests.parity import compare_full
from workloads import Workload, normal

pytestmark = pytest.mark.gpu

KNOWN_SITES = set(range(1, 11))


def small():
    shape = (1, 2, 300, 128)
    return Workload("stall", 0, "BNSD", "bf16", 2, normal(shape, "bf16", 61), normal(shape, "bf16", 62),
                    normal(shape, "bf16", 63), scale=128 ** -0.5, next_tokens=0)


@pytest.mark.parametrize("kernel", ["two_tile", "wide", "rope"])
def test_stalled_wait_reports_timeout_and_context_survives(monkeypatch, kernel):
    from attention_forward_20_b200 import build
    build.build()
    fa.device_error()  # start clean
    w = small()
    monkeypatch.setenv("FA_DEBUG_STALL", "1")
    if kernel == "wide":  # head dim 256: the one-tile kernel
        x = normal((1, 2, 300, 256), "f16", 64).cuda()
        fa.fa_fwd(x, x, x, input_layout="BNSD", head_num=2, next_tokens=0)
    elif kernel == "rope":  # the rope variant, with its keyRope ring
        q, k, v = w.q.cuda(), w.k.cuda(), w.v.cuda()
        r = normal((1, 2, 300, 64), "bf16", 65).cuda()
        fa.fa_fwd(q, k, v, input_layout="BNSD", head_num=2, next_tokens=0, query_rope=r, key_rope=r)
    else:
        q, k, v = w.q.cuda(), w.k.cuda(), w.v.cuda()
        fa.fa_fwd(q, k, v, input_layout="BNSD", head_num=2, next_tokens=0)
    status, word = fa.device_error()  # synchronises
    assert status == fa.FA_ERR_DEVICE_TIMEOUT
    assert (word >> 32) in KNOWN_SITES and 1 <= (word & 0xFFFFFFFF) <= 148
    monkeypatch.delenv("FA_DEBUG_STALL")
    # the context is intact: the next call is correct and clean
    compare_full(w)
    assert fa.device_error() == (fa.FA_SUCCESS, 0)
    torch.cuda.synchronize()
