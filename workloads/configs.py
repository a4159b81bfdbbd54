"""The five attention-forward workloads, as data, and a builder for their inputs.

Shapes follow the example calls on the mindie-sd "core acceleration API" page
(attention_forward: [2,4096,24,128] fp16; attention_forward_varlen: T=8192,
N=24, D=128) and the operator limits on the aclnnFlashAttentionScore /
aclnnFlashAttentionVarLenScoreV5 pages.  Seeds: q = 1000*c+1, k = +2, v = +3,
sink = +4 for workload number c.
"""
from dataclasses import dataclass, field
from typing import Optional, List

import torch

from .gen import normal, varlen_lengths, cumulative, causal_mask_u8, alibi_slopes

INT64_MAX = 2**63 - 1


@dataclass
class Workload:
    name: str
    number: int
    layout: str
    dtype: str
    head_num: int
    q: torch.Tensor
    k: torch.Tensor
    v: torch.Tensor
    scale: float
    pre_tokens: int = INT64_MAX
    next_tokens: int = INT64_MAX
    pse: Optional[torch.Tensor] = None
    pse_type: int = 0
    atten_mask: Optional[torch.Tensor] = None
    mask_mode: int = 0
    sink: Optional[torch.Tensor] = None
    actual_seq_q: Optional[List[int]] = None   # cumulative, no leading zero
    actual_seq_kv: Optional[List[int]] = None
    softmax_out_layout: str = ""
    extra: dict = field(default_factory=dict)


CONFIGS = {
    1: "tiny BNSD fp32 [1,2,128,64], no mask",
    2: "dense BNSD fp16 [2,24,4096,128], no mask",
    3: "causal BSND bf16 [4,8192,32,128], lower-triangular attenMask, per-head sink",
    4: "varlen TND bf16 T=8192 N=24 D=128, 8 sequences, causal",
    5: "band BSH fp16 [2,16384,1024] N=16 D=64, preTokens=2048 nextTokens=0, ALiBi slopes",
}


def build(number, seq_scale=1, with_mask_tensor=True):
    """Inputs of workload `number` (CPU tensors).

    `seq_scale` > 1 divides every sequence length by that factor (kept >= 1), for
    parity runs that the float64 oracle finishes quickly at the same structure.
    """
    c = number
    sq = lambda s: max(1, s // seq_scale)  # noqa: E731
    if c == 1:
        shape = (1, 2, sq(128), 64)
        return Workload("tiny", 1, "BNSD", "f32", 2,
                        normal(shape, "f32", 1001), normal(shape, "f32", 1002),
                        normal(shape, "f32", 1003), scale=1.0 / 8.0)
    if c == 2:
        shape = (2, 24, sq(4096), 128)
        return Workload("dense", 2, "BNSD", "f16", 24,
                        normal(shape, "f16", 2001), normal(shape, "f16", 2002),
                        normal(shape, "f16", 2003), scale=128 ** -0.5)
    if c == 3:
        s = sq(8192)
        shape = (4, s, 32, 128)
        w = Workload("causal_sink", 3, "BSND", "bf16", 32,
                     normal(shape, "bf16", 3001), normal(shape, "bf16", 3002),
                     normal(shape, "bf16", 3003), scale=128 ** -0.5,
                     pre_tokens=INT64_MAX, next_tokens=0,
                     sink=normal((32,), "f32", 3004))
        if with_mask_tensor:
            w.atten_mask = causal_mask_u8(s, s)
            w.mask_mode = 1
        return w
    if c == 4:
        lens = varlen_lengths(8192, 8, 256, 2048, seed=4)
        if seq_scale > 1:
            lens = [max(1, x // seq_scale) for x in lens]
        t = sum(lens)
        shape = (t, 24, 128)
        cum = cumulative(lens, leading_zero=False)
        w = Workload("varlen_causal", 4, "TND", "bf16", 24,
                     normal(shape, "bf16", 4001), normal(shape, "bf16", 4002),
                     normal(shape, "bf16", 4003), scale=128 ** -0.5,
                     pre_tokens=INT64_MAX, next_tokens=0,
                     actual_seq_q=cum, actual_seq_kv=list(cum))
        w.extra["lengths"] = lens
        w.extra["cu_seqlens"] = cumulative(lens, leading_zero=True)
        return w
    if c == 5:
        s = sq(16384)
        shape = (2, s, 1024)
        return Workload("band_alibi", 5, "BSH", "f16", 16,
                        normal(shape, "f16", 5001), normal(shape, "f16", 5002),
                        normal(shape, "f16", 5003), scale=64 ** -0.5,
                        pre_tokens=max(1, 2048 // seq_scale), next_tokens=0,
                        pse=alibi_slopes(16), pse_type=2)
    raise ValueError(f"unknown workload {number}")
