"""Seeded random tensors and integer/boolean structure for attention inputs.

Everything is drawn on the CPU from an explicit seed so that the oracle and the
GPU path see bit-identical inputs.  Floating values are drawn in fp32 from a
torch.Generator and then rounded to the target dtype (round to nearest even).
"""
import numpy as np
import torch

TORCH_DTYPES = {
    "f32": torch.float32,
    "f16": torch.float16,
    "bf16": torch.bfloat16,
}


def normal(shape, dtype, seed):
    """N(0,1) tensor of `shape`, drawn in fp32 with `seed`, rounded to `dtype` ("f32"/"f16"/"bf16")."""
    g = torch.Generator().manual_seed(int(seed))
    x = torch.randn(*shape, generator=g, dtype=torch.float32)
    return x.to(TORCH_DTYPES[dtype])


def varlen_lengths(total=8192, count=8, lo=256, hi=2048, seed=4):
    """Sequence lengths in [lo, hi] summing to `total`.

    Draws count-1 lengths uniformly in [lo, hi] with numpy's default_rng(seed);
    the last one is total minus their sum; the draw repeats until that last
    length also falls in [lo, hi].
    """
    rng = np.random.default_rng(seed)
    while True:
        head = rng.integers(lo, hi + 1, size=count - 1)
        last = total - int(head.sum())
        if lo <= last <= hi:
            return [int(x) for x in head] + [last]


def cumulative(lengths, leading_zero):
    """Cumulative sums of `lengths`; with `leading_zero` the (B+1,) cu_seqlens form."""
    c = np.cumsum(np.asarray(lengths, dtype=np.int64))
    if leading_zero:
        c = np.concatenate([[0], c])
    return [int(x) for x in c]


def causal_mask_u8(sq, skv):
    """uint8 [sq, skv] mask with 1 (excluded) strictly above the diagonal, j > i."""
    i = torch.arange(sq).unsqueeze(1)
    j = torch.arange(skv).unsqueeze(0)
    return (j > i).to(torch.uint8)


def alibi_slopes(n_heads):
    """fp32 [n_heads] slopes 2^(-8 h / N) with h = 1..N (head index n = h - 1)."""
    h = torch.arange(1, n_heads + 1, dtype=torch.float64)
    return torch.pow(2.0, -8.0 * h / n_heads).to(torch.float32)
