"""The five attention workloads this library is tested and measured on.

Each entry fixes the shape [B, H, N, d], the element type, the masks, the dropout
rate, the seed and the factor that scales the unit-normal draws.  The shapes are
the ones the FlashAttention write-ups discuss: a small fp32 head, a 1k-token
self-attention block, a GPT-style causal decoder head at N=4096, d=128, a
BERT-large block with key padding and dropout, and a 64k-token causal context.
Nothing in this module computes attention.
"""
from dataclasses import dataclass, field
from typing import Optional, Tuple


@dataclass(frozen=True)
class Workload:
    name: str
    dtype: str            # "f32" or "bf16": element type of q, k, v, o and the gradients
    B: int
    H: int
    N: int
    d: int
    causal: bool
    seed: int
    factor: float = 1.0   # the N(0,1) draws are multiplied by this
    key_len_range: Optional[Tuple[int, int]] = None   # inclusive [lo, hi], per batch entry
    dropout_p: float = 0.0
    backward: bool = True
    # sampled-row checking for contexts too long to materialise N x N on the host
    sample_rows: Optional[int] = None
    bwd_check_heads: Optional[Tuple[int, ...]] = None
    extra: dict = field(default_factory=dict)

    @property
    def scale(self) -> float:
        return 1.0 / float(self.d) ** 0.5

    def fwd_flops(self) -> float:
        """4 N^2 d B H, halved under a causal mask (the nominal count; padding is not discounted)."""
        f = 4.0 * self.N * self.N * self.d * self.B * self.H
        return f / 2 if self.causal else f

    def fwd_bwd_flops(self) -> float:
        """Forward plus backward, the backward counted as 2.5 times the forward."""
        return 3.5 * self.fwd_flops()


WORKLOADS = {
    w.name: w
    for w in [
        Workload("fp32_1x1x128x64", "f32", 1, 1, 128, 64, False, seed=0, backward=False),
        Workload("bf16_4x16x1024x64", "bf16", 4, 16, 1024, 64, False, seed=1),
        Workload("bf16_causal_2x16x4096x128", "bf16", 2, 16, 4096, 128, True, seed=2, factor=0.5),
        Workload("bf16_keypad_dropout_16x16x512x64", "bf16", 16, 16, 512, 64, False, seed=3,
                 key_len_range=(256, 512), dropout_p=0.1),
        Workload("bf16_causal_1x16x65536x64", "bf16", 1, 16, 65536, 64, True, seed=4,
                 sample_rows=256, bwd_check_heads=(0,)),
    ]
}

# The workload the throughput figure is quoted on.
HEADLINE = "bf16_causal_2x16x4096x128"
