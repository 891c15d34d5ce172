"""Drop-in differentiable attention: ``flash_attention(q, k, v, ...)`` returns O and lets autograd
reach dQ, dK and dV through the library's backward.

This module only marshals arguments. The forward calls ``fa_fwd`` (``fa_fwd_f32`` for fp32
inputs) and saves q, k, v, O and the per-row logsumexp. The backward recomputes P from them, so
the N x N probabilities are never stored. This is the recomputation of "48 FlashAttention", block
"Tiling и online softmax", backward paragraph, and of "Flash Attention：如何通过硬件感知优化重塑注意力
机制的未来", section 2.2.
The backward calls ``fa_bwd`` with the same scale, mask, dropout probability and seed, so it
regenerates the forward's dropout mask from the same counter hash. Only bf16 inputs have a
backward; for fp32 inputs the forward runs and a backward raises NotImplementedError.

Layout: q, k, v are [B, H, N, d] CUDA tensors. Non-contiguous inputs are copied once to
contiguous ones. The result has the input dtype.
"""
import math

import torch

from .api import attention_bwd, attention_fwd


class FlashAttentionFunction(torch.autograd.Function):
    """Exact attention O = dropout(softmax(mask(scale * Q K^T))) V with a library backward."""

    @staticmethod
    def forward(ctx, q, k, v, scale, causal, key_lens, dropout_p, seed):
        q, k, v = (t.contiguous() for t in (q, k, v))
        o, lse = attention_fwd(q, k, v, scale, causal, key_lens, dropout_p, seed)
        ctx.save_for_backward(q, k, v, o, lse)
        ctx.key_lens = key_lens
        ctx.args = (scale, causal, dropout_p, seed)
        return o

    @staticmethod
    def backward(ctx, do):
        q, k, v, o, lse = ctx.saved_tensors
        if q.dtype != torch.bfloat16:
            raise NotImplementedError("the attention backward is implemented for bf16 inputs only")
        scale, causal, dropout_p, seed = ctx.args
        do = do.to(torch.bfloat16).contiguous()
        dq, dk, dv = attention_bwd(q, k, v, o, lse, do, scale, causal, ctx.key_lens, dropout_p, seed)
        return dq, dk, dv, None, None, None, None, None


def flash_attention(q, k, v, scale=None, causal=False, key_lens=None, dropout_p=0.0, seed=None):
    """Exact attention of [B, H, N, d] CUDA tensors, differentiable in q, k and v.

    scale: the logit scale (default 1/sqrt(d)). causal: keep key j for query i only when j <= i.
    key_lens: int32 CUDA tensor [B]; keys j >= key_lens[b] are masked. dropout_p: probability of
    dropping each attention weight (inverted dropout); seed: the counter-hash seed (drawn from
    torch's default generator when None and dropout_p > 0). The backward reuses the same seed.
    """
    d = q.shape[-1]
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    if seed is None:
        seed = int(torch.randint(0, 2**62, (1,)).item()) if dropout_p > 0 else 0
    return FlashAttentionFunction.apply(q, k, v, scale, bool(causal), key_lens, float(dropout_p), int(seed))
