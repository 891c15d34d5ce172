"""Exact IO-aware attention for NVIDIA B200 (sm_100a).

The computation lives in ``libfa_sm100.so`` (C ABI: ``include/fa.h``); this package passes
device pointers and the current CUDA stream to it.  PyTorch provides device memory and streams
only.  Importing the package does not load the library; the first call does, and fails loudly
when it is missing.
"""
from .api import attention_bwd, attention_decode, attention_fwd, bwd_workspace, check, dropout_mask
from .autograd import FlashAttentionFunction, flash_attention

__all__ = ["attention_fwd", "attention_bwd", "attention_decode", "bwd_workspace", "check", "dropout_mask", "flash_attention",
           "FlashAttentionFunction"]
