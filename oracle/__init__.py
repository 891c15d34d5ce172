"""Host-side fp64 oracle for exact attention: TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py``
may import this package.  The library (``exact_io_aware_68_b200``) never calls it and
has no CPU fallback: it fails when its CUDA extension is missing.

What it computes is the plain definition of scaled-dot-product attention, written
out step by step in the order the sources give (matmul, scale, mask, softmax,
dropout, matmul), materialising the score matrix S and the probabilities P:

* "FlashAttention 的第一原则" (reader.mx), section 2 "简要解释注意力": one head maps
  Q, K, V (N x d) through the N x N intermediates to O (N x d); mask and dropout are
  optional and elementwise; section 3.2 lists the kernel chain matmul -> scale ->
  mask -> softmax -> dropout.
* "48 FlashAttention" (ml-canon), block "PyTorch FlashAttention под капотом sdpa":
  the output equals softmax(Q K^T / sqrt(d)) V; block "Backward — тоже без N×N": the
  backward works from Q, K, V and the saved normalisers (m, l).

The gradients are the exact derivatives of that forward function (the pages give no
backward formulas).  Each function names the passage it follows.  Every function here
is pinned by ``tests/test_oracle.py`` against brute force, closed forms, invariants,
finite differences and published hash vectors; none is "parity unpinned".
"""
from .attention import allowed_mask, forward, backward, forward_rows, backward_head_blocked, forward_decode
from .dropout import keep_mask, keep_threshold

__all__ = ["allowed_mask", "forward", "backward", "forward_rows", "backward_head_blocked", "forward_decode",
           "keep_mask", "keep_threshold"]
