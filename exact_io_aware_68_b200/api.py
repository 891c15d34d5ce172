"""Tensor-level calls of the C ABI (same names as ``include/fa.h`` minus the prefix).

Arguments are CUDA tensors in the [B, H, N, d] layout; results are written into tensors
allocated here (or passed in).  Work runs on the current torch CUDA stream of the inputs' device,
with that device made current for the call (the library launches on the current device).
"""
import math

import torch

from . import _lib


def _stream(t: torch.Tensor) -> int:
    return torch.cuda.current_stream(t.device).cuda_stream


def _ptr(t):
    return None if t is None else t.data_ptr()


def _check_tensor(name, t, dtype, shape=None):
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")


def attention_fwd(q, k, v, scale=None, causal=False, key_lens=None, dropout_p=0.0, seed=0, o=None, lse=None):
    """O and lse of exact attention (``fa_fwd`` for bf16 inputs, ``fa_fwd_f32`` for fp32)."""
    B, H, N, d = q.shape
    dtype = q.dtype
    for name, t in (("q", q), ("k", k), ("v", v)):
        _check_tensor(name, t, dtype, (B, H, N, d))
    if key_lens is not None:
        _check_tensor("key_lens", key_lens, torch.int32, (B,))
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    if o is None:
        o = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
    name = {torch.bfloat16: "fa_fwd", torch.float32: "fa_fwd_f32"}.get(dtype)
    if name is None:
        raise ValueError(f"unsupported dtype {dtype}")
    with torch.cuda.device(q.device):   # the library launches on the current device
        _lib.call(name, q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), B, H, N, d, scale,
                  int(bool(causal)), _ptr(key_lens), float(dropout_p), int(seed), _stream(q))
    return o, lse


def bwd_workspace(B, H, N, d, device):
    """A workspace tensor of ``fa_bwd_workspace_size`` bytes (torch allocations are 256-byte aligned)."""
    n = _lib.load().fa_bwd_workspace_size(B, H, N, d)
    return torch.empty(n, dtype=torch.uint8, device=device)


def attention_bwd(q, k, v, o, lse, do, scale=None, causal=False, key_lens=None, dropout_p=0.0, seed=0,
                  workspace=None, dq=None, dk=None, dv=None, separate_dq=False):
    """dQ, dK, dV of exact attention (``fa_bwd``; ``fa_bwd_split`` with ``separate_dq``)."""
    B, H, N, d = q.shape
    for name, t in (("q", q), ("k", k), ("v", v), ("o", o), ("do", do)):
        _check_tensor(name, t, torch.bfloat16, (B, H, N, d))
    _check_tensor("lse", lse, torch.float32, (B, H, N))
    if key_lens is not None:
        _check_tensor("key_lens", key_lens, torch.int32, (B,))
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    if workspace is None:
        workspace = bwd_workspace(B, H, N, d, q.device)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    with torch.cuda.device(q.device):   # the library launches on the current device
        _lib.call("fa_bwd_split" if separate_dq else "fa_bwd", q.data_ptr(), k.data_ptr(), v.data_ptr(),
                  o.data_ptr(), lse.data_ptr(), do.data_ptr(),
                  dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), B, H, N, d, scale, int(bool(causal)),
                  _ptr(key_lens), float(dropout_p), int(seed), workspace.data_ptr(), workspace.numel(), _stream(q))
    return dq, dk, dv


def attention_decode(q, k, v, scale=None, causal=False, key_lens=None, workspace=None, o=None, lse=None):
    """O and lse of Nq query rows against a cache of Nkv keys (``fa_fwd_decode``).

    q: bf16 [B, H, Nq, d]; k, v: bf16 [B, H, Nkv, d]; key_lens: int32 [B] valid cache lengths."""
    B, H, Nq, d = q.shape
    Nkv = k.shape[2]
    _check_tensor("q", q, torch.bfloat16, (B, H, Nq, d))
    for name, t in (("k", k), ("v", v)):
        _check_tensor(name, t, torch.bfloat16, (B, H, Nkv, d))
    if key_lens is not None:
        _check_tensor("key_lens", key_lens, torch.int32, (B,))
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    if workspace is None:
        n = _lib.load().fa_fwd_decode_workspace_size(B, H, Nq, Nkv, d)
        workspace = torch.empty(n, dtype=torch.uint8, device=q.device)
    o = torch.empty_like(q) if o is None else o
    lse = torch.empty((B, H, Nq), dtype=torch.float32, device=q.device) if lse is None else lse
    with torch.cuda.device(q.device):
        _lib.call("fa_fwd_decode", q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), B, H, Nq,
                  Nkv, d, scale, int(bool(causal)), _ptr(key_lens), workspace.data_ptr(), workspace.numel(), _stream(q))
    return o, lse


def dropout_mask(B, H, N, dropout_p, seed, device="cuda"):
    """uint8 [B, H, N, N] keep decisions of the counter hash (``fa_dropout_mask``)."""
    keep = torch.empty((B, H, N, N), dtype=torch.uint8, device=device)
    with torch.cuda.device(keep.device):
        _lib.call("fa_dropout_mask", keep.data_ptr(), B, H, N, float(dropout_p), int(seed), _stream(keep))
    return keep


def check(stream=None):
    """``fa_check`` on the current stream: raises FAError on a device-reported failure."""
    s = torch.cuda.current_stream().cuda_stream if stream is None else stream
    _lib.call("fa_check", s)
