"""CUDA path vs the fp64 oracle, element by element, on seeded inputs (needs a B200).

Sizes span several 128-row tiles plus ragged tails; edge cases: N = 1, N < 128, key lengths
that cut tiles, a zero key length (fully masked rows), dropout, causal + padding combined."""
import math

import numpy as np
import pytest
import torch

import oracle
from exact_io_aware_68_b200 import _lib, api
from exact_io_aware_68_b200.inputs import make_inputs
from exact_io_aware_68_b200.workloads import Workload
from helpers import (GRAD_REL_L2, LSE_MAX_ABS, O_MAX_ABS_BF16, O_MAX_ABS_F32, assert_o_close, bf16_product_bound,
                     key_lens_device, rel_l2, run_fwd, to_device, to_f64)

pytestmark = pytest.mark.gpu


def wl(B, H, N, d, causal=False, pad=None, p=0.0, seed=11, dtype="bf16", factor=1.0):
    return Workload("case", dtype, B, H, N, d, causal, seed=seed, factor=factor, key_len_range=pad, dropout_p=p)


FWD_CASES = [
    wl(1, 2, 1, 64), wl(1, 1, 3, 128), wl(2, 2, 127, 64), wl(1, 2, 128, 128), wl(2, 1, 129, 64),
    wl(1, 2, 300, 128, causal=True), wl(2, 2, 383, 64, causal=True), wl(1, 3, 512, 128, factor=2.0),
    wl(3, 2, 333, 64, pad=(1, 333)), wl(2, 2, 260, 128, causal=True, pad=(100, 260)),
    wl(2, 2, 300, 64, p=0.2, seed=5), wl(2, 1, 257, 128, causal=True, pad=(130, 257), p=0.1, seed=7),
]


@pytest.mark.parametrize("w", FWD_CASES, ids=lambda w: f"{w.B}x{w.H}x{w.N}x{w.d}-c{int(w.causal)}-"
                                                      f"pad{int(w.key_len_range is not None)}-p{w.dropout_p}")
def test_forward_matches_oracle(w):
    x = make_inputs(w, with_do=False)
    *_, o, lse = run_fwd(x)
    O, L = oracle.forward(x["q64"], x["k64"], x["v64"], x["scale"], w.causal, x["key_lens"], w.dropout_p, x["seed"])
    _, extra = bf16_product_bound(x, w)
    assert_o_close(to_f64(o), O, O_MAX_ABS_BF16, extra=extra)
    np.testing.assert_allclose(lse.cpu().numpy(), L, rtol=0, atol=LSE_MAX_ABS)


def test_forward_fp32_path():
    w = wl(1, 1, 128, 64, dtype="f32", seed=0)
    x = make_inputs(w, with_do=False)
    *_, o, lse = run_fwd(x)
    O, L = oracle.forward(x["q64"], x["k64"], x["v64"], x["scale"])
    assert np.abs(o.double().cpu().numpy() - O).max() <= O_MAX_ABS_F32
    np.testing.assert_allclose(lse.cpu().numpy(), L, rtol=0, atol=LSE_MAX_ABS)
    # fp32 with masks and dropout, d = 128, ragged N
    w = wl(2, 2, 200, 128, causal=True, pad=(50, 200), p=0.3, dtype="f32", seed=3)
    x = make_inputs(w, with_do=False)
    *_, o, lse = run_fwd(x)
    O, L = oracle.forward(x["q64"], x["k64"], x["v64"], x["scale"], True, x["key_lens"], 0.3, 3)
    assert np.abs(o.double().cpu().numpy() - O).max() <= O_MAX_ABS_F32
    np.testing.assert_allclose(lse.cpu().numpy(), L, rtol=0, atol=LSE_MAX_ABS)


def test_zero_key_length_rows():
    w = wl(3, 2, 200, 64, pad=(0, 0))
    x = make_inputs(w, with_do=True)
    x["key_lens"] = np.array([0, 150, 0], dtype=np.int32)
    q, k, v, o, lse = run_fwd(x)
    O, L = oracle.forward(x["q64"], x["k64"], x["v64"], x["scale"], False, x["key_lens"])
    assert torch.all(o[0] == 0) and torch.all(torch.isneginf(lse[0]))
    assert_o_close(to_f64(o), O, O_MAX_ABS_BF16)
    do = to_device(x, "do")
    dq, dk, dv = api.attention_bwd(q, k, v, o, lse, do, x["scale"], False, key_lens_device(x))
    api.check()
    for g in (dq, dk, dv):
        assert torch.all(g[0] == 0) and torch.all(g[2] == 0) and torch.isfinite(g.float()).all()


def test_dropout_mask_bit_exact():
    B, H, N, p, seed = 2, 3, 97, 0.37, 123456789
    keep = api.dropout_mask(B, H, N, p, seed).cpu().numpy().astype(bool)
    for b in range(B):
        for h in range(H):
            ref = oracle.keep_mask(seed, b, h, H, N, np.arange(N), np.arange(N), p)
            np.testing.assert_array_equal(keep[b, h], ref)


def test_identity_values_expose_the_kernel_dropout_mask():
    """V = I (N <= d): O = P * Z / (1 - p), so O == 0 exactly where the fused kernel dropped."""
    B, H, N, d, p, seed = 2, 2, 64, 64, 0.3, 99
    x = make_inputs(wl(B, H, N, d, p=p, seed=seed, factor=0.3), with_do=False)
    eye = np.zeros((B, H, N, d))
    eye[:, :, np.arange(N), np.arange(N)] = 1.0
    q, k = to_device(x, "q"), to_device(x, "k")
    v = torch.from_numpy(eye).to(torch.bfloat16).cuda()
    o, _ = api.attention_fwd(q, k, v, x["scale"], False, None, p, seed)
    api.check()
    got_drop = (o.float().cpu().numpy()[..., :N] == 0.0)
    for b in range(B):
        for h in range(H):
            ref_keep = oracle.keep_mask(seed, b, h, H, N, np.arange(N), np.arange(N), p)
            np.testing.assert_array_equal(got_drop[b, h], ~ref_keep)


BWD_CASES = [
    wl(1, 2, 128, 64), wl(1, 2, 128, 128), wl(2, 1, 200, 64, causal=True), wl(1, 2, 300, 128, causal=True),
    wl(2, 2, 257, 64, pad=(100, 257)), wl(1, 2, 384, 128), wl(2, 2, 300, 64, p=0.2, seed=5),
    wl(2, 1, 260, 128, causal=True, pad=(130, 260), p=0.1, seed=7), wl(1, 1, 1, 64), wl(1, 1, 5, 128),
]


@pytest.mark.parametrize("w", BWD_CASES, ids=lambda w: f"{w.B}x{w.H}x{w.N}x{w.d}-c{int(w.causal)}-"
                                                      f"pad{int(w.key_len_range is not None)}-p{w.dropout_p}")
def test_backward_matches_oracle(w):
    x = make_inputs(w)
    q, k, v, o, lse = run_fwd(x)
    do = to_device(x, "do")
    dq, dk, dv = api.attention_bwd(q, k, v, o, lse, do, x["scale"], w.causal, key_lens_device(x), w.dropout_p,
                                   x["seed"])
    api.check()
    ref = oracle.backward(x["q64"], x["k64"], x["v64"], x["do64"], x["scale"], w.causal, x["key_lens"],
                          w.dropout_p, x["seed"])
    for name, g, r in zip(("dq", "dk", "dv"), (dq, dk, dv), ref):
        err = rel_l2(to_f64(g), r)
        assert err <= GRAD_REL_L2, (name, err)


def test_forward_is_deterministic():
    x = make_inputs(wl(2, 2, 333, 128, causal=True), with_do=False)
    *_, o1, l1 = run_fwd(x)
    *_, o2, l2 = run_fwd(x)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_bounded_wait_reports_timeout_and_context_survives():
    lib = _lib.load()
    x = make_inputs(wl(1, 2, 256, 64), with_do=False)
    q, k, v = (to_device(x, n) for n in ("q", "k", "v"))
    lib.fa_set_wait_limit_ns(100_000_000)   # 0.1 s
    lib.fa_debug_set_flags(1)               # the load warp never delivers block 0
    try:
        o, lse = api.attention_fwd(q, k, v)
        st = lib.fa_check(torch.cuda.current_stream().cuda_stream)
    finally:
        lib.fa_debug_set_flags(0)
        lib.fa_set_wait_limit_ns(0)          # back to the default
    assert st == _lib.FA_ERR_TIMEOUT
    # the context is still usable and the next call is correct
    *_, o, lse = run_fwd(x)
    O, L = oracle.forward(x["q64"], x["k64"], x["v64"], x["scale"])
    assert_o_close(to_f64(o), O, O_MAX_ABS_BF16)


def test_outputs_only_16_byte_aligned():
    """Outputs that are 16- but not 32-byte aligned take the 16-byte store path of the epilogues."""
    w = wl(2, 2, 200, 128, causal=True, seed=31)
    x = make_inputs(w)
    q, k, v, do = (to_device(x, n) for n in ("q", "k", "v", "do"))
    n = q.numel()
    bufs = [torch.empty(n + 8, dtype=torch.bfloat16, device="cuda") for _ in range(4)]   # 8 bf16 = 16 bytes
    o, dq, dk, dv = (b[8:8 + n].view(q.shape) for b in bufs)
    assert all(t.data_ptr() % 32 == 16 for t in (o, dq, dk, dv))
    o, lse = api.attention_fwd(q, k, v, w.scale, True, o=o)
    api.attention_bwd(q, k, v, o, lse, do, w.scale, True, dq=dq, dk=dk, dv=dv)
    api.check()
    O, L = oracle.forward(x["q64"], x["k64"], x["v64"], w.scale, True)
    assert_o_close(to_f64(o), O, O_MAX_ABS_BF16)
    ref = oracle.backward(x["q64"], x["k64"], x["v64"], x["do64"], w.scale, True)
    for g, r in zip((dq, dk, dv), ref):
        assert rel_l2(to_f64(g), r) <= GRAD_REL_L2
