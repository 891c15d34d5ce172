"""The autograd wrapper: marshalling checks on the CPU, gradients against the fp64 oracle on a
B200 (same seeded inputs, same tolerances as the direct backward parity tests)."""
import numpy as np
import pytest
import torch

import oracle
from exact_io_aware_68_b200 import api, flash_attention
from exact_io_aware_68_b200.inputs import make_inputs
from exact_io_aware_68_b200.workloads import Workload
from helpers import GRAD_REL_L2, O_MAX_ABS_BF16, assert_o_close, key_lens_device, rel_l2, to_device, to_f64


def wl(B, H, N, d, causal=False, pad=None, p=0.0, seed=11):
    return Workload("case", "bf16", B, H, N, d, causal, seed=seed, factor=1.0, key_len_range=pad, dropout_p=p)


def test_host_tensors_are_rejected_before_any_library_call():
    q = torch.zeros(1, 1, 4, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="CUDA"):
        flash_attention(q, q, q)


AG_CASES = [wl(1, 2, 200, 64, causal=True), wl(2, 1, 260, 128, causal=True, pad=(130, 260), p=0.1, seed=7),
            wl(1, 2, 128, 128, pad=(60, 128))]


@pytest.mark.gpu
@pytest.mark.parametrize("w", AG_CASES, ids=lambda w: f"{w.B}x{w.H}x{w.N}x{w.d}-c{int(w.causal)}-p{w.dropout_p}")
def test_autograd_gradients_match_oracle(w):
    x = make_inputs(w)
    q, k, v = (to_device(x, n).requires_grad_() for n in ("q", "k", "v"))
    do = to_device(x, "do")
    o = flash_attention(q, k, v, x["scale"], w.causal, key_lens_device(x), w.dropout_p, x["seed"])
    o.backward(do)
    api.check()
    O, _ = oracle.forward(x["q64"], x["k64"], x["v64"], x["scale"], w.causal, x["key_lens"], w.dropout_p, x["seed"])
    assert_o_close(to_f64(o.detach()), O, O_MAX_ABS_BF16)
    ref = oracle.backward(x["q64"], x["k64"], x["v64"], x["do64"], x["scale"], w.causal, x["key_lens"],
                          w.dropout_p, x["seed"])
    for name, g, r in zip(("dq", "dk", "dv"), (q.grad, k.grad, v.grad), ref):
        err = rel_l2(to_f64(g), r)
        assert err <= GRAD_REL_L2, (name, err)


@pytest.mark.gpu
def test_autograd_forward_equals_direct_call():
    w = wl(2, 2, 300, 64, causal=True)
    x = make_inputs(w, with_do=False)
    q, k, v = (to_device(x, n) for n in ("q", "k", "v"))
    o1 = flash_attention(q, k, v, x["scale"], True)
    o2, _ = api.attention_fwd(q, k, v, x["scale"], True)
    api.check()
    assert torch.equal(o1, o2)
