"""fa_bwd_noalloc: the backward for callers that cannot allocate device memory (needs a B200).

Such callers are, for example, plugins inside a runtime that owns all device memory and hands
them no workspace, or latency-critical loops that cannot afford cudaMalloc's implicit device
synchronisation.  The entry point keeps its scratch in a fixed array inside the library; its
gradients must match those of fa_bwd (which takes a caller workspace), call after call, because
the array keeps the previous call's contents and each call must clear what has to start at zero.

This file is collected last on purpose, so that a stop at the first failure has already run
every other test; it also passes on its own in a fresh process.
"""
import numpy as np
import pytest
import torch

from exact_io_aware_68_b200 import _lib, api
from exact_io_aware_68_b200.inputs import make_inputs
from exact_io_aware_68_b200.workloads import Workload
from helpers import GRAD_REL_L2, key_lens_device, rel_l2, run_fwd, to_device, to_f64

pytestmark = pytest.mark.gpu


def _noalloc(lib, q, k, v, o, lse, do, w, key_lens):
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    st = lib.fa_bwd_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), do.data_ptr(),
                            dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), w.B, w.H, w.N, w.d, w.scale,
                            int(w.causal), None if key_lens is None else key_lens.data_ptr(), w.dropout_p, w.seed,
                            torch.cuda.current_stream().cuda_stream)
    assert st == _lib.FA_OK, lib.fa_get_error()
    assert lib.fa_check(torch.cuda.current_stream().cuda_stream) == _lib.FA_OK, lib.fa_get_error()
    return dq, dk, dv


@pytest.mark.parametrize("w", [
    Workload("noalloc-causal", "bf16", 2, 4, 300, 128, True, seed=21, factor=0.5),
    Workload("noalloc-pad-dropout", "bf16", 3, 2, 257, 64, False, seed=22, key_len_range=(100, 257), dropout_p=0.1),
])
def test_noalloc_matches_workspace_backward_on_consecutive_calls(w):
    lib = _lib.load()
    x = make_inputs(w)
    q, k, v, o, lse = run_fwd(x)
    do = to_device(x, "do")
    kl = key_lens_device(x)
    ref = api.attention_bwd(q, k, v, o, lse, do, w.scale, w.causal, kl, w.dropout_p, w.seed)
    api.check()
    for _ in range(2):   # the second call starts from the first call's leftovers in the array
        got = _noalloc(lib, q, k, v, o, lse, do, w, kl)
        for name, g, r in zip(("dq", "dk", "dv"), got, ref):
            err = rel_l2(to_f64(g), to_f64(r))
            assert err <= GRAD_REL_L2, (name, err)
        # dK and dV involve no atomics: identical to the workspace path bit for bit
        assert torch.equal(got[1], ref[1]) and torch.equal(got[2], ref[2])


def test_noalloc_rejects_sizes_beyond_its_array():
    lib = _lib.load()
    cap = lib.fa_bwd_noalloc_max_scratch()
    assert cap == 48 << 20
    B, H, N, d = 2, 16, 4096, 128            # needs ~68 MB of scratch
    assert lib.fa_bwd_workspace_size(B, H, N, d) > cap
    fake = 0x10000                            # never dereferenced: the size check comes first
    st = lib.fa_bwd_noalloc(fake, fake, fake, fake, fake, fake, fake, fake, fake, B, H, N, d, 0.088, 1, None, 0.0,
                            0, None)
    assert st == _lib.FA_ERR_INVALID_ARG
    assert b"static" in lib.fa_get_error()
