"""Decode-shaped forward (fa_fwd_decode) against the fp64 oracle (needs a B200), plus its host-side
argument checks (CPU).  Nq new query rows per head against a cache of Nkv keys; query i sits at
position L - Nq + i of a cache of L valid keys."""
import numpy as np
import pytest
import torch

import oracle
from exact_io_aware_68_b200 import _lib, api
from exact_io_aware_68_b200.build import build
from exact_io_aware_68_b200.inputs import make_decode_inputs
from helpers import LSE_MAX_ABS, O_MAX_ABS_BF16, assert_o_close, to_f64


def _up(a):
    return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).cuda()


def _check(B, H, Nq, Nkv, d, causal, lens, seed):
    x = make_decode_inputs(B, H, Nq, Nkv, d, seed, key_len_range=lens)
    kl = None if x["key_lens"] is None else torch.from_numpy(x["key_lens"]).cuda()
    o, lse = api.attention_decode(_up(x["q"]), _up(x["k"]), _up(x["v"]), x["scale"], causal, kl)
    api.check()
    O, L = oracle.forward_decode(x["q64"], x["k64"], x["v64"], x["scale"], causal, x["key_lens"])
    res = assert_o_close(to_f64(o), O, O_MAX_ABS_BF16, large_ok=True)
    lse_h = lse.cpu().numpy()
    assert np.array_equal(np.isneginf(lse_h), np.isneginf(L))
    fin = np.isfinite(L)
    l_err = float(np.abs(lse_h[fin] - L[fin]).max()) if fin.any() else 0.0
    assert l_err <= LSE_MAX_ABS, l_err
    assert res["max_err_small"] <= O_MAX_ABS_BF16
    return res["max_err"], l_err


CASES = [
    (1, 2, 1, 1, 64, False, None), (2, 2, 1, 200, 128, False, None), (1, 3, 5, 1000, 64, True, None),
    (2, 2, 16, 777, 128, True, (0, 777)), (3, 1, 8, 5000, 64, False, (3, 5000)), (1, 2, 64, 300, 128, True, None),
    (2, 1, 13, 129, 64, True, (5, 20)), (1, 4, 16, 4096, 128, False, None),
    (2, 3, 64, 1000, 64, True, (0, 1000)), (3, 2, 1, 1, 128, True, None),
]


@pytest.mark.gpu
@pytest.mark.parametrize("B,H,Nq,Nkv,d,causal,lens", CASES)
def test_decode_matches_oracle(B, H, Nq, Nkv, d, causal, lens):
    o_err, l_err = _check(B, H, Nq, Nkv, d, causal, lens, seed=80 + Nq + d)
    print(f"decode {B}x{H} Nq={Nq} Nkv={Nkv} d={d} causal={causal}: O max-abs {o_err:.3e}, lse {l_err:.3e}")


@pytest.mark.gpu
@pytest.mark.parametrize("Nq", [1, 8])
def test_decode_long_cache_64k(Nq):
    """Nq in {1, 8} against a 65,536-key cache, 16 heads, causal, every row checked."""
    o_err, l_err = _check(1, 16, Nq, 65536, 128, True, None, seed=90 + Nq)
    print(f"decode 64k Nq={Nq}: O max-abs {o_err:.3e}, lse {l_err:.3e}")


def test_decode_host_validation():
    build()
    lib = _lib.load()
    fake = 0x2000
    st = lib.fa_fwd_decode(fake, fake, fake, fake, fake, 1, 1, 65, 128, 64, 0.125, 0, None, 0x10000, 1 << 30, None)
    assert st == _lib.FA_ERR_UNSUPPORTED and b"Nq" in lib.fa_get_error()
    st = lib.fa_fwd_decode(fake, fake, fake, fake, fake, 1, 1, 4, 128, 96, 0.125, 0, None, 0x10000, 1 << 30, None)
    assert st == _lib.FA_ERR_UNSUPPORTED
    need = lib.fa_fwd_decode_workspace_size(1, 1, 4, 128, 64)
    assert need > 0 and need % 256 == 0
    st = lib.fa_fwd_decode(fake, fake, fake, fake, fake, 1, 1, 4, 128, 64, 0.125, 0, None, 0x10000, need - 1, None)
    assert st == _lib.FA_ERR_INVALID_ARG and b"workspace" in lib.fa_get_error()
    assert lib.fa_fwd_decode_workspace_size(0, 1, 4, 128, 64) == 0


def test_decode_split_fills_the_sms():
    """The key-range split: one CTA per SM, so the grid should fill whole waves of SMs with as few
    splits as that takes, in chunks of whole 128-key blocks of at least 512 keys."""
    build()
    lib = _lib.load()

    def split(BH, Nkv, sms):
        n = lib.fa_fwd_decode_split(1, BH, Nkv, sms)
        chunk = -(-Nkv // n)
        chunk = max(512, -(-chunk // 128) * 128)
        assert -(-Nkv // chunk) == n   # every split holds keys
        return n

    assert split(16, 65536, 148) == 9            # 144 CTAs: one wave (19 splits took three)
    assert split(16, 65536, 132) == 8            # 128 CTAs on a 132-SM part
    assert split(1, 4096, 148) == 8              # one head: the finest split, 512 keys each
    assert split(1, 1, 148) == 1
    assert split(444, 4096, 148) == 1            # three full waves already
    assert split(148, 65536, 148) == 1
    assert split(16, 65536, 0) == 128            # no device: the finest split bounds the workspace
    for BH, Nkv, sms in [(16, 65536, 148), (3, 5000, 148), (64, 32768, 148), (7, 100000, 148)]:
        n = split(BH, Nkv, sms)
        assert n <= split(BH, Nkv, 0)
        waves = -(-BH * n // sms)
        assert BH * n > (waves - 1) * sms       # no wave is empty
    assert lib.fa_fwd_decode_split(0, 1, 10, 148) == 0
