"""The C-ABI library builds for sm_100a, loads, exports every declared symbol, and rejects bad
arguments on the host before any device work (CPU only: no compute calls)."""
import ctypes
import os
import re

import pytest

from exact_io_aware_68_b200 import _lib
from exact_io_aware_68_b200.build import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build()
    return _lib.load()


def declared_symbols():
    text = open(os.path.join(ROOT, "include", "fa.h")).read()
    return re.findall(r"FA_API\s+[\w\s\*]+?\b(fa_\w+)\s*\(", text)


def test_every_declared_symbol_is_exported(lib):
    names = declared_symbols()
    assert len(names) >= 13
    for n in names:
        assert hasattr(lib, n), n
        assert n in _lib.SIGNATURES, n
    assert set(_lib.SIGNATURES) == set(names)


def test_version_and_workspace_size(lib):
    assert b"sm_100a" in lib.fa_version()
    B, H, N, d = 2, 16, 4096, 128
    dq = B * H * N * d * 4
    dvec = B * H * N * 4
    size = lib.fa_bwd_workspace_size(B, H, N, d)
    assert size == ((dq + 255) // 256) * 256 + ((dvec + 255) // 256) * 256 + 256   # + the work counter
    assert lib.fa_bwd_workspace_size(0, 1, 1, 64) == 0
    # ragged N keeps the second part 256-byte aligned
    assert lib.fa_bwd_workspace_size(1, 1, 3, 64) % 256 == 0


@pytest.mark.parametrize("args,status", [
    (dict(B=0), _lib.FA_ERR_INVALID_ARG),
    (dict(N=0), _lib.FA_ERR_INVALID_ARG),
    (dict(d=96), _lib.FA_ERR_UNSUPPORTED),
    (dict(d=512), _lib.FA_ERR_UNSUPPORTED),
    (dict(scale=0.0), _lib.FA_ERR_INVALID_ARG),
    (dict(scale=float("nan")), _lib.FA_ERR_INVALID_ARG),
    (dict(p=1.0), _lib.FA_ERR_INVALID_ARG),
    (dict(p=-0.1), _lib.FA_ERR_INVALID_ARG),
    (dict(q=0), _lib.FA_ERR_INVALID_ARG),
    (dict(q=0x1008), _lib.FA_ERR_INVALID_ARG),
    (dict(B=300, H=300), _lib.FA_ERR_UNSUPPORTED),
])
def test_host_validation_rejects_before_launch(lib, args, status):
    a = dict(q=0x1000, B=1, H=1, N=128, d=64, scale=0.125, p=0.0)
    a.update(args)
    fake = 0x2000   # never dereferenced: validation fails first
    st = lib.fa_fwd(a["q"], fake, fake, fake, fake, a["B"], a["H"], a["N"], a["d"], a["scale"], 0, None, a["p"], 0,
                    None)
    assert st == status
    assert len(lib.fa_get_error()) > 0


@pytest.mark.parametrize("d,status", [(0, _lib.FA_ERR_UNSUPPORTED), (129, _lib.FA_ERR_UNSUPPORTED),
                                      (256, _lib.FA_ERR_UNSUPPORTED)])
def test_fp32_head_dim_range(lib, d, status):
    """fa_fwd_f32 takes 1 <= d <= 128; outside that it refuses before touching the (fake) pointers."""
    fake = 0x2000
    st = lib.fa_fwd_f32(fake, fake, fake, fake, fake, 1, 1, 16, d, 0.125, 0, None, 0.0, 0, None)
    assert st == status and b"fp32" in lib.fa_get_error()


def test_backward_refuses_head_dim_256(lib):
    """d = 256 has a forward only; every backward entry point refuses it before any device work."""
    fake = 0x2000
    st = lib.fa_bwd(fake, fake, fake, fake, fake, fake, fake, fake, fake, 1, 1, 128, 256, 0.0625, 0, None, 0.0, 0,
                    0x10000, 1 << 30, None)
    assert st == _lib.FA_ERR_UNSUPPORTED and b"256" in lib.fa_get_error()


def test_bwd_workspace_validation(lib):
    fake = 0x2000
    # workspace too small / misaligned are rejected on the host
    st = lib.fa_bwd(fake, fake, fake, fake, fake, fake, fake, fake, fake, 1, 1, 128, 64, 0.125, 0, None, 0.0, 0,
                    fake, 16, None)
    assert st == _lib.FA_ERR_INVALID_ARG and b"workspace" in lib.fa_get_error()
    st = lib.fa_bwd(fake, fake, fake, fake, fake, fake, fake, fake, fake, 1, 1, 128, 64, 0.125, 0, None, 0.0, 0,
                    0x2010, 1 << 30, None)
    assert st == _lib.FA_ERR_INVALID_ARG and b"aligned" in lib.fa_get_error()
    st = lib.fa_dropout_mask(None, 1, 1, 4, 0.1, 0, None)
    assert st == _lib.FA_ERR_INVALID_ARG


def test_missing_library_fails_loudly(tmp_path, monkeypatch):
    monkeypatch.setattr(_lib, "_lib", None)
    with pytest.raises(RuntimeError, match="no fallback"):
        _lib.load(str(tmp_path / "absent.so"))


@pytest.mark.parametrize("l2,N,d,group", [
    (126 << 20, 4096, 128, 8),     # B200: Q, dO, dQ accumulator of 8 heads (4 MB each) in a quarter of L2
    (50 << 20, 4096, 128, 3),      # a smaller L2 holds fewer heads
    (126 << 20, 512, 64, 16),      # short heads: clamped to 16
    (126 << 20, 65536, 64, 1),     # one 32 MB head fills a quarter of L2 by itself
    (50 << 20, 1024, 64, 16),
    (6 << 20, 1024, 64, 3),
])
def test_backward_head_group_follows_the_l2_size(lib, l2, N, d, group):
    assert lib.fa_bwd_head_group(N, d, l2) == group
    assert lib.fa_bwd_head_group(0, d, l2) == 1
