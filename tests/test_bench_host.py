"""Host-side logic of bench.py (CPU only): the kernel-code hash that ties the committed ncu
traffic figures to the sources they were measured on."""
import os
import shutil

import bench


def _copy_sources(tmp_path):
    src = os.path.join(bench.ROOT, "exact_io_aware_68_b200", "csrc")
    dst = tmp_path / "csrc"
    shutil.copytree(src, dst)
    return dst


def test_hash_ignores_comments_and_whitespace(tmp_path):
    dst = _copy_sources(tmp_path)
    before = bench.csrc_hash(str(dst))
    f = dst / "bwd_sm100.cuh"
    text = f.read_text(encoding="utf-8")
    f.write_text("// an added line comment\n/* an added\n   block comment */\n\n" + text.replace("\n", "\n  ", 3),
                 encoding="utf-8")
    assert bench.csrc_hash(str(dst)) == before


def test_hash_changes_with_code(tmp_path):
    dst = _copy_sources(tmp_path)
    before = bench.csrc_hash(str(dst))
    f = dst / "fwd_sm100.cuh"
    text = f.read_text(encoding="utf-8")
    assert "kRescaleThreshold = 8.0f" in text
    f.write_text(text.replace("kRescaleThreshold = 8.0f", "kRescaleThreshold = 7.0f"), encoding="utf-8")
    assert bench.csrc_hash(str(dst)) != before

