"""Host-side pieces of bench.py that need no GPU: the kernel-source hash that
guards the recorded ncu traffic changes with the code, not with comments."""
import os
import shutil

import bench


def _copy_sources(tmp_path):
    src = os.path.join(bench.ROOT, "decode_flashattention_b200", "csrc")
    dst = tmp_path / "decode_flashattention_b200" / "csrc"
    shutil.copytree(src, dst)
    return dst


def test_source_hash_ignores_comments_and_tracks_code(tmp_path, monkeypatch):
    dst = _copy_sources(tmp_path)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    h0 = bench.kernel_source_hash()
    f = dst / "fa_combine.cu"
    text = f.read_text()
    f.write_text("// a new comment\n" + text.replace("namespace fa {", "namespace fa {  /* and another */", 1))
    assert bench.kernel_source_hash() == h0
    f.write_text(text.replace("kPartsPerPass = 8", "kPartsPerPass = 4", 1))
    assert bench.kernel_source_hash() != h0
