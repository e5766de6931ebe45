"""Host-side pieces of bench.py that need no GPU: the kernel-source hash that
guards the recorded ncu traffic changes with the code, not with comments; the
recorded traffic is used only for the sources it was taken on; the tensor
roofline of the prefill-shaped workloads counts the call's flops."""
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


def test_recorded_traffic_only_for_the_current_sources(tmp_path, monkeypatch):
    import json

    _copy_sources(tmp_path)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    (tmp_path / "profiles").mkdir()
    h = bench.kernel_source_hash()
    rec = {"decode_hld_fp16": {"dram_bytes_per_launch": 123, "kernel_hash": h},
           "specdec_hld_fp16": {"dram_bytes_per_launch": 456, "kernel_hash": "0" * 16}}
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps(rec))
    assert bench.recorded_traffic("decode_hld_fp16") == 123
    assert bench.recorded_traffic("specdec_hld_fp16") is None  # taken on other sources
    assert bench.recorded_traffic("gqa_kvcache_bf16") is None  # never taken


def test_tensor_roofline_charges_the_call_with_its_flops():
    from decode_flashattention_b200 import workloads as wl

    w = wl.WORKLOADS["mla_prefill2k_bf16"]
    assert w.tensor_bound and wl.WORKLOADS["gqa_prefill4k_bf16"].tensor_bound
    assert not wl.WORKLOADS["decode_hld_fp16"].tensor_bound
    flops = wl.attn_flops(w)
    # causal 2048 queries over 8192 keys: query i sees 6144 + i + 1 keys
    visible = sum(6144 + i + 1 for i in range(2048)) * 32
    assert flops == 2 * (192 + 128) * visible
    prof = {"main_ms": 2.0, "main_launches": 4, "combine_ms": 0.4}
    r = bench.tensor_roofline(w, None, 0.5, prof, None, "split-KV kernel + combine (whole call)")
    assert r["bound"] == "tensor" and r["unit"] == "TFLOP/s"
    assert r["algorithmic_flops_per_launch"] == flops
    assert abs(r["achieved"] - flops / 0.5e-3 / 1e12) < 0.01
    assert abs(r["frac"] - r["achieved"] / r["peak"]) < 1e-4
    assert r["isolated_us"] == {"main": 500.0, "combine": 100.0}
    assert r["kernel"] == "split-KV kernel + combine (whole call)"
