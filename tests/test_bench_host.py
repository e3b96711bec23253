"""bench.py's host arithmetic on the CPU: the algorithmic bytes and flops each
roofline figure divides by, and the validity check of the committed ncu
traffic figures against the kernel sources."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_algorithmic_bytes_and_flops():
    # decode QKV, M = 1: x 8 KB + W' 4096 x 6144 bf16 + y 12 KB
    by, fl = bench.algorithmic(1, 4096, 6144, False)
    assert by == 1 * 4096 * 2 + 4096 * 6144 * 2 + 1 * 6144 * 2
    assert fl == 2.0 * 1 * 4096 * 6144
    # SwiGLU reads both halves of the weight but writes N outputs
    by, fl = bench.algorithmic(16, 4096, 14336, True)
    assert by == 16 * 4096 * 2 + 4096 * 28672 * 2 + 16 * 14336 * 2
    assert fl == 2.0 * 16 * 4096 * 28672
    # fp8 weights: one byte per element (the 128x128 block scales are ignored here)
    by, _ = bench.algorithmic(1, 5120, 13824, True, wbytes_per_elem=1)
    assert by == 5120 * 2 + 5120 * 27648 + 13824 * 2


def test_algorithmic_bytes_nvfp4_output():
    # half a byte per output and one scale byte per 16 outputs
    by, fl = bench.algorithmic(4096, 4096, 14336, True, out="nvfp4")
    assert by == 4096 * 4096 * 2 + 4096 * 28672 * 2 + 4096 * 14336 // 2 + 4096 * 14336 // 16
    assert fl == 2.0 * 4096 * 4096 * 28672


def test_profile_traffic_requires_matching_sources(tmp_path, monkeypatch):
    names = ["tc.cu", "ptx.cuh", "nvfp4.cuh"]
    h = bench.kernel_source_hash(names)
    prof = tmp_path / "profiles"
    prof.mkdir()
    (prof / "k.md").write_text(f"# k\n\n- source_sha256: {h}\n- dram_bytes_per_launch: 1234\n")
    (prof / "old.md").write_text("# k\n\n- source_sha256: 0000000000000000\n- dram_bytes_per_launch: 99\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))   # only the profiles folder moves
    assert bench.profile_traffic("k.md", h) == 1234.0
    assert bench.profile_traffic("old.md", h) is None
    assert bench.profile_traffic("missing.md", h) is None
