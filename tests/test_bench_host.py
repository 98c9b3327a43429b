"""Host-side logic of bench.py that decides what the JSON line reports (no GPU).

The roofline's `traffic` comes from a committed ncu summary and is reported only while the
kernel's code is the code that was captured: the hash ignores comments and blank lines, and
changes with any edit of the code itself.
"""

import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

KERNEL = """// a kernel
#include "x.cuh"

/* block comment
   over two lines */
__global__ void k(float* p) {   // trailing comment
    p[threadIdx.x] += 1.0f;
}
"""


def _fake_tree(tmp_path, kernel_src, summary=None):
    csrc = tmp_path / "post_weight_quantization_24_b200" / "csrc"
    csrc.mkdir(parents=True)
    (csrc / "k.cu").write_text(kernel_src)
    if summary is not None:
        (tmp_path / "profiles").mkdir()
        (tmp_path / "profiles" / "k.md").write_text(summary)


def test_code_hash_ignores_comments_and_blank_lines(tmp_path, monkeypatch):
    import bench
    _fake_tree(tmp_path, KERNEL)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    h0 = bench.code_sha("k.cu")
    edited = KERNEL.replace("// a kernel", "// the same kernel, reworded\n\n// more notes")
    edited = edited.replace("// trailing comment", "// another comment")
    edited = edited.replace("/* block comment\n   over two lines */", "/* one line */")
    (tmp_path / "post_weight_quantization_24_b200" / "csrc" / "k.cu").write_text(edited)
    assert bench.code_sha("k.cu") == h0


def test_code_hash_changes_with_the_code(tmp_path, monkeypatch):
    import bench
    _fake_tree(tmp_path, KERNEL)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    h0 = bench.code_sha("k.cu")
    (tmp_path / "post_weight_quantization_24_b200" / "csrc" / "k.cu").write_text(
        KERNEL.replace("+= 1.0f", "+= 2.0f"))
    assert bench.code_sha("k.cu") != h0


def test_traffic_reported_only_for_the_captured_code(tmp_path, monkeypatch):
    import bench
    _fake_tree(tmp_path, KERNEL)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    h = bench.code_sha("k.cu")
    (tmp_path / "profiles").mkdir()
    summary = tmp_path / "profiles" / "k.md"
    summary.write_text(f"kernel_code_sha256: {h} (csrc/k.cu)\n\ndram_bytes_per_launch_full_size: 2.5e9\n")
    traffic, path = bench.ncu_traffic("k.md", "k.cu")
    assert traffic == 2.5e9 and path == str(summary)
    # the kernel changes after the capture: no traffic
    (tmp_path / "post_weight_quantization_24_b200" / "csrc" / "k.cu").write_text(
        KERNEL.replace("+= 1.0f", "*= 3.0f"))
    assert bench.ncu_traffic("k.md", "k.cu")[0] is None
    # a summary without the figure, or no summary at all
    summary.write_text(f"kernel_code_sha256: {h} (csrc/k.cu)\n")
    assert bench.ncu_traffic("k.md", "k.cu")[0] is None
    assert bench.ncu_traffic("missing.md", "k.cu") == (None, None)
