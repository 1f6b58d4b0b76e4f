"""bench.py's host-side bookkeeping, without a GPU: the profile staleness check.

The stream kernel's DRAM traffic is reported from the committed ncu summary only while the
kernel source's code matches the capture: comment edits keep it, code edits withdraw it.
"""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402

SRC = """// a comment
__global__ void k(float *x) {  // trailing comment
    /* block
       comment */ x[0] = 1.0f;
}
"""


def test_code_hash_ignores_comments_and_blank_space(tmp_path):
    a = tmp_path / "a.cu"
    a.write_text(SRC)
    b = tmp_path / "b.cu"
    b.write_text(SRC.replace("// a comment", "// another comment\n\n").replace("block", "other"))
    c = tmp_path / "c.cu"
    c.write_text(SRC.replace("1.0f", "2.0f"))
    assert bench.code_hash(str(a)) == bench.code_hash(str(b))
    assert bench.code_hash(str(a)) != bench.code_hash(str(c))


def test_profiled_traffic_only_while_the_code_matches(tmp_path, monkeypatch):
    src = tmp_path / "k.cu"
    src.write_text(SRC)
    prof = tmp_path / "p.md"
    prof.write_text(f"code-sha256: {bench.code_hash(str(src))}\ntraffic-bytes-per-launch: 123\n")
    monkeypatch.setattr(bench, "PROFILE", str(prof))
    monkeypatch.setattr(bench, "KERNEL_SRC", str(src))
    assert bench.profiled_traffic() == 123.0
    src.write_text(SRC.replace("1.0f", "3.0f"))
    assert bench.profiled_traffic() is None



def test_launch_count_per_step():
    assert bench.launches_per_step(4, 64, 1, 4096 * 4096) == 4      # zero, stream, fixup, dequant
    assert bench.launches_per_step(4, 128, 0, 4096 * 4096) == 4     # G = 131072 fills words
    assert bench.launches_per_step(4, 16, 0, 30 * 32) == 5          # G = 60: byte staging + pack
