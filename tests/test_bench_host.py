"""Host-side pieces of bench.py that need no GPU."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_code_hash_ignores_comments_only(tmp_path):
    src = "__global__ void f(int* p) {  // store\n    p[0] = 1; /* one */\n}\n"
    a = tmp_path / "a.cu"
    a.write_text(src)
    b = tmp_path / "b.cu"
    b.write_text("// header\n" + src.replace("// store", "// writes one"))
    c = tmp_path / "c.cu"
    c.write_text(src.replace("p[0] = 1", "p[0] = 2"))
    assert bench.source_code_sha256(str(a)) == bench.source_code_sha256(str(b))
    assert bench.source_code_sha256(str(a)) != bench.source_code_sha256(str(c))


def test_decode_bytes_match_the_algorithmic_count():
    # state read + write per (sequence, V head) plus the per-token inputs and outputs
    assert bench.decode_bytes(256, 1) == 1_080_098_816
    assert bench.decode_bytes(256, 4) == 1_099_169_792
