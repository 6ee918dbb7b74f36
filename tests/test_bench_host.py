"""Host logic of bench.py on CPU: the source hash that decides whether a recorded ncu traffic
figure still describes the kernel (comments and spacing do not count, code does), and the
lookup that reports the figure or null."""

import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402

SRC = """// a kernel
__global__ void k(float* x) {  /* body */
  x[threadIdx.x] *= 2.f;
}
"""


def _write(tmp_path, name, text):
    p = tmp_path / name
    p.write_text(text, encoding="utf-8")
    return str(p)


def test_hash_ignores_comments_and_spacing(tmp_path):
    a = _write(tmp_path, "a.cu", SRC)
    b = _write(tmp_path, "b.cu", SRC.replace("// a kernel", "// the same kernel, new comment")
               .replace("/* body */", "/* another\n   block comment */").replace("  x[", "\tx["))
    assert bench.kernel_source_hash([a]) == bench.kernel_source_hash([b])


def test_hash_changes_with_code(tmp_path):
    a = _write(tmp_path, "a.cu", SRC)
    c = _write(tmp_path, "c.cu", SRC.replace("2.f", "3.f"))
    assert bench.kernel_source_hash([a]) != bench.kernel_source_hash([c])


def test_hash_covers_every_file_in_order(tmp_path):
    a = _write(tmp_path, "a.cu", SRC)
    d = _write(tmp_path, "d.h", "#define N 4\n")
    assert bench.kernel_source_hash([a, d]) != bench.kernel_source_hash([a])
    assert bench.kernel_source_hash([a, d]) != bench.kernel_source_hash([d, a])


def test_traffic_reported_only_while_the_sources_match(tmp_path):
    a = _write(tmp_path, "a.cu", SRC)
    rec = {"sources": [a], "sha256": bench.kernel_source_hash([a]), "bytes": 12345}
    assert bench.decode_traffic(rec) == 12345
    with open(a, "a", encoding="utf-8") as fh:
        fh.write("__device__ int extra;\n")
    assert bench.decode_traffic(rec) is None


def test_traffic_null_when_a_source_is_missing(tmp_path):
    rec = {"sources": [str(tmp_path / "gone.cu")], "sha256": "0" * 64, "bytes": 1}
    assert bench.decode_traffic(rec) is None


def test_recorded_captures_name_existing_sources():
    for rec in (bench.DECODE_TRAFFIC, bench.SERVING_TRAFFIC, bench.ENCODE_TRAFFIC):
        for f in rec["sources"]:
            assert os.path.isfile(os.path.join(ROOT, f)), f
        assert len(rec["sha256"]) == 64 and rec["bytes"] > 0
