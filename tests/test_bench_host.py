"""Host-side logic of bench.py that needs no GPU: the key that ties a recorded DRAM-traffic
figure to the GEMM sources it was captured on."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402

KERNEL = """// a kernel
#include "x.cuh"
__device__ int f(int a) {  // doubles
  /* block
     comment */
  return 2 * a;
}
"""


def _key(tmp_path, text, name="k.cuh"):
    (tmp_path / name).write_text(text)
    return bench.source_sha16(name, csrc=str(tmp_path))


def test_key_ignores_comments_and_blank_lines(tmp_path):
    base = _key(tmp_path, KERNEL)
    reworded = KERNEL.replace("// a kernel", "// the same kernel, described differently")
    reworded = reworded.replace("/* block\n     comment */", "/* one line */")
    assert _key(tmp_path, reworded) == base
    assert _key(tmp_path, KERNEL.replace("{  // doubles", "{\n\n")) == base


def test_key_follows_the_code(tmp_path):
    base = _key(tmp_path, KERNEL)
    assert _key(tmp_path, KERNEL.replace("2 * a", "3 * a")) != base
    assert _key(tmp_path, KERNEL.replace("int a", "long a")) != base


def test_key_depends_on_every_file_and_its_order(tmp_path):
    (tmp_path / "a.cuh").write_text("int a;\n")
    (tmp_path / "b.cuh").write_text("int b;\n")
    ab = bench.source_sha16("a.cuh", "b.cuh", csrc=str(tmp_path))
    assert ab != bench.source_sha16("b.cuh", "a.cuh", csrc=str(tmp_path))
    assert ab != bench.source_sha16("a.cuh", csrc=str(tmp_path))


def test_recorded_traffic_entries_are_well_formed():
    for (workload, T), rec in bench.GATE_UP_TRAFFIC.items():
        assert isinstance(workload, str) and T > 0
        assert rec["bytes"] > 0 and len(rec["sha16"]) == 16
        int(rec["sha16"], 16)


def test_prefill_traffic_record_is_keyed_on_the_current_gemm_sources():
    # the recorded figure is reported only while the GEMM code it was captured on is unchanged
    rec = bench.traffic_record("k3_prefill_t8192", 8192)
    key = bench.source_sha16(*bench.GEMM_SOURCES)
    stored = bench.GATE_UP_TRAFFIC[("k3_prefill_t8192", 8192)]["sha16"]
    assert (rec is not None) == (key == stored)
    assert bench.traffic_record("k3_decode_t64", 64) is None
