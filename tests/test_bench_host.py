"""Host-side pieces of bench.py that need no GPU: the code-only source hash that keys the DRAM
counters in profiles/traffic.json, and the clock sampler without NVML."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402

SRC = """// header comment
#include <x.h>
/* a block
   comment */
int f(int a) {   // trailing comment
    return a + 1;

}
"""


def test_code_only_drops_comments_and_blank_lines():
    assert bench.code_only(SRC) == "#include <x.h>\nint f(int a) {\n    return a + 1;\n}"


def test_comment_edits_keep_the_code_and_code_edits_change_it():
    reworded = SRC.replace("trailing comment", "another remark").replace("a block", "one more block")
    assert bench.code_only(reworded) == bench.code_only(SRC)
    assert bench.code_only(SRC.replace("a + 1", "a + 2")) != bench.code_only(SRC)


def test_source_hash_is_stable_and_covers_the_gemm_sources():
    assert set(bench.GEMM_SOURCES) == {"fp8q.cu", "gemm.cuh", "ptx.cuh"}
    h = bench.source_hash()
    assert h == bench.source_hash() and len(h) == 16


def test_clock_sampler_without_nvml_reports_unavailable():
    s = bench.ClockSampler(0)
    s._nvml = None            # as on a host without the NVIDIA management library
    with s:
        pass
    assert s.summary(10)["reasons"] == ["unavailable"]
