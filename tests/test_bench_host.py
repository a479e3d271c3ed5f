"""Host-side logic of bench.py that needs no GPU."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_kernel_code_text_ignores_comments_but_not_code():
    a = "int f(int x) {  // doubles\n  return 2 * x; /* fast */\n}\n"
    b = "// a comment added\nint f(int x) {\n    return 2 * x;\n}\n"
    c = "int f(int x) {\n  return 3 * x;\n}\n"
    assert bench.code_text(a) == bench.code_text(b)
    assert bench.code_text(a) != bench.code_text(c)


def test_traffic_entries_match_the_current_kernel_sources():
    # every committed ncu traffic figure names the kernel code it was taken on;
    # bench.py reports it only while the code is unchanged
    import json
    with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
        t = json.load(f)
    for cfg, kinds in t.items():
        for kind, e in kinds.items():
            assert kind in bench.KERNEL_SOURCES
            assert e["dram_bytes_per_launch"] > 0
            got = bench.captured_traffic(kind, cfg)
            assert got is None or got == e["dram_bytes_per_launch"]
