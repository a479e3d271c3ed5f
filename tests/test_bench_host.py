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


def test_open_loop_server_serves_every_request_in_arrival_order():
    import time

    import numpy as np

    class FakeRanker:  # a call takes 2 ms plus 0.1 ms per request
        def __init__(self):
            self.batches = []

        def score(self, prefix, poff, branch, coff, b):
            self.batches.append(len(poff) - 1)
            time.sleep(0.002 + 0.0001 * (len(poff) - 1))

    n = 60
    packed = [(np.arange(5, dtype=np.int32), np.arange(3, dtype=np.int32), 3) for _ in range(n)]
    arrive = np.cumsum(np.full(n, 0.0005))  # faster than the server: batches form
    rk = FakeRanker()
    lat = bench.open_loop_run(rk, packed, arrive, cap=8)
    assert len(lat) == n and np.all(lat > 0)
    assert sum(rk.batches) == n and max(rk.batches) <= 8 and max(rk.batches) > 1
