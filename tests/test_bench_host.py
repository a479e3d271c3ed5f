"""Host-side logic of bench.py that needs no GPU."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import bench  # noqa: E402
from synth import workloads as W  # noqa: E402


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


def test_reuse_batches_rebuild_the_full_prefixes():
    import bench
    wl = W.c64(n_requests=12)
    p, po, b, co = wl.packed()
    for kind in ("append", "rescore"):
        ru = bench.Reuse(wl, kind)
        warm_ids, warm_off, _, _, _, slots, zeros, warm_keep = ru.warm
        new_ids, new_off, b2, co2, bl, slots2, cached, keep = ru.step
        assert np.array_equal(b2, b) and np.array_equal(co2, co) and bl == wl.branch_len
        assert list(warm_keep) == list(cached) and not np.any(zeros)
        for q, r in enumerate(wl.requests):
            full = np.concatenate([warm_ids[warm_off[q]:warm_off[q + 1]], new_ids[new_off[q]:new_off[q + 1]]])
            assert np.array_equal(full, r.prefix_ids)
            assert 0 <= keep[q] <= new_off[q + 1] - new_off[q]
            assert cached[q] + keep[q] <= ru.slot_tokens
        if kind == "append":
            # the new tokens are the last history item (marker, VID, feedback) and the header, kept but the header
            for q, r in enumerate(wl.requests):
                assert keep[q] == 2 + len(r.feedback[-1])
                assert new_ids[new_off[q]] == wl.template.marker
        else:
            assert new_off[-1] == 0 and not any(keep)


def test_attention_pairs_with_cached_prefixes():
    import bench
    wl = W.c64(n_requests=5)
    full = bench.attention_pairs(wl, False)
    assert bench.attention_pairs(wl, False, [0] * 5) == full
    # everything cached: only the branch queries remain
    assert bench.attention_pairs(wl, False, [r.L for r in wl.requests]) == sum(r.K * (r.L + 1) for r in wl.requests)
    c = [3] * 5
    assert full - bench.attention_pairs(wl, False, c) == 5 * (1 + 2 + 3)
