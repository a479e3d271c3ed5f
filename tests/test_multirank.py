"""The N-GPU path of bench.py on CPU: two gloo ranks, no GPU.

Requests shard across ranks (every rank scores an independent batch of the
same recipe, weak scaling, no collective on the data path); the only
collectives are the two reductions that turn per-rank figures into the
whole-job line: the slowest rank's time and the total units scored.
"""
import hashlib
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _digest(wl) -> str:
    h = hashlib.sha256()
    for a in wl.packed():
        h.update(np.ascontiguousarray(a).tobytes())
    return h.hexdigest()


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, world: int, port: int, out_dir: str) -> None:
    import datetime
    import json
    import sys

    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        wl = bench.workload("c64", rank)
        ms_local = 5.0 + 3.0 * rank
        ms_max, total = bench.combine_ranks(dist, ms_local, wl.n_candidates, "cpu")
        digests = [None] * world
        dist.all_gather_object(digests, _digest(wl))
        with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
            json.dump({"ms_max": ms_max, "total": total, "n_cand": wl.n_candidates, "digests": digests}, f)
    finally:
        dist.destroy_process_group()


@pytest.mark.slow
def test_two_gloo_ranks_shard_requests_and_combine(tmp_path):
    import json
    world = 2
    mp.start_processes(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True,
                       start_method="spawn")
    res = [json.load(open(tmp_path / f"rank{r}.json")) for r in range(world)]

    import sys
    sys.path.insert(0, ROOT)
    import bench
    for r in range(world):
        # the slowest rank's time, the units of all ranks
        assert res[r]["ms_max"] == 8.0
        assert res[r]["total"] == sum(x["n_cand"] for x in res) == world * 6400
        # every rank saw the same gathered list
        assert res[r]["digests"] == res[0]["digests"]
    d = res[0]["digests"]
    assert len(set(d)) == world, "ranks scored the same requests"
    # a rank's shard does not depend on the world size or on the process
    for r in range(world):
        assert d[r] == _digest(bench.workload("c64", r))
    assert d[0] == _digest(bench.workload("c64", 0)) and d[1] != _digest(bench.workload("c64", 0))


def test_single_rank_combine_is_identity():
    import sys
    sys.path.insert(0, ROOT)
    import bench
    assert bench.combine_ranks(None, 12.5, 6400, "cpu") == (12.5, 6400)


def test_reference_arm_other_ranks_do_no_work(capsys):
    import sys
    sys.path.insert(0, ROOT)
    import bench

    class Args:  # any access to an argument would mean the rank did work
        def __getattr__(self, k):
            raise AssertionError(f"rank 1 read --{k}")
    bench.run_reference(Args(), 1, 2)
    assert capsys.readouterr().out == ""

