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


# --------------------------------------------------------------------------
# bench.py's own control flow under two ranks, the GPU replaced by a stand-in
# --------------------------------------------------------------------------

class _FakeClock:
    t = 0.0


class _FakeEvent:
    def record(self, stream=None):
        self.t = _FakeClock.t

    def elapsed_time(self, other):
        return other.t - self.t


class _FakeRanker:
    """The library calls run_ours makes, each advancing a fake device clock:
    rank r's pass takes 1 + r ms, its host-buffer call 1.5 + r ms."""

    def __init__(self, rank):
        self.rank = rank
        self.n_tokens = 0

    def vid_table_build(self, *a):
        pass

    def embedding_rho(self):
        return 0.02

    def set_graph(self, on):
        pass

    def prepare(self, p, po, b, co, branch_len, mode):
        self.n_tokens = len(p) + len(b)

    def execute(self):
        _FakeClock.t += 1.0 + self.rank

    def sync(self):
        pass

    def score(self, *a, out=None):
        _FakeClock.t += 1.5 + self.rank
        out[:] = 0.0

    def plan_bytes(self):
        return 1000

    def launches_per_execute(self):
        return 142

    def debug_layout(self):
        return np.zeros(self.n_tokens, np.int32), np.zeros(self.n_tokens, np.int32)

    def profile(self, n):
        from shared_prefix_item_b200 import _lib
        return {k: (0.1 * n, 28 * n) for k in _lib.Ranker.PROFILE_CLASSES}

    def close(self):
        pass


class _FakeDevice:
    dist_backend = "gloo"
    tensor_device = "cpu"
    stream = None

    def __init__(self, local_rank):
        self.local_rank = local_rank

    def ranker(self, shape, weights):
        return _FakeRanker(int(os.environ["RANK"]))

    def events(self):
        return _FakeEvent(), _FakeEvent()

    def synchronize(self):
        pass

    def clock_sampler(self):
        import contextlib

        class _C:
            def summary(self):
                return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        return contextlib.nullcontext(_C())


def _bench_main_rank(rank: int, world: int, port: int, out_dir: str) -> None:
    import sys
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update({"RANK": str(rank), "LOCAL_RANK": str(rank), "WORLD_SIZE": str(world),
                       "MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})
    bench.CudaDevice = _FakeDevice
    bench.load_table = lambda rk, n, d: "stand-in table"
    bench.W.model_weights = lambda shape: []
    sys.argv = ["bench.py", "--gpus", str(world), "--steps", "4", "--warmup", "3", "--skip-cpu"]
    with open(os.path.join(out_dir, f"out{rank}.txt"), "w") as f:
        sys.stdout = f
        try:
            bench.main()
        finally:
            sys.stdout.flush()
            sys.stdout = sys.__stdout__


@pytest.mark.slow
def test_bench_main_under_two_ranks_prints_one_combined_line(tmp_path):
    import json
    world = 2
    mp.start_processes(_bench_main_rank, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True,
                       start_method="spawn")
    out0 = (tmp_path / "out0.txt").read_text().strip().splitlines()
    out1 = (tmp_path / "out1.txt").read_text().strip()
    assert out1 == "", "only rank 0 prints"
    assert len(out0) == 1
    line = json.loads(out0[0])
    assert line["n_gpus"] == 2 and line["scaling"] == "weak"
    assert line["config"]["parallelism"] == "dp2"
    # the slowest rank (rank 1: 2 ms a pass, 2.5 ms a host-buffer call)
    # sets the time; both ranks' candidates count
    assert line["ms_per_step"] == pytest.approx(2.0)
    assert line["value"] == pytest.approx(2 * 6400 / 2.0e-3)
    assert line["e2e"]["value"] == pytest.approx(2 * 6400 / 2.5e-3)
    assert line["gpu_launches"] == 142 * 4


def test_gpus_must_match_the_launched_world(monkeypatch):
    import sys
    sys.path.insert(0, ROOT)
    import bench
    monkeypatch.setenv("WORLD_SIZE", "2")
    monkeypatch.setattr(sys, "argv", ["bench.py", "--gpus", "4"])
    with pytest.raises(SystemExit) as e:
        bench.main()
    assert "WORLD_SIZE" in str(e.value)


def test_gpus_without_a_launcher_relaunches_n_ranks(monkeypatch):
    import subprocess
    import sys
    sys.path.insert(0, ROOT)
    import bench
    seen = {}
    monkeypatch.delenv("WORLD_SIZE", raising=False)
    monkeypatch.setattr(subprocess, "call", lambda cmd: seen.setdefault("cmd", cmd) and 0)
    monkeypatch.setattr(sys, "argv", ["bench.py", "--gpus", "4", "--steps", "3"])
    with pytest.raises(SystemExit) as e:
        bench.main()
    assert e.value.code == 0
    cmd = seen["cmd"]
    assert cmd[1:3] == ["-m", "torch.distributed.run"]
    assert "--nproc-per-node=4" in cmd and "--master-addr=127.0.0.1" in cmd
    assert cmd[-4:] == ["--gpus", "4", "--steps", "3"]
