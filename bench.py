"""Throughput of the DuoLM multi-item-scoring ranker: candidate scores/s.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--config c64|c1|stress|catalog-c64|catalog-c8|catalog-c1]
                    [--mode mis|independent] [--reuse append|rescore|template] [--no-graph] [--skip-cpu]
                    [--profile-steps N]

One step is one pass of the whole hot path (virtual-id gather, 28 decoder
layers with shared-prefix tree-masked attention, score head) over one batch
of synthetic requests.  Default workload: 64 ragged requests of the
Qwen3-0.6B-shaped ranker with K = 100 candidates each (the configuration the
pages' headline throughput is quoted on).  Under torchrun every rank scores
its own batch of the same recipe (requests are independent: weak scaling,
no data-path collective); the time is the max over ranks.

Prints one JSON line (rank 0).  `value` times device-resident batches
(duolm_execute replays of the prepared batch); `e2e` times duolm_score from
host buffers (validation, packing, host->device copy, pass, scores back).
`--impl reference` times the oracle (plain fp64 CPU code) on the host cores
instead, one request of the same workload per step.

`--reuse` runs the same requests from a prefix KV store: `append` stores each
request's prefix up to its last history item beforehand, and every step
appends that item and the header (the new history arrives) before scoring;
`rescore` stores the whole prefix and every step scores the K candidates
only; `template` stores the instruction every prompt starts with in one
slot that all requests read.  The scores are those of the full sequences in
every case.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time
from typing import Optional

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

from synth import workloads as W  # noqa: E402
from synth.rng import Stream  # noqa: E402

METRIC = "candidate scores/sec on 1 B200 (Qwen3-0.6B shape, K=100) + % of roofline"
UNIT = "candidate scores/s"
# the pages' figures for this metric (1x H100, 100 candidates per request; context, not targets)
PAGES_CAND_PER_S = {("c64", "mis"): 26404.0, ("c1", "mis"): 8870.0, ("c64", "independent"): 851.48}


def workload(name: str, shard: int) -> W.Workload:
    if name == "c64":
        return W.c64(shard=shard)
    if name == "c1":
        return W.c1(shard=shard)
    if name == "stress":
        return W.stress(shard=shard)
    if name.startswith("fir-m"):
        return W.fir(int(name[len("fir-m"):]), shard=shard)
    if name.startswith("catalog-c"):
        return W.catalog(int(name[len("catalog-c"):]), shard=shard)
    raise SystemExit(f"unknown config {name}")


def combine_ranks(dist, ms: float, units: int, device) -> tuple:
    """Whole-job figures from one rank's own: the slowest rank's time (every
    rank scores its own shard, so the job ends when the last one does) and
    the units scored by all ranks together.  ``dist`` is None on one rank."""
    import torch
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    u = torch.tensor([units], dtype=torch.int64, device=device)
    if dist is not None:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        dist.all_reduce(u, op=dist.ReduceOp.SUM)
    return float(t.item()), int(u.item())


def describe(wl: W.Workload, mode: str, graph: bool, n: int) -> dict:
    Ls = [r.L for r in wl.requests]
    return {
        "workload": f"{wl.name}: {len(wl.requests)} requests x K={wl.requests[0].K} candidates, "
                    f"b={wl.branch_len}, Qwen3-0.6B-shaped ranker, {wl.n_items}-item FP16 table",
        "requests_per_gpu": len(wl.requests),
        "candidates_per_gpu": wl.n_candidates,
        "tokens_per_gpu": wl.n_tokens,
        "prefix_len_mean": round(float(np.mean(Ls)), 1),
        "mode": mode,
        "cuda_graph": graph,
        "parallelism": f"dp{n}",
        "weights": "bf16 values, stored exactly as fp16 x 2^s",
        "l2": "no flush: the step's working set (0.88 GB weights + activations) exceeds the 126 MB L2",
    }


# ---------------------------------------------------------------------------
# algorithmic work per step
# ---------------------------------------------------------------------------

def gemm_flops(shape: W.ModelShape, T: int) -> float:
    d, qd, kd, F = shape.d, shape.q_dim, shape.kv_dim, shape.ffn
    return 2.0 * T * (d * (qd + 2 * kd) + qd * d + d * 2 * F + F * d) * shape.n_layers


def attention_pairs(wl: W.Workload, independent: bool, cached=None) -> int:
    """(query, key) pairs of one pass; with cached[q] prefix tokens of request
    q already stored, only the queries after them are computed."""
    b = wl.branch_len
    tot = 0
    for q, r in enumerate(wl.requests):
        L, K = r.L, r.K
        c = cached[q] if cached is not None else 0
        if independent:
            tot += K * (L + b) * (L + b + 1) // 2
        else:
            tot += (L * (L + 1) - c * (c + 1)) // 2 + K * sum(L + i + 1 for i in range(b))
    return tot


def attention_flops(shape: W.ModelShape, wl: W.Workload, independent: bool, cached=None) -> float:
    # QK^T and PV: 2 * head_dim each per (query, key) pair and query head
    return 4.0 * shape.head_dim * shape.n_q_heads * attention_pairs(wl, independent, cached) * shape.n_layers


class Reuse:
    """Arguments of the prefix-reuse runs: `warm` fills the store (request q
    in slot q), `step` is the batch every timed step runs."""

    def __init__(self, wl: W.Workload, kind: str):
        R = len(wl.requests)
        n_header = len(wl.template.header)
        p, po, b, co = wl.packed()
        if kind == "append":
            # everything before the last history item
            self.cached = [wl.history_offsets(q)[-1] for q in range(R)]
            keep = [r.L - c - n_header for r, c in zip(wl.requests, self.cached)]
        elif kind == "rescore":
            self.cached = [r.L for r in wl.requests]
            keep = [0] * R
        elif kind == "template":
            # one slot holds the instruction every prompt starts with; every
            # request reads it (exact cross-request reuse of a common prefix)
            n_instr = len(wl.template.instr)
            assert all(np.array_equal(r.prefix_ids[:n_instr], wl.template.instr) for r in wl.requests)
            self.cached = [n_instr] * R
            keep = [0] * R
            r0 = wl.requests[0]
            self.slot_tokens = n_instr
            self.warm = (np.asarray(wl.template.instr, np.int32), np.array([0, n_instr]), r0.branch_ids.reshape(-1),
                         np.array([0, r0.K]), wl.branch_len, np.array([0]), np.zeros(1), np.array([n_instr]))
            new_ids = np.concatenate([r.prefix_ids[n_instr:] for r in wl.requests])
            new_off = np.cumsum([0] + [r.L - n_instr for r in wl.requests])
            self.step = (new_ids, new_off, b, co, wl.branch_len, np.zeros(R, np.int64), self.cached, keep)
            self.n_slots = 1
            self.note = (f"template: the {n_instr}-token instruction of every request read from one shared KV slot, "
                         f"{int(new_off[-1])} new prefix tokens per step")
            return
        else:
            raise SystemExit(f"unknown --reuse {kind}")
        self.n_slots = R
        warm_ids = np.concatenate([r.prefix_ids[:c] for r, c in zip(wl.requests, self.cached)])
        warm_off = np.cumsum([0] + self.cached)
        new_ids = np.concatenate([r.prefix_ids[c:] for r, c in zip(wl.requests, self.cached)])
        new_off = np.cumsum([0] + [r.L - c for r, c in zip(wl.requests, self.cached)])
        slots = np.arange(R)
        self.slot_tokens = max(r.L for r in wl.requests)
        self.warm = (warm_ids, warm_off, b, co, wl.branch_len, slots, np.zeros(R), self.cached)
        self.step = (new_ids, new_off, b, co, wl.branch_len, slots, self.cached, keep)
        self.note = (f"{kind}: {sum(self.cached)} of {sum(r.L for r in wl.requests)} prefix tokens read from "
                     f"the KV store, {int(new_off[-1])} new prefix tokens per step")


def class_flops(shape: W.ModelShape, wl: W.Workload, T: int, independent: bool, cached=None) -> dict:
    """Algorithmic FLOPs per step of each kernel class (multiply-add = 2)."""
    d, qd, kd, F, L = shape.d, shape.q_dim, shape.kv_dim, shape.ffn, shape.n_layers
    return {
        "gemm_qkv": 2.0 * T * d * (qd + 2 * kd) * L,
        "gemm_o": 2.0 * T * qd * d * L,
        "gemm_gate_up": 2.0 * T * d * 2 * F * L,
        "gemm_down": 2.0 * T * F * d * L,
        "attention": attention_flops(shape, wl, independent, cached),
    }


KERNEL_SOURCES = {  # the files a kernel class is built from (its ncu traffic is stale once they change)
    "gemm_qkv": ("gemm_tc.cu", "common.cuh"), "gemm_o": ("gemm_tc.cu", "common.cuh"),
    "gemm_gate_up": ("gemm_tc.cu", "common.cuh"), "gemm_down": ("gemm_tc.cu", "common.cuh"),
    "attention": ("attention_tc.cu", "common.cuh"),
}


def code_text(src: str) -> str:
    """The code of a C++/CUDA source without its comments and with
    whitespace collapsed (an edit to a comment does not change a kernel)."""
    import re
    src = re.sub(r"/\*.*?\*/", " ", src, flags=re.S)
    src = re.sub(r"//[^\n]*", " ", src)
    return " ".join(src.split())


def source_hash(kind: str) -> str:
    import hashlib
    h = hashlib.sha256()
    for f in KERNEL_SOURCES[kind]:
        with open(os.path.join(ROOT, "shared_prefix_item_b200", "csrc", f), encoding="utf-8") as fh:
            h.update(code_text(fh.read()).encode())
    return h.hexdigest()[:16]


def captured_traffic(kind: str, config: str):
    """DRAM bytes per launch (read + write) of a kernel class from the committed
    ncu summary, or None when there is none for this workload or the kernel's
    sources changed since it was taken."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        t = json.load(f).get(config, {}).get(kind)
    if not t or t.get("source_hash") != source_hash(kind):
        return None
    return t["dram_bytes_per_launch"]


def attention_bytes(shape: W.ModelShape, T: int) -> float:
    # q read, k and v read once, o written (fp16), per layer
    return 2.0 * T * (2 * shape.q_dim + 2 * shape.kv_dim) * shape.n_layers


def peaks() -> dict:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            m = json.load(f)
        return {"hbm": m["hbm_gbs"], "tc": m["bf16_tflops"], "tc_sustained": m["bf16_tflops_sustained"],
                "src": "measured"}
    return {"hbm": 6650.0, "tc": 1590.0, "tc_sustained": 1400.0, "src": "fallback"}


# ---------------------------------------------------------------------------
# clocks during the timed region
# ---------------------------------------------------------------------------

class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.gpu_id = gpu_id
        self.rows = []
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.gpu_id, f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.rows.append([c.strip() for c in line.split(",")])

    def __exit__(self, *a):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self) -> dict:
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in self.rows:
            try:
                sm.append(float(r[0]))
                mx = float(r[1])
                for n, v in zip(names, r[3:7]):
                    if v.lower() == "active":
                        reasons.add(n)
            except (ValueError, IndexError):
                continue
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        loaded = [v for v in sm if v > 0.5 * (mx or max(sm))] or sm
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ---------------------------------------------------------------------------
# CPU oracle timing
# ---------------------------------------------------------------------------

def oracle_time(wl: W.Workload, requests, warmup: int = 1, independent_cands: int = 0,
                budget_s: float = 0.0) -> tuple:
    """Score the given requests with the oracle; returns (seconds per request,
    candidates).  `warmup` short calls first load the library and page in the
    weights.  With independent_cands > 0, only that many candidates of each
    request are scored, in independent mode (each candidate's whole prefix +
    branch sequence on its own).  With budget_s > 0 the requests are taken in
    order until that much time has been spent (at least one)."""
    from oracle import ranker as R
    om = R.OracleModel(wl.model, W.model_weights(wl.model))
    rho = R.embedding_rho(om.embed)
    a = W.item_vectors(wl.n_items, wl.model.d)
    rows = set()
    for q in requests:
        r = wl.requests[q]
        for i in np.concatenate([r.prefix_ids, r.branch_ids.reshape(-1)]):
            if i >= wl.model.vocab:
                rows.add(int(i) - wl.model.vocab)
    rows = np.array(sorted(rows), np.int64)
    sub = R.table_f32(R.interface(a[rows], 0.0, rho))
    remap = {int(r): i for i, r in enumerate(rows)}

    def rm(ids):
        return np.array([i if i < wl.model.vocab else wl.model.vocab + remap[int(i) - wl.model.vocab]
                         for i in ids.reshape(-1)], np.int32).reshape(ids.shape)

    local = [W.Request(rm(wl.requests[q].prefix_ids), rm(wl.requests[q].branch_ids)) for q in requests]
    if independent_cands:
        local = [W.Request(r.prefix_ids, r.branch_ids[:independent_cands]) for r in local]
    score = R.score_independent if independent_cands else R.score_mis
    for _ in range(max(1, warmup)):
        R.score_mis(om, sub, W.Request(local[0].prefix_ids[:4], local[0].branch_ids[:1]))
    per = []
    n = 0
    for req in local:
        t = time.perf_counter()
        score(om, sub, req)
        per.append(time.perf_counter() - t)
        n += req.K
        if budget_s and sum(per) >= budget_s:
            break
    return per, n


def compile_rate(wl: W.Workload, reps: int = 20) -> Optional[dict]:
    """Host request compilation (duolm_compile) of the whole batch from its
    records, on all host threads and on one: requests/s and candidates/s."""
    import shared_prefix_item_b200 as S
    if wl.template is None:
        return None
    t = wl.template
    hist, hoff, fb, foff, cand, coff = wl.records()
    out = {}
    for label, nt in [("all_threads", 0), ("one_thread", 1)]:
        def once():
            return S.compile_requests(wl.model.vocab, t.marker, wl.m, t.instr, t.header,
                                      t.branch_header[: wl.branch_len - wl.m], hist, hoff, fb, foff, cand, coff,
                                      wl.n_items // wl.m, nt)
        once()
        t0 = time.perf_counter()
        for _ in range(reps):
            once()
        sec = (time.perf_counter() - t0) / reps
        out[label] = {"us_per_batch": round(sec * 1e6, 1), "requests_per_s": round(len(wl.requests) / sec),
                      "cand_per_s": round(wl.n_candidates / sec)}
    out["threads"] = os.cpu_count()
    out["note"] = "records (item ids, feedback tokens) to packed ids, output arrays included; not in the timed step"
    return out


def cpu_count() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


# ---------------------------------------------------------------------------

def run_reference(args, rank: int, world: int) -> None:
    if rank != 0:
        return
    wl = workload(args.config, 0)
    steps, warm = args.steps, args.warmup
    n_req = len(wl.requests)
    order = [i % n_req for i in range(steps)]
    per, _ = oracle_time(wl, order, warmup=warm)
    cands = sum(wl.requests[q].K for q in order)
    total = sum(per)
    value = cands / total
    sample = (f"{steps} timed steps, step i = request i of the {wl.name} batch (all its candidates) scored by "
              f"the oracle's packed layout; {warm} warm-up calls on a 4-token slice of request 0")
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": steps, "warmup": warm,
        "ms_per_step": 1e3 * total / steps, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f64", "data": "synthetic", "impl": "reference",
        "config": describe(wl, args.mode, False, world),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cpu_count(), "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


TABLE_BUILD_ROWS = 100_000


def load_table(rk, n_rows: int, d: int) -> str:
    """The item table of a workload: built through the library's interface
    kernel from the seeded item vectors; above TABLE_BUILD_ROWS rows the first
    TABLE_BUILD_ROWS are built and tiled (the values do not affect the
    timing, and generating millions of vectors on the host takes minutes).
    Returns a note for the config."""
    base = min(n_rows, TABLE_BUILD_ROWS)
    rk.vid_table_build(W.item_vectors(base, d), 0.0, rk.embedding_rho())
    if base == n_rows:
        return f"{n_rows} rows from the seeded item vectors"
    reps = -(-n_rows // base)
    rk.vid_table_load(np.tile(rk.debug_table(base), (reps, 1))[:n_rows])
    return f"{n_rows} rows: {base} from the seeded item vectors, tiled"


GATHER_LOOKUPS = 4_194_304
GATHER_TABLE_ROWS = 1_000_000


def run_gather(args, rank: int, world: int, local_rank: int) -> None:
    """The VID gather alone (duolm_gather): GATHER_LOOKUPS Zipf(1.1) lookups
    over a GATHER_TABLE_ROWS-row FP16 item table, each writing the fp32 row,
    its fp16 normed operand and its sum of squares; HBM bound."""
    import torch

    import shared_prefix_item_b200 as S
    torch.cuda.set_device(local_rank)
    shape = W.QWEN3_06B
    stream = torch.cuda.Stream()
    torch.cuda.set_stream(stream)
    rk = S.Ranker(shape, W.model_weights(shape), device=local_rank, stream=stream.cuda_stream)
    load_table(rk, GATHER_TABLE_ROWS, shape.d)
    n, d = GATHER_LOOKUPS, shape.d
    ids = torch.from_numpy((shape.vocab + W.zipf_lookups(n, GATHER_TABLE_ROWS)).astype(np.int32)).cuda()
    x = torch.empty((n, d), dtype=torch.float32, device="cuda")
    xg = torch.empty((n, d), dtype=torch.int16, device="cuda")
    ssp = torch.empty((n, d // 64), dtype=torch.float32, device="cuda")

    def step():
        rk.gather(ids.data_ptr(), n, x.data_ptr(), xg.data_ptr(), ssp.data_ptr())

    for _ in range(args.warmup):
        step()
    rk.sync()
    props = torch.cuda.get_device_properties(local_rank)
    gpu_id = f"GPU-{props.uuid}" if getattr(props, "uuid", None) else str(local_rank)
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(gpu_id) as clk:
        torch.cuda.synchronize()
        start.record(stream)
        for _ in range(args.steps):
            step()
        end.record(stream)
        torch.cuda.synchronize()
    rk.sync()
    ms = start.elapsed_time(end) / args.steps
    pk = peaks()
    bytes_per = 2 * d + 4 * d + 2 * d + 4 * (d // 64)  # fp16 row read; fp32 x, fp16 x g, sums written
    gbs = n * bytes_per / (ms / 1e3) / 1e9
    if rank == 0:
        print(json.dumps({
            "metric": "VID gather lookups/s (standalone, Zipf(1.1) over a 1M-row FP16 table)",
            "value": n / (ms / 1e3), "unit": "lookups/s", "n_gpus": 1, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f16", "data": "synthetic",
            "config": {"workload": f"gather: {n} lookups, Zipf(1.1) over {GATHER_TABLE_ROWS} rows x {d} fp16",
                       "bytes_per_lookup": bytes_per, "l2": "no flush: 2 GB table, 27 GB written per step"},
            "e2e": None,
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": pk["hbm"], "unit": "GB/s",
                         "frac": gbs / pk["hbm"], "traffic": None,
                         "kernel": "embed_gain_kernel (through duolm_gather)",
                         "peak_note": f"{pk['src']} copy bandwidth"},
            "gpu_launches": args.steps,
            "clocks": clk.summary(),
            "cpu_baseline": None,
        }), flush=True)
    rk.close()


LATENCY_CALLS = {1: 200, 8: 100, 64: 40}
OPEN_LOOP_REQUESTS = 1024
SEED_OPEN_LOOP = 7007


def open_loop_run(rk, packed, arrive_s, cap: int) -> np.ndarray:
    """Serve requests that arrive at the given times (seconds from start):
    each call takes every request that has arrived and is not yet served, at
    most `cap`, scores them through duolm_score and completes them together.
    Returns each request's latency (completion - arrival) in ms."""
    n = len(packed)
    done = np.zeros(n)
    t0 = time.perf_counter()
    i = 0
    while i < n:
        now = time.perf_counter() - t0
        if arrive_s[i] > now:
            time.sleep(arrive_s[i] - now)
            now = time.perf_counter() - t0
        j = i
        while j < n and j - i < cap and arrive_s[j] <= now:
            j += 1
        batch = packed[i:j]
        prefix = np.concatenate([p for p, _, _ in batch]).astype(np.int32)
        poff = np.concatenate([[0], np.cumsum([len(p) for p, _, _ in batch])]).astype(np.int64)
        branch = np.concatenate([b for _, b, _ in batch]).astype(np.int32)
        coff = np.concatenate([[0], np.cumsum([k for _, _, k in batch])]).astype(np.int64)
        rk.score(prefix, poff, branch, coff, 1)
        done[i:j] = time.perf_counter() - t0
        i = j
    return (done - arrive_s) * 1e3


def run_latency(args, rank: int, world: int, local_rank: int) -> None:
    """Latency of the public call.  Closed loop: for C in {1, 8, 64}, each
    call scores a fresh batch of C requests of the 64-request recipe from
    host buffers (duolm_score: validation, packing, host->device plan copy,
    the pass, scores back), timed on the host clock around the blocking call;
    p50/p99 over the calls, with the CUDA graph on and off.  Open loop:
    requests arrive as a Poisson stream at 50% and 90% of the closed-loop
    capacity at C, and a server loop scores whatever has arrived (at most C
    per call); p50/p99 of each request's arrival-to-completion time."""
    import torch

    import shared_prefix_item_b200 as S
    torch.cuda.set_device(local_rank)
    shape = W.QWEN3_06B
    rk = S.Ranker(shape, W.model_weights(shape), device=local_rank)
    table_note = load_table(rk, 100_000, shape.d)
    out = {}
    capacity = {}
    for C, n_calls in LATENCY_CALLS.items():
        batches = [W.c64(n_requests=C, shard=1000 + i).packed() for i in range(n_calls)]
        rk.reserve(max(int(len(b[0]) + len(b[2])) for b in batches), C, C * 100)
        res = {}
        for graph in (True, False):
            rk.set_graph(graph)
            for b in batches[:3]:  # warm-up (graph capture at this capacity)
                rk.score(b[0], b[1], b[2], b[3], 1)
            t = []
            for b in batches:
                t0 = time.perf_counter()
                rk.score(b[0], b[1], b[2], b[3], 1)
                t.append((time.perf_counter() - t0) * 1e3)
            t = np.array(t)
            res["graph" if graph else "eager"] = {"p50_ms": float(np.percentile(t, 50)),
                                                  "p99_ms": float(np.percentile(t, 99)),
                                                  "mean_ms": float(t.mean()), "calls": n_calls}
            if graph:
                capacity[C] = C / (float(np.median(t)) / 1e3)  # requests/s when every call is full
        out[f"C={C}"] = res
    # open loop: Poisson arrivals; the server scores whatever has arrived
    # (at most C requests) each call, one call at a time
    pool = W.c64(n_requests=OPEN_LOOP_REQUESTS, shard=2000).requests
    packed = [(r.prefix_ids, r.branch_ids.reshape(-1), r.K) for r in pool]
    arrivals_u = Stream(SEED_OPEN_LOOP, 0).uniform(OPEN_LOOP_REQUESTS)
    sizes = sorted((len(p) + len(b) for p, b, _ in packed), reverse=True)
    rk.reserve(sum(sizes[:64]), 64, 64 * 100)  # any batch fits: no growth (and no re-capture) mid-run
    open_loop = {}
    for C in LATENCY_CALLS:
        for load in (0.5, 0.9):
            rate = load * capacity[C]
            gaps = -np.log1p(-arrivals_u) / rate  # exponential inter-arrival times
            for graph in (True, False):
                rk.set_graph(graph)
                lat = open_loop_run(rk, packed, np.cumsum(gaps), C)
                open_loop[f"C={C} load={load} {'graph' if graph else 'eager'}"] = {
                    "rate_req_per_s": rate, "p50_ms": float(np.percentile(lat, 50)),
                    "p99_ms": float(np.percentile(lat, 99)), "requests": len(lat)}
    if rank == 0:
        print(json.dumps({
            "metric": "per-call latency of duolm_score, closed loop (p99, C=64, graph)",
            "value": out["C=64"]["graph"]["p99_ms"], "unit": "ms", "n_gpus": 1, "steps": None,
            "warmup": 3, "higher_is_better": False, "scaling": None, "vs_baseline": None, "dtype": "f16",
            "data": "synthetic",
            "config": {"workload": "fresh batches of C requests of the 64-request recipe (K=100, b=1) per call",
                       "table": table_note, "timing": "host clock around the blocking call"},
            "latency": out,
            "open_loop": open_loop,
        }), flush=True)
    rk.close()


class CudaDevice:
    """What run_ours needs from this rank's GPU: the library's context on
    it, the stream the library launches on (the CUDA events are recorded on
    it), a device synchronise, the process-group backend and the clock
    sampler.  The multi-rank CPU test passes a stand-in with the same
    methods, so that the control flow under N ranks runs without a GPU."""
    dist_backend = "nccl"
    tensor_device = "cuda"

    def __init__(self, local_rank: int):
        import torch
        torch.cuda.set_device(local_rank)
        self.torch = torch
        self.local_rank = local_rank
        self.stream = torch.cuda.Stream()
        torch.cuda.set_stream(self.stream)

    def ranker(self, shape, weights):
        import shared_prefix_item_b200 as S
        return S.Ranker(shape, weights, device=self.local_rank, stream=self.stream.cuda_stream)

    def events(self):
        E = self.torch.cuda.Event
        return E(enable_timing=True), E(enable_timing=True)

    def synchronize(self):
        self.torch.cuda.synchronize()

    def clock_sampler(self):
        props = self.torch.cuda.get_device_properties(self.local_rank)
        gpu_id = f"GPU-{props.uuid}" if getattr(props, "uuid", None) else str(self.local_rank)
        return ClockSampler(gpu_id)


def run_ours(args, rank: int, world: int, local_rank: int, dev=None) -> None:
    import shared_prefix_item_b200 as S

    dev = dev or CudaDevice(local_rank)
    dist = None
    if world > 1:
        import datetime

        import torch.distributed as dist
        dist.init_process_group(dev.dist_backend, timeout=datetime.timedelta(seconds=300))

    wl = workload(args.config, rank)
    shape = wl.model
    mode = S.MODE_INDEPENDENT if args.mode == "independent" else S.MODE_MIS
    # the library launches on dev.stream; the events below are recorded on it
    stream = dev.stream
    rk = dev.ranker(shape, W.model_weights(shape))
    table_note = load_table(rk, wl.n_items, shape.d)
    rk.set_graph(not args.no_graph)
    p, po, b, co = wl.packed()
    reuse = None
    if args.reuse:
        if mode != S.MODE_MIS:
            raise SystemExit("--reuse needs --mode mis")
        reuse = Reuse(wl, args.reuse)
        rk.kv_store_reserve(reuse.n_slots, reuse.slot_tokens)
        rk.score_cached(*reuse.warm)

        def prepare():
            rk.prepare_cached(*reuse.step)

        def score_host(out):
            rk.score_cached(*reuse.step, out=out)
    else:
        def prepare():
            rk.prepare(p, po, b, co, wl.branch_len, mode)

        def score_host(out):
            rk.score(p, po, b, co, wl.branch_len, mode, out=out)
    prepare()
    n_cand = wl.n_candidates
    T = int(rk.debug_layout()[0].shape[0])

    if args.profile_steps:
        # a short run for ncu captures: N passes kernel by kernel, no timing
        rk.set_graph(False)
        for _ in range(args.profile_steps):
            rk.execute()
        rk.sync()
        rk.close()
        return

    for _ in range(args.warmup):
        rk.execute()
    rk.sync()

    def barrier():
        if dist:
            dist.barrier()
        dev.synchronize()

    start, end = dev.events()
    with dev.clock_sampler() as clk:
        barrier()
        start.record(stream)
        for _ in range(args.steps):
            rk.execute()
        end.record(stream)
        barrier()
    rk.sync()
    ms = start.elapsed_time(end) / args.steps
    ms_max, n_total = combine_ranks(dist, ms, n_cand, dev.tensor_device)
    value = n_total / (ms_max / 1e3)
    launches = rk.launches_per_execute()

    # e2e: the public call from host buffers, scores back to the host every step
    out = np.empty(n_cand, np.float32)
    score_host(out)
    h2d = rk.plan_bytes()
    barrier()
    start.record(stream)
    for _ in range(args.steps):
        score_host(out)
    end.record(stream)
    barrier()
    e2e_ms = start.elapsed_time(end) / args.steps
    e2e_max, _ = combine_ranks(dist, e2e_ms, n_cand, dev.tensor_device)
    e2e_value = n_total / (e2e_max / 1e3)

    # per-kernel-class device time (eager launches with an event after each)
    prepare()
    prof = rk.profile(max(2, min(args.steps, 5)))
    steps_prof = max(2, min(args.steps, 5))
    pk = peaks()
    indep = mode == S.MODE_INDEPENDENT
    cf = class_flops(shape, wl, T, indep, reuse.cached if reuse else None)
    gf = sum(v for k, v in cf.items() if k != "attention")
    af = cf["attention"]
    kernels = {k: {"ms_per_step": round(v[0] / steps_prof, 4), "launches_per_step": v[1] // steps_prof}
               for k, v in prof.items()}
    tot_ms = sum(v["ms_per_step"] for v in kernels.values())
    for v in kernels.values():
        v["share"] = round(v["ms_per_step"] / tot_ms, 4) if tot_ms else None
    names = {"gemm_qkv": "gemm_tc_kernel<EpiQkv> (QKV projection, QK-norm, RoPE)",
             "kv_append": "kv_append_kernel (new prefix K/V into the store)",
             "gemm_o": "gemm_tc_kernel<EpiResid> (O projection + residual)",
             "gemm_gate_up": "gemm_tc_kernel<EpiSwiglu> (gate/up projection + SwiGLU)",
             "gemm_down": "gemm_tc_kernel<EpiResid> (down projection + residual)",
             "attention": "attention_tc_kernel (shared-prefix tree attention)"}
    roofs = {}
    for k, fl in cf.items():
        ms_k = prof[k][0] / steps_prof
        n_k = max(prof[k][1] // steps_prof, 1)
        if ms_k <= 0:
            continue
        r = {"bound": "tensor", "achieved": fl / (ms_k / 1e3) / 1e12, "peak": pk["tc_sustained"],
             "unit": "TFLOP/s", "kernel": names[k], "launches_per_step": n_k, "flops_per_launch": fl / n_k,
             "us_per_launch": ms_k * 1e3 / n_k,
             "peak_note": f"{pk['src']} sustained bf16 dense (fp16 runs at the bf16 rate)",
             "traffic": None if reuse else captured_traffic(k, args.config)}
        r["frac"] = r["achieved"] / r["peak"]
        if k == "attention":
            # the kernel's floor is the slower of its FLOPs at the tensor peak
            # and its bytes (q, k, v read, o written) at the HBM peak; report
            # against whichever is larger
            by = attention_bytes(shape, T)
            t_s = ms_k / 1e3
            t_flop = fl / (pk["tc_sustained"] * 1e12)
            t_byte = by / (pk["hbm"] * 1e9)
            r["hbm_gbs_algorithmic"] = by / t_s / 1e9
            r["bytes_per_launch"] = by / n_k
            r["floor_us_per_launch"] = max(t_flop, t_byte) * 1e6 / n_k
            r["tensor_frac"] = r["frac"]
            if t_byte > t_flop:
                r.update({"bound": "hbm", "achieved": by / t_s / 1e9, "peak": pk["hbm"], "unit": "GB/s",
                          "peak_note": f"{pk['src']} HBM copy bandwidth (the byte floor is above the FLOP floor)"})
            r["frac"] = max(t_flop, t_byte) / t_s
            if reuse:
                r["note"] = "K/V read from the store not counted in the algorithmic bytes"
        roofs[k] = r
    dom_key = max(roofs, key=lambda k: prof[k][0])
    dominant = roofs[dom_key]
    step_roof_ms = max((gf + af) / (pk["tc_sustained"] * 1e12), 0.0) * 1e3
    cpu = None
    if rank == 0 and world == 1 and not args.skip_cpu and not reuse:
        per, nc = oracle_time(wl, range(len(wl.requests)), budget_s=12.0)
        per_i, nc_i = oracle_time(wl, [0], independent_cands=4)
        Ls = [wl.requests[q].L for q in range(len(per))]
        cpu = {"value": nc / sum(per), "unit": UNIT, "cores": cpu_count(), "kind": "oracle",
               "sample": f"the first {len(per)} requests of the {wl.name} batch (L = {min(Ls)}..{max(Ls)}, "
                         f"{nc} candidates) through the oracle's packed layout, {sum(per):.1f} s",
               "independent": {"value": nc_i / sum(per_i), "unit": UNIT,
                               "sample": f"4 candidates of request 0 scored independently (each its own "
                                         f"L + b sequence), {sum(per_i):.1f} s"}}
    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_max, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": (value / PAGES_CAND_PER_S[(args.config, args.mode)]
                            if (args.config, args.mode) in PAGES_CAND_PER_S and not reuse else None),
            "dtype": "f16", "data": "synthetic",
            "config": {**describe(wl, args.mode, not args.no_graph, world), "table": table_note,
                       **({"reuse": reuse.note, "tokens_per_step": T} if reuse else {})},
            "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": 4 * n_cand},
            "roofline": dominant,
            "roofline_step": {"flops_per_step": gf + af, "ms_at_peak": step_roof_ms,
                              "frac": step_roof_ms / ms_max, "peak": pk["tc_sustained"],
                              "unit": "TFLOP/s", "note": "whole step vs max(FLOPs/peak, bytes/HBM BW)"},
            "roofline_other": {k: v for k, v in roofs.items() if k != dom_key},
            "kernels": kernels,
            "gpu_launches": launches * args.steps,
            "clocks": clk.summary(),
            "cpu_baseline": cpu,
            "host_compile": compile_rate(wl),
        }
        print(json.dumps(line), flush=True)
    rk.close()
    if dist:
        dist.barrier()
        dist.destroy_process_group()


def relaunch(n: int, argv=None) -> int:
    """`--gpus N` without a launcher: run this same command as N ranks, one
    process per GPU, through torch's own launcher on this node (rendezvous
    on 127.0.0.1); returns the launcher's exit status."""
    import socket
    with socket.socket() as so:
        so.bind(("127.0.0.1", 0))
        port = so.getsockname()[1]
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={n}",
           "--master-addr=127.0.0.1", f"--master-port={port}", os.path.abspath(__file__),
           *(sys.argv[1:] if argv is None else argv)]
    return subprocess.call(cmd)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--config", default="c64")
    ap.add_argument("--mode", choices=["mis", "independent"], default="mis")
    ap.add_argument("--reuse", choices=["append", "rescore", "template"], default=None,
                    help="score from a prefix KV store (see the module docstring)")
    ap.add_argument("--no-graph", action="store_true")
    ap.add_argument("--skip-cpu", action="store_true")
    ap.add_argument("--profile-steps", type=int, default=0,
                    help="only run this many passes kernel by kernel (for ncu), print nothing")
    args = ap.parse_args()
    if args.warmup < 3:
        print(f"note: --warmup {args.warmup} is below the 3 warm-up steps a reported number needs",
              file=sys.stderr)
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if "WORLD_SIZE" not in os.environ and args.gpus > 1:
        sys.exit(relaunch(args.gpus))
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE is {world}: launch one process per GPU")
    if args.impl == "reference":
        run_reference(args, rank, world)
    elif args.config == "gather":
        run_gather(args, rank, world, local_rank)
    elif args.config == "latency":
        run_latency(args, rank, world, local_rank)
    else:
        run_ours(args, rank, world, local_rank)


if __name__ == "__main__":
    main()
