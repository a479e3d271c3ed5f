"""Seeded synthetic models and requests shaped like the DuoLM serving workloads.

Nothing here computes any step of the ranking method: weights are drawn,
rounded to their storage type and handed out; item vectors are the raw
encoder outputs ``a`` (the continuous interface that turns them into table
rows is the method's, and lives with each implementation); requests are
lists of token ids.

Request layout (DuoLM summary page, paper.rainbus.top, 核心方法 and
方法步骤详情 step 4; onedev.kr page, 어떻게 동작하나): an instruction,
then per history item a marker token, the item's virtual id and its feedback
text, then an optional candidate header; each candidate branch is ``b``
tokens whose last token is the candidate's virtual id.  A virtual id is
``V + item`` where ``V`` is the ranker vocabulary size.
"""
from __future__ import annotations

import functools
from dataclasses import dataclass, field
from typing import List, Optional

import numpy as np

from .rng import Stream, bf16_round

# Seeds: weights, item vectors, requests (requests add the config index).
SEED_WEIGHTS = 1234
SEED_ITEMS = 1235
SEED_REQUESTS = 1000


@dataclass(frozen=True)
class ModelShape:
    name: str
    n_layers: int
    d: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    ffn: int
    vocab: int
    rope_theta: float
    rms_eps: float
    dtype: str  # "fp32" or "bf16": storage and compute type of the GPU path

    @property
    def q_dim(self) -> int:
        return self.n_q_heads * self.head_dim

    @property
    def kv_dim(self) -> int:
        return self.n_kv_heads * self.head_dim


TINY = ModelShape("tiny-fp32", 2, 128, 4, 2, 32, 256, 512, 1e4, 1e-6, "fp32")
QWEN3_06B = ModelShape("qwen3-0.6b-shape", 28, 1024, 16, 8, 128, 3072, 151936, 1e6, 1e-6, "bf16")

WEIGHT_STD = 0.02


def weight_names(shape: ModelShape) -> List[tuple]:
    """(name, shape, init) of every model tensor, in the fixed load order.

    Matrices are stored [out_features, in_features], row-major.  ``init`` is
    "normal" (N(0, WEIGHT_STD)) or "ones" (norm gains).
    """
    d, qd, kd, f, hd = shape.d, shape.q_dim, shape.kv_dim, shape.ffn, shape.head_dim
    out = [("embed", (shape.vocab, d), "normal")]
    for l in range(shape.n_layers):
        out += [
            (f"l{l}.attn_norm", (d,), "ones"),
            (f"l{l}.wq", (qd, d), "normal"),
            (f"l{l}.wk", (kd, d), "normal"),
            (f"l{l}.wv", (kd, d), "normal"),
            (f"l{l}.q_norm", (hd,), "ones"),
            (f"l{l}.k_norm", (hd,), "ones"),
            (f"l{l}.wo", (d, qd), "normal"),
            (f"l{l}.mlp_norm", (d,), "ones"),
            (f"l{l}.w_gate", (f, d), "normal"),
            (f"l{l}.w_up", (f, d), "normal"),
            (f"l{l}.w_down", (d, f), "normal"),
        ]
    out += [("final_norm", (d,), "ones"), ("head", (d,), "normal")]
    return out


def _draw(seed: int, tag: int, shp, init: str, dtype: str) -> np.ndarray:
    n = int(np.prod(shp))
    if init == "ones":
        vals = np.ones(n, dtype=np.float64)
    else:
        vals = Stream(seed, tag).normal(n) * WEIGHT_STD
    if dtype == "bf16":
        return bf16_round(vals).reshape(shp)
    return vals.astype(np.float32).reshape(shp)


@functools.lru_cache(maxsize=4)
def model_weights(shape: ModelShape, seed: int = SEED_WEIGHTS) -> tuple:
    """All tensors in load order: uint16 bfloat16 bit patterns for bf16
    models, float32 for fp32 models.  Each tensor has its own stream."""
    return tuple(
        _draw(seed, tag, shp, init, shape.dtype)
        for tag, (_, shp, init) in enumerate(weight_names(shape))
    )


@functools.lru_cache(maxsize=4)
def item_vectors(n_items: int, d: int, seed: int = SEED_ITEMS) -> np.ndarray:
    """Raw encoder outputs a_i ~ N(0, 1)^d as float32 [n_items, d]."""
    return Stream(seed, 0).normal(n_items * d).astype(np.float32).reshape(n_items, d)


@dataclass
class Request:
    prefix_ids: np.ndarray          # int32 [L] ranker ids (vocab ids and V + item)
    branch_ids: np.ndarray          # int32 [K, b] ranker ids; last column is the candidate VID
    history_items: np.ndarray = field(default_factory=lambda: np.zeros(0, np.int64))
    cand_items: np.ndarray = field(default_factory=lambda: np.zeros(0, np.int64))
    feedback: List[np.ndarray] = field(default_factory=list)  # feedback tokens per history item

    @property
    def L(self) -> int:
        return int(self.prefix_ids.shape[0])

    @property
    def K(self) -> int:
        return int(self.branch_ids.shape[0])


@dataclass
class Workload:
    name: str
    model: ModelShape
    n_items: int
    branch_len: int
    requests: List[Request]
    note: str = ""
    template: Optional["_Template"] = None  # the prompt text the requests were built from
    m: int = 1                              # table rows per item

    @property
    def n_candidates(self) -> int:
        return sum(r.K for r in self.requests)

    @property
    def n_tokens(self) -> int:
        return sum(r.L + r.K * self.branch_len for r in self.requests)

    def packed(self):
        """The C-ABI view: prefix ids + offsets, branch ids + candidate offsets."""
        prefix = np.concatenate([r.prefix_ids for r in self.requests]).astype(np.int32) \
            if self.requests else np.zeros(0, np.int32)
        poff = np.zeros(len(self.requests) + 1, np.int64)
        poff[1:] = np.cumsum([r.L for r in self.requests])
        branch = np.concatenate([r.branch_ids.reshape(-1) for r in self.requests]).astype(np.int32) \
            if self.requests else np.zeros(0, np.int32)
        coff = np.zeros(len(self.requests) + 1, np.int64)
        coff[1:] = np.cumsum([r.K for r in self.requests])
        return prefix, poff, branch, coff

    def history_offsets(self, q: int) -> List[int]:
        """Prefix offset of each history item of request q (its marker)."""
        o, out = len(self.template.instr), []
        for f in self.requests[q].feedback:
            out.append(o)
            o += 1 + self.m + len(f)
        return out

    def records(self):
        """The requests as records (item ids and feedback tokens, no ids of
        the ranker's sequence): history items + offsets, feedback tokens +
        per-history-item offsets, candidate items + offsets."""
        def flat(arrs, dtype):
            off = np.zeros(len(arrs) + 1, np.int64)
            off[1:] = np.cumsum([len(a) for a in arrs])
            return (np.concatenate(arrs).astype(dtype) if arrs else np.zeros(0, dtype)), off
        hist, hoff = flat([r.history_items for r in self.requests], np.int64)
        fb, foff = flat([f for r in self.requests for f in r.feedback], np.int32)
        cand, coff = flat([r.cand_items for r in self.requests], np.int64)
        return hist, hoff, fb, foff, cand, coff


class _Template:
    """Template text of one configuration: instruction, marker, headers."""

    def __init__(self, s: Stream, vocab: int, n_instr: int, n_header: int, n_branch_header: int):
        self.instr = s.integers(n_instr, 0, vocab)
        self.marker = int(s.integers(1, 0, vocab)[0])
        self.header = s.integers(n_header, 0, vocab)
        self.branch_header = s.integers(n_branch_header, 0, vocab)


def _zipf_sampler(n_items: int, s_exp: float):
    ranks = np.arange(1, n_items + 1, dtype=np.float64)
    cdf = np.cumsum(ranks ** -s_exp)
    cdf /= cdf[-1]

    def draw(stream: Stream, n: int, exclude=()) -> np.ndarray:
        seen = set(int(e) for e in exclude)
        out = []
        while len(out) < n:
            u = stream.uniform(1)[0]
            v = int(min(np.searchsorted(cdf, u, side="right"), n_items - 1))
            if v not in seen:
                seen.add(v)
                out.append(v)
        return np.array(out, dtype=np.int64)

    return draw


def zipf_lookups(n: int, n_items: int = 1_000_000, s_exp: float = 1.1, seed: int = SEED_REQUESTS + 5) -> np.ndarray:
    """n item-table row indices drawn Zipf(s_exp) over n_items rows, with
    replacement: the stream of VID reads that many requests' histories and
    candidates produce on a large catalog (popular items recur)."""
    ranks = np.arange(1, n_items + 1, dtype=np.float64)
    cdf = np.cumsum(ranks ** -s_exp)
    cdf /= cdf[-1]
    u = Stream(seed, 0).uniform(n)
    return np.minimum(np.searchsorted(cdf, u, side="right"), n_items - 1).astype(np.int64)


def make_request(s: Stream, tpl: _Template, vocab: int, n_items: int, n_hist: int,
                 feedback_lens, n_cand: int, branch_len: int, item_draw=None,
                 random_branch_header: bool = False) -> Request:
    if item_draw is None:
        item_draw = lambda st, n, exclude=(): st.distinct(n, 0, n_items, exclude)
    hist = item_draw(s, n_hist)
    cands = item_draw(s, n_cand, exclude=hist)
    parts = [tpl.instr]
    fbs = []
    for i, it in enumerate(hist):
        fb = s.integers(int(feedback_lens[i]), 0, vocab)
        fbs.append(fb)
        parts += [np.array([tpl.marker, vocab + it]), fb]
    parts.append(tpl.header)
    prefix = np.concatenate([np.asarray(p, np.int64) for p in parts]).astype(np.int32)
    branch = np.empty((n_cand, branch_len), np.int64)
    if branch_len > 1:
        if random_branch_header:
            branch[:, :-1] = s.integers(n_cand * (branch_len - 1), 0, vocab).reshape(n_cand, branch_len - 1)
        else:
            branch[:, :-1] = np.broadcast_to(tpl.branch_header[: branch_len - 1], (n_cand, branch_len - 1))
    branch[:, -1] = vocab + cands
    return Request(prefix, branch.astype(np.int32), hist, cands, fbs)


def make_mv_request(s: Stream, tpl: _Template, vocab: int, n_items: int, m: int, n_hist: int, feedback_lens,
                    n_cand: int) -> Request:
    """A request over multi-vector items: item i is the m table rows i m ..
    i m + m - 1 (ids V + i m + k).  A history item is the marker followed by
    its m VIDs and its feedback tokens; a candidate branch is its m VIDs (b = m),
    scored at the last one."""
    hist = s.distinct(n_hist, 0, n_items)
    cands = s.distinct(n_cand, 0, n_items, hist)
    parts = [tpl.instr]
    fbs = []
    for i, it in enumerate(hist):
        fb = s.integers(int(feedback_lens[i]), 0, vocab)
        fbs.append(fb)
        parts += [np.array([tpl.marker]), vocab + it * m + np.arange(m), fb]
    parts.append(tpl.header)
    prefix = np.concatenate([np.asarray(p, np.int64) for p in parts]).astype(np.int32)
    branch = vocab + cands[:, None] * m + np.arange(m)[None, :]
    return Request(prefix, branch.astype(np.int32), hist, cands, fbs)


def fir(m: int = 8, n_requests: int = 64, shard: int = 0) -> Workload:
    """The 64-request recipe with multi-vector items of m rows each: history
    U{1..20} items, U{8..48} feedback tokens per item, K = 100 candidates of
    m tokens, 100k items = 100k m table rows."""
    model = QWEN3_06B
    n_items = 100_000
    s = Stream(SEED_REQUESTS + 6, shard)
    tpl = _Template(s, model.vocab, 32, 4, 0)
    reqs = []
    for _ in range(n_requests):
        h = int(s.integers(1, 1, 21)[0])
        f = s.integers(h, 8, 49)
        reqs.append(make_mv_request(s, tpl, model.vocab, n_items, m, h, f, 100))
    return Workload(f"fir-m{m}", model, n_items * m, m, reqs, template=tpl, m=m)


def custom_fir(model: ModelShape, n_items: int, seed: int, n_requests: int, n_hist: int, feedback: int,
               n_cand: int, m: int) -> Workload:
    """Small multi-vector workloads for parity tests (n_items items, n_items m
    table rows)."""
    s = Stream(seed, 11)
    tpl = _Template(s, model.vocab, 3, 2, 0)
    reqs = [make_mv_request(s, tpl, model.vocab, n_items, m, n_hist, [feedback] * n_hist, n_cand)
            for _ in range(n_requests)]
    return Workload(f"custom-fir-m{m}", model, n_items * m, m, reqs, template=tpl, m=m)


def tiny(seed_offset: int = 0) -> Workload:
    """Tiny fp32 ranker, one request: L = 8 + 4 x (1 + 1 + 8) = 48, K = 8, b = 1."""
    m = TINY
    s = Stream(SEED_REQUESTS + 0 + seed_offset, 0)
    tpl = _Template(s, m.vocab, 8, 0, 0)
    r = make_request(s, tpl, m.vocab, 64, 4, [8] * 4, 8, 1)
    return Workload("tiny", m, 64, 1, [r], template=tpl)


def c1(shard: int = 0) -> Workload:
    """Qwen3-0.6B shape, one request: L = 32 + 10 x (2 + 24) + 4 = 296, K = 100, b = 1."""
    m = QWEN3_06B
    s = Stream(SEED_REQUESTS + 1, shard)
    tpl = _Template(s, m.vocab, 32, 4, 0)
    r = make_request(s, tpl, m.vocab, 100_000, 10, [24] * 10, 100, 1)
    return Workload("c1", m, 100_000, 1, [r], template=tpl)


def c64(n_requests: int = 64, shard: int = 0) -> Workload:
    """Qwen3-0.6B shape, 64 ragged requests: history U{1..20} items, feedback
    U{8..48} tokens per item, K = 100, items uniform over 100k.  ``shard``
    selects an independent batch of the same recipe (one per GPU)."""
    m = QWEN3_06B
    s = Stream(SEED_REQUESTS + 2, shard)
    tpl = _Template(s, m.vocab, 32, 4, 0)
    reqs = []
    for _ in range(n_requests):
        h = int(s.integers(1, 1, 21)[0])
        f = s.integers(h, 8, 49)
        reqs.append(make_request(s, tpl, m.vocab, 100_000, h, f, 100, 1))
    return Workload("c64", m, 100_000, 1, reqs, template=tpl)


def stress(n_requests: int = 16, shard: int = 0) -> Workload:
    """Long history: 16 requests, L = 32 + 50 x (2 + 40) = 2132, K = 256,
    b = 4 (3 fixed header tokens + the candidate VID)."""
    m = QWEN3_06B
    s = Stream(SEED_REQUESTS + 3, shard)
    tpl = _Template(s, m.vocab, 32, 0, 3)
    reqs = [make_request(s, tpl, m.vocab, 100_000, 50, [40] * 50, 256, 4) for _ in range(n_requests)]
    return Workload("stress", m, 100_000, 4, reqs, template=tpl)


def catalog(concurrency: int, shard: int = 0) -> Workload:
    """1M-item table, Zipf(1.1) item ids, history 10 x 24 feedback tokens,
    K = 100, header 4; concurrency C in {1, 8, 64}."""
    m = QWEN3_06B
    n_items = 1_000_000
    s = Stream(SEED_REQUESTS + 4, concurrency + 1000 * shard)
    tpl = _Template(s, m.vocab, 32, 4, 0)
    draw = _zipf_sampler(n_items, 1.1)
    reqs = [make_request(s, tpl, m.vocab, n_items, 10, [24] * 10, 100, 1, item_draw=draw)
            for _ in range(concurrency)]
    return Workload(f"catalog-c{concurrency}", m, n_items, 1, reqs, template=tpl)


def custom(model: ModelShape, n_items: int, seed: int, n_requests: int, n_hist, feedback,
           n_cand, branch_len: int, n_instr: int = 4, n_header: int = 0,
           random_branch_header: bool = True) -> Workload:
    """Small ragged workloads for edge cases.  ``n_hist``/``feedback``/``n_cand``
    are ints or (low, high) inclusive ranges drawn per request/item."""
    s = Stream(seed, 7)
    tpl = _Template(s, model.vocab, n_instr, n_header, max(branch_len - 1, 0))

    def pick(v):
        if isinstance(v, tuple):
            return int(s.integers(1, v[0], v[1] + 1)[0])
        return int(v)

    reqs = []
    for _ in range(n_requests):
        h = pick(n_hist)
        f = [pick(feedback) for _ in range(h)]
        k = pick(n_cand)
        reqs.append(make_request(s, tpl, model.vocab, n_items, h, f, k, branch_len,
                                 random_branch_header=random_branch_header))
    return Workload(f"custom-{seed}", model, n_items, branch_len, reqs,
                    template=None if random_branch_header else tpl)


CONFIGS = {"tiny": tiny, "c1": c1, "c64": c64, "stress": stress}
