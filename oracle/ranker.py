"""Oracle for the DuoLM multi-item-scoring (MIS) forward -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this module.  It shares no code with the CUDA
library; the two meet only at the seeded inputs from ``synth``.

Definitions it follows (page titles and sections):

* DuoLM summary page (paper.rainbus.top, "DuoLM:基于语言模型的快速高效个性化推荐框架"),
  核心方法: the ranker reads the instruction, the ordered history entries and
  the candidate vector; a shared linear head gives s_{q,j} = w^T h_{q,j} at the
  candidate's last hidden state, with no decoding.
* Same page, 方法步骤详情 step 3: item vectors z_i are stored in FP16 in a
  GPU-resident table D; virtual id V + i reads row i.
* Same page, 方法步骤详情 step 4 and 研究动机: the K candidates are packed
  behind one shared prefix P_q that is prefilled once; candidate j sees only the
  prefix and itself (tree mask) and sits at logical position L_q; the scores
  come back in input order; in exact arithmetic s^MIS_{q,j} = s_{q,j}, and each
  layer drops (K_q - 1) L_q (L_q + 1) / 2 duplicate prefix query-key pairs.
* Same page, 前置知识 (连续输入接口) and 核心方法: the continuous interface
  z_i = e^gamma * rho * a_i / RMS(a_i).

The score of a candidate is defined on its own independent sequence
P_q || branch_j with positions 0 .. L_q + b - 1 and a causal mask
(:func:`independent_layout`).  The packed layout (:func:`mis_layout`) puts the
prefix once, then every branch, and gives each branch row the prefix keys
followed by its own branch keys, in the same order as the independent
sequence, so both layouts reach the same bits through the C core.

Readings taken where the pages are silent:
branch token i of a b-token branch sits at position L + i and sees branch
tokens 0..i; h is the output of the final RMSNorm; there is no score bias;
RMS in the interface has no epsilon; the interface output is rounded to FP16
with round-to-nearest-even; the reference scale rho of the synthetic
configurations is the mean over embedding rows of each row's RMS.  Every
arithmetic step runs in fp64 where a plain fp32 ranker would do: fp64 is the
stricter reading (its own rounding sits far below both tolerances, 1e-4 for
the fp32 model and 2e-2 std(s) for the bf16-valued one), so a disagreement
with the GPU path is the GPU path's.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass
from typing import Optional, Sequence

import numpy as np

from synth.rng import bf16_to_f32
from synth.workloads import ModelShape, Request, Workload

from . import build as _build

_lib = None


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        L.oracle_forward.restype = ctypes.c_int
        L.oracle_forward.argtypes = [
            ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64,
            ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
            ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]
        L.oracle_attend.restype = None
        L.oracle_attend.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int,
                                    ctypes.c_int, ctypes.c_long, ctypes.c_double, ctypes.c_void_p,
                                    ctypes.c_void_p, ctypes.c_void_p]
        L.oracle_rope.restype = None
        L.oracle_rope.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_double]
        L.oracle_rmsnorm.restype = None
        L.oracle_rmsnorm.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, ctypes.c_double,
                                     ctypes.c_void_p]
        _lib = L
    return _lib


def _ptr(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data


# ----------------------------------------------------------------------------
# model and item table
# ----------------------------------------------------------------------------

class OracleModel:
    """The ranker's weights widened exactly to float32 (load order of
    ``synth.workloads.weight_names``)."""

    def __init__(self, shape: ModelShape, weights: Sequence[np.ndarray]):
        self.shape = shape
        w32 = []
        for a in weights:
            if a.dtype == np.uint16:
                w32.append(np.ascontiguousarray(bf16_to_f32(a)))
            else:
                w32.append(np.ascontiguousarray(a, dtype=np.float32))
        self.w32 = w32
        self._ptrs = (ctypes.c_void_p * len(w32))(*[a.ctypes.data for a in w32])
        self._shape_i = np.array([shape.n_layers, shape.d, shape.n_q_heads, shape.n_kv_heads,
                                  shape.head_dim, shape.ffn, shape.vocab], dtype=np.int32)
        self._shape_f = np.array([shape.rope_theta, shape.rms_eps], dtype=np.float64)

    @property
    def embed(self) -> np.ndarray:
        return self.w32[0]


def rms(a: np.ndarray) -> np.ndarray:
    """Root mean square of each row, no epsilon: sqrt(mean(a^2))."""
    a = np.asarray(a, dtype=np.float64)
    return np.sqrt(np.mean(a * a, axis=-1))


def embedding_rho(embed: np.ndarray) -> float:
    """Reference scale rho estimated from the ranker's native embeddings:
    the mean over vocabulary rows of each row's RMS (the pages fix rho for
    real Qwen3 weights only; for random weights this is the plain reading)."""
    return float(np.mean(rms(embed)))


def interface(a: np.ndarray, gamma: float, rho: float) -> np.ndarray:
    """Continuous interface z = e^gamma * rho * a / RMS(a), per row, in fp64,
    then stored as FP16 (round to nearest even).  Returns float16 [n, d]."""
    a = np.asarray(a, dtype=np.float64)
    z = (np.exp(gamma) * rho) * a / rms(a)[:, None]
    return z.astype(np.float16)


def table_f32(table_fp16: np.ndarray) -> np.ndarray:
    """The FP16 table widened exactly, as the C core reads it."""
    return np.ascontiguousarray(np.asarray(table_fp16, dtype=np.float16).astype(np.float32))


# ----------------------------------------------------------------------------
# layouts: rows, positions and key lists
# ----------------------------------------------------------------------------

@dataclass
class Layout:
    ids: np.ndarray       # int32 [n_rows]
    pos: np.ndarray       # int32 [n_rows]
    key_ptr: np.ndarray   # int64 [n_rows + 1]
    key_idx: np.ndarray   # int32 [n_keys]
    out_rows: np.ndarray  # int32 [n_out]

    @property
    def n_rows(self) -> int:
        return int(self.ids.shape[0])

    def n_pairs(self) -> int:
        return int(self.key_ptr[-1])


def _layout(ids, pos, keys, out_rows) -> Layout:
    ptr = np.zeros(len(keys) + 1, np.int64)
    ptr[1:] = np.cumsum([len(k) for k in keys])
    idx = np.concatenate([np.asarray(k, np.int32) for k in keys]) if keys else np.zeros(0, np.int32)
    return Layout(np.asarray(ids, np.int32), np.asarray(pos, np.int32), ptr,
                  idx.astype(np.int32), np.asarray(out_rows, np.int32))


def independent_layout(prefix_ids: np.ndarray, branch: np.ndarray) -> Layout:
    """One candidate's own sequence P || branch: positions 0..L+b-1, causal."""
    ids = np.concatenate([prefix_ids, branch]).astype(np.int32)
    n = ids.shape[0]
    keys = [np.arange(t + 1) for t in range(n)]
    return _layout(ids, np.arange(n), keys, [n - 1])


def mis_layout(prefix_ids: np.ndarray, branches: np.ndarray) -> Layout:
    """Packed multi-item layout: the prefix once (rows 0..L-1), then branch j
    token i at row L + j*b + i.  Prefix row t sees prefix rows 0..t; branch
    row (j, i) sees prefix rows 0..L-1 then its own branch rows 0..i (tree
    mask) and sits at position L + i (unified logical position)."""
    L = int(prefix_ids.shape[0])
    K, b = branches.shape
    ids = np.concatenate([prefix_ids, branches.reshape(-1)]).astype(np.int32)
    pos = np.concatenate([np.arange(L), np.tile(L + np.arange(b), K)])
    keys = [np.arange(t + 1) for t in range(L)]
    pre = np.arange(L)
    for j in range(K):
        base = L + j * b
        for i in range(b):
            keys.append(np.concatenate([pre, base + np.arange(i + 1)]))
    out_rows = [L + j * b + b - 1 for j in range(K)]
    return _layout(ids, pos, keys, out_rows)


def tree_mask(L: int, K: int, b: int) -> np.ndarray:
    """Visibility of every (query row, key row) pair of the packed layout,
    evaluated pair by pair from the rule: a prefix row sees earlier-or-equal
    prefix rows; a branch row sees every prefix row and the rows of its own
    branch up to itself; nothing else."""
    T = L + K * b
    m = np.zeros((T, T), dtype=bool)
    for qr in range(T):
        for kr in range(T):
            if qr < L:
                m[qr, kr] = kr <= qr
            elif kr < L:
                m[qr, kr] = True
            else:
                qj, qi = divmod(qr - L, b)
                kj, ki = divmod(kr - L, b)
                m[qr, kr] = (qj == kj) and (ki <= qi)
    return m


def mis_positions(L: int, K: int, b: int) -> np.ndarray:
    """Position ids of the packed layout: prefix t -> t, branch token i -> L + i."""
    return mis_layout(np.zeros(L, np.int32), np.zeros((K, b), np.int32)).pos


# ----------------------------------------------------------------------------
# forward and scores
# ----------------------------------------------------------------------------

def forward(model: OracleModel, table: np.ndarray, lay: Layout, want_hidden: bool = False,
            want_layers: bool = False):
    """Run the C core over a layout.  ``table`` is float32 [n_items, d]."""
    s = model.shape
    table = np.ascontiguousarray(table, dtype=np.float32)
    scores = np.zeros(lay.out_rows.shape[0], np.float64)
    hidden = np.zeros((lay.out_rows.shape[0], s.d), np.float64) if want_hidden else None
    layers = np.zeros((s.n_layers + 1, lay.n_rows, s.d), np.float64) if want_layers else None
    rc = lib().oracle_forward(
        _ptr(model._shape_i), _ptr(model._shape_f), ctypes.addressof(model._ptrs), _ptr(table),
        table.shape[0], lay.n_rows, _ptr(lay.ids), _ptr(lay.pos), _ptr(lay.key_ptr),
        _ptr(lay.key_idx), lay.out_rows.shape[0], _ptr(lay.out_rows), _ptr(scores),
        _ptr(hidden), _ptr(layers))
    if rc != 0:
        raise ValueError(f"oracle_forward rejected its input (code {rc})")
    out = [scores]
    if want_hidden:
        out.append(hidden)
    if want_layers:
        out.append(layers)
    return out[0] if len(out) == 1 else tuple(out)


def score_independent(model: OracleModel, table: np.ndarray, req: Request,
                      cands: Optional[Sequence[int]] = None) -> np.ndarray:
    """Scores of the chosen candidates, each from its own full sequence."""
    cands = range(req.K) if cands is None else cands
    return np.array([forward(model, table, independent_layout(req.prefix_ids, req.branch_ids[j]))[0]
                     for j in cands], dtype=np.float64)


def score_mis(model: OracleModel, table: np.ndarray, req: Request,
              cands: Optional[Sequence[int]] = None) -> np.ndarray:
    """Scores of the chosen candidates (default all, input order) from one
    packed pass: prefix once, branches behind it under the tree mask."""
    br = req.branch_ids if cands is None else req.branch_ids[np.asarray(list(cands), np.int64)]
    return forward(model, table, mis_layout(req.prefix_ids, br))


def score_workload(model: OracleModel, table: np.ndarray, wl: Workload,
                   requests: Optional[Sequence[int]] = None) -> list:
    """Per-request score arrays (MIS form) for the chosen requests."""
    idx = range(len(wl.requests)) if requests is None else requests
    return [score_mis(model, table, wl.requests[i]) for i in idx]


# ----------------------------------------------------------------------------
# single steps, exposed for the pins
# ----------------------------------------------------------------------------

def attend(q: np.ndarray, K: np.ndarray, V: np.ndarray, scale: float):
    """Softmax attention of one query over rows of K/V -> (probs, out)."""
    q = np.ascontiguousarray(q, np.float64)
    K = np.ascontiguousarray(K, np.float64)
    V = np.ascontiguousarray(V, np.float64)
    n, hd = K.shape
    probs = np.zeros(n, np.float64)
    out = np.zeros(hd, np.float64)
    work = np.zeros(max(n, 1), np.float64)
    lib().oracle_attend(_ptr(q), _ptr(K), _ptr(V), n, hd, hd, scale, _ptr(probs), _ptr(out), _ptr(work))
    return probs, out


def rope(v: np.ndarray, pos: int, theta: float) -> np.ndarray:
    v = np.array(v, dtype=np.float64, copy=True)
    lib().oracle_rope(_ptr(v), v.shape[0], int(pos), float(theta))
    return v


def rmsnorm(x: np.ndarray, g: np.ndarray, eps: float) -> np.ndarray:
    x = np.ascontiguousarray(x, np.float64)
    g = np.ascontiguousarray(g, np.float32)
    y = np.zeros_like(x)
    lib().oracle_rmsnorm(_ptr(x), _ptr(g), x.shape[0], float(eps), _ptr(y))
    return y
