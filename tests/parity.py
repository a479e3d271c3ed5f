"""Shared helpers of the GPU parity tests: cached models on both sides and the
comparison rules.

Tolerances (stated for the ranker's scores): |ds| <= 1e-4 for the fp32 model;
|ds| <= 2e-2 * std(s) for the bf16-weight model, std over the oracle's scores
of the request; top-10 order per request identical except where the oracle's
scores of the swapped candidates differ by no more than that tolerance.
"""
from __future__ import annotations

import functools

import numpy as np

from oracle import ranker as R
from synth import workloads as W

TOL_FP32 = 1e-4
TOL_BF16_REL_STD = 2e-2


@functools.lru_cache(maxsize=4)
def oracle_model(shape: W.ModelShape):
    return R.OracleModel(shape, W.model_weights(shape))


@functools.lru_cache(maxsize=4)
def oracle_rho(shape: W.ModelShape) -> float:
    return R.embedding_rho(oracle_model(shape).embed)


@functools.lru_cache(maxsize=2)
def oracle_table(shape: W.ModelShape, n_items: int):
    """Returns (float32 table for the oracle, fp16 table, rho)."""
    rho = oracle_rho(shape)
    t16 = R.interface(W.item_vectors(n_items, shape.d), 0.0, rho)
    return R.table_f32(t16), t16, rho


_rankers = {}


def ranker(shape: W.ModelShape, n_items: int):
    """GPU ranker with its item table built on the device from the same raw
    item vectors (through the library's own interface kernel)."""
    import shared_prefix_item_b200 as S
    key = (shape, n_items)
    if key not in _rankers:
        for k in list(_rankers):
            _rankers.pop(k).close()
        rk = S.Ranker(shape, W.model_weights(shape))
        rk.vid_table_build(W.item_vectors(n_items, shape.d), 0.0, oracle_rho(shape))
        _rankers[key] = rk
    return _rankers[key]


def tolerance(shape: W.ModelShape, ref: np.ndarray) -> float:
    if shape.dtype == "fp32":
        return TOL_FP32
    return TOL_BF16_REL_STD * float(np.std(ref))


def assert_scores_match(shape, got: np.ndarray, ref: np.ndarray, what: str = ""):
    got = np.asarray(got, np.float64)
    tol = tolerance(shape, ref)
    err = np.abs(got - ref)
    assert err.max() <= tol, f"{what}: max |ds| {err.max():.3e} > tol {tol:.3e} (at {int(err.argmax())})"
    # top-10 order (ties broken by lower index on both sides)
    k = min(10, len(ref))
    top_ref = np.argsort(-ref, kind="stable")[:k]
    top_got = np.argsort(-got, kind="stable")[:k]
    for i in range(k):
        if top_ref[i] != top_got[i]:
            assert abs(ref[top_ref[i]] - ref[top_got[i]]) <= tol, \
                f"{what}: top-10 rank {i} differs beyond tolerance"
    return err.max(), tol


def split_scores(wl: W.Workload, flat: np.ndarray):
    out, o = [], 0
    for r in wl.requests:
        out.append(flat[o:o + r.K])
        o += r.K
    return out


def single_candidate_tolerance(shape: W.ModelShape, om, otab, req: W.Request, n_items: int, seed: int = 7) -> float:
    """Tolerance for a request with K = 1, where the std over its own scores
    is 0: 2e-2 times the std of the oracle's scores of 16 seeded random
    candidates on the same prefix (branches of the same length, the last
    token a table row, the others vocabulary tokens)."""
    if shape.dtype == "fp32":
        return TOL_FP32
    rng = np.random.default_rng(seed)
    b = req.branch_ids.shape[1]
    br = np.empty((16, b), np.int32)
    br[:, :-1] = rng.integers(0, shape.vocab, size=(16, b - 1))
    br[:, -1] = shape.vocab + rng.choice(n_items, size=16, replace=False)
    ref = R.score_mis(om, otab, W.Request(req.prefix_ids, br))
    return TOL_BF16_REL_STD * float(np.std(ref))
