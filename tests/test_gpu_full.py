"""GPU parity at the full Qwen3-0.6B-shaped configurations, in the launch
configuration the benchmark times (one duolm_score call over the whole
batch, CUDA graph on).  The oracle scores every candidate of the C=1
request, and sampled requests (or a sampled subset of candidates, whose
scores do not depend on the other candidates) of the larger batches."""
import numpy as np
import pytest

from oracle import ranker as R
from synth import workloads as W

import parity as P

pytestmark = pytest.mark.gpu

Q = W.QWEN3_06B


def test_c1_all_candidates_and_independent_mode():
    wl = W.c1()
    rk = P.ranker(Q, wl.n_items)
    otab = P.oracle_table(Q, wl.n_items)[0]
    om = P.oracle_model(Q)
    req = wl.requests[0]
    got = rk.score_workload(wl)
    ref = R.score_mis(om, otab, req)
    P.assert_scores_match(Q, got, ref, "c1 MIS")
    # independent mode: every candidate as its own sequence on the GPU; the
    # oracle's own independent sequences for four of them
    got_ind = rk.score_workload(wl, 1)
    P.assert_scores_match(Q, got_ind, ref, "c1 independent")
    pick = [0, 37, 63, 99]
    ref_ind = R.score_independent(om, otab, req, pick)
    assert np.array_equal(ref_ind, ref[pick])  # s^MIS = s inside the oracle, bit for bit
    assert np.abs(got_ind[pick] - ref_ind).max() <= P.tolerance(Q, ref)


def test_c64_sampled_requests():
    wl = W.c64()
    rk = P.ranker(Q, wl.n_items)
    otab = P.oracle_table(Q, wl.n_items)[0]
    om = P.oracle_model(Q)
    got = P.split_scores(wl, rk.score_workload(wl))
    Ls = [r.L for r in wl.requests]
    for q in sorted({0, int(np.argmax(Ls)), int(np.argmin(Ls)), 63}):
        ref = R.score_mis(om, otab, wl.requests[q])
        P.assert_scores_match(Q, got[q], ref, f"c64 request {q} (L={Ls[q]})")


def _oracle_scores(wl: W.Workload, q: int, pick=None) -> np.ndarray:
    """The oracle's scores of request q, from only the table rows the request
    touches (interface output of the same seeded item vectors)."""
    om = P.oracle_model(Q)
    req = wl.requests[q]
    rows = np.unique(np.concatenate([req.prefix_ids, req.branch_ids.reshape(-1)]))
    rows = rows[rows >= Q.vocab] - Q.vocab
    # the item-vector stream is counter-based: its first n rows are the
    # first n rows of any longer draw, so only rows up to the largest are made
    a = W.item_vectors(int(rows.max()) + 1, Q.d)[rows]
    sub = R.table_f32(R.interface(a, 0.0, P.oracle_rho(Q)))
    remap = {int(r): i for i, r in enumerate(rows)}

    def rm(ids):
        return np.array([i if i < Q.vocab else Q.vocab + remap[int(i) - Q.vocab] for i in ids.reshape(-1)],
                        np.int32).reshape(ids.shape)
    return R.score_mis(om, sub, W.Request(rm(req.prefix_ids), rm(req.branch_ids)), pick)


def test_stress_every_candidate_of_one_request():
    """Long history (L = 2132) and 4-token branches: all 256 candidates of
    one request, intra-branch causal attention, against the oracle."""
    wl = W.stress()
    rk = P.ranker(Q, wl.n_items)
    got = P.split_scores(wl, rk.score_workload(wl))
    q = 5
    ref = _oracle_scores(wl, q)
    P.assert_scores_match(Q, got[q], ref, f"stress request {q} (L={wl.requests[q].L})")


@pytest.mark.parametrize("conc", [1, 8, 64])
def test_catalog_zipf_sampled(conc):
    """1M-row item table, Zipf(1.1) item ids; at C = 64 the first, the last
    and the longest request."""
    wl = W.catalog(conc)
    rk = P.ranker(Q, wl.n_items)
    got = P.split_scores(wl, rk.score_workload(wl))
    Ls = [r.L for r in wl.requests]
    for q in sorted({conc - 1, 0, int(np.argmax(Ls))}):
        ref = _oracle_scores(wl, q)
        P.assert_scores_match(Q, got[q], ref, f"catalog C={conc} request {q} (L={Ls[q]})")
    # the device table holds exactly the interface output for the rows the
    # last request touches
    req = wl.requests[conc - 1]
    rows = np.unique(np.concatenate([req.prefix_ids, req.branch_ids.reshape(-1)]))
    rows = rows[rows >= Q.vocab] - Q.vocab
    a = W.item_vectors(int(rows.max()) + 1, Q.d)[rows]
    tab = rk.debug_table(wl.n_items)
    assert np.array_equal(tab[rows], R.interface(a, 0.0, P.oracle_rho(Q)).view(np.uint16))


def test_fir_m8_full_recipe_sampled_requests():
    """Multi-vector items at full size: the 64-request recipe with m = 8 rows
    per item (800k table rows, b = 8, T about 79k tokens); every candidate of
    the longest request and of request 0."""
    wl = W.fir(8)
    assert wl.branch_len == 8 and wl.n_items == 800_000
    rk = P.ranker(Q, wl.n_items)
    got = P.split_scores(wl, rk.score_workload(wl))
    Ls = [r.L for r in wl.requests]
    for q in sorted({0, int(np.argmax(Ls))}):
        ref = _oracle_scores(wl, q)
        P.assert_scores_match(Q, got[q], ref, f"fir-m8 request {q} (L={Ls[q]})")
