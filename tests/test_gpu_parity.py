"""GPU parity of the C-ABI library against the oracle (tiny and ragged
workloads; full-size configurations are in test_gpu_full.py).

Bit-exact: the item table built through the interface, the packed layout and
position ids, the attention kernels' visibility rule and the virtual-id
gather.  Within tolerance (see parity.py): scores in both modes, raw
tensor-core GEMMs against fp64 products of the same fp16 operands.
"""
import dataclasses

import numpy as np
import pytest

from oracle import ranker as R
from synth import workloads as W
from synth.rng import bf16_to_f32

import parity as P

pytestmark = pytest.mark.gpu

TINY = W.TINY
# Qwen3-0.6B layer shapes with 2 layers and a small vocabulary: every kernel
# of the bf16 path at its production shape, with an oracle that runs in seconds.
Q2 = dataclasses.replace(W.QWEN3_06B, n_layers=2, vocab=4096, name="qwen3-shape-2layer")
Q2_ITEMS = 1000


def _check_layout_mask_gather(rk, shape, wl, otab):
    p, po, b, co = wl.packed()
    rk.prepare(p, po, b, co, wl.branch_len)
    ids, pos = rk.debug_layout()
    lays = [R.mis_layout(r.prefix_ids, r.branch_ids) for r in wl.requests]
    assert np.array_equal(ids, np.concatenate([l.ids for l in lays]))
    assert np.array_equal(pos, np.concatenate([l.pos for l in lays]))
    for q, r in enumerate(wl.requests[:4]):
        tq = r.L + r.K * wl.branch_len
        assert np.array_equal(rk.debug_mask(q, tq), R.tree_mask(r.L, r.K, wl.branch_len))
    x0 = rk.debug_residual(0, len(ids))
    om = P.oracle_model(shape)
    exp = np.stack([om.embed[i] if i < shape.vocab else otab[i - shape.vocab] for i in ids])
    assert np.array_equal(x0, exp)


# --------------------------------------------------------------------------
# tiny fp32 ranker
# --------------------------------------------------------------------------

def test_table_build_bit_exact_and_rho():
    rk = P.ranker(TINY, 64)
    otab, t16, rho = P.oracle_table(TINY, 64)
    assert np.array_equal(rk.debug_table(64), t16.view(np.uint16))
    assert rk.embedding_rho() == pytest.approx(rho, rel=1e-12)


def test_tiny_layout_mask_gather_bit_exact():
    _check_layout_mask_gather(P.ranker(TINY, 64), TINY, W.tiny(), P.oracle_table(TINY, 64)[0])


@pytest.mark.parametrize("mode", [0, 1])
def test_tiny_scores(mode):
    wl = W.tiny()
    rk = P.ranker(TINY, 64)
    got = rk.score_workload(wl, mode)
    ref = R.score_independent(P.oracle_model(TINY), P.oracle_table(TINY, 64)[0], wl.requests[0])
    P.assert_scores_match(TINY, got, ref, f"tiny mode {mode}")


@pytest.mark.parametrize("seed,n_req,n_hist,fb,K,b", [
    (101, 1, 0, 1, 1, 1),          # L = 1, K = 1: a single prefix token, one candidate
    (102, 3, (0, 3), (1, 9), (1, 7), 4),
    (103, 2, (2, 5), (10, 30), (20, 40), 2),
    (104, 4, (1, 4), (5, 17), (1, 9), 5),
])
def test_tiny_ragged(seed, n_req, n_hist, fb, K, b):
    wl = W.custom(TINY, 64, seed, n_req, n_hist, fb, K, b, n_instr=1 + seed % 3)
    rk = P.ranker(TINY, 64)
    otab = P.oracle_table(TINY, 64)[0]
    _check_layout_mask_gather(rk, TINY, wl, otab)
    got = P.split_scores(wl, rk.score_workload(wl))
    got_ind = P.split_scores(wl, rk.score_workload(wl, 1))
    om = P.oracle_model(TINY)
    for q, r in enumerate(wl.requests):
        ref = R.score_mis(om, otab, r)
        P.assert_scores_match(TINY, got[q], ref, f"req {q}")
        P.assert_scores_match(TINY, got_ind[q], ref, f"req {q} independent")


# --------------------------------------------------------------------------
# bf16-weight path at Qwen3-0.6B layer shapes
# --------------------------------------------------------------------------

@pytest.mark.parametrize("T_req", [(1, 1), (126, 2), (127, 2), (300, 7)])
def test_tcgen05_gemm_against_fp64(T_req):
    """Raw projections through the tensor-core GEMM: out = a W^T for token
    counts 2 (one partial tile), 128 (one exact tile), 129 and 307 (ragged
    multi-tile)."""
    L, K = T_req
    wl = W.custom(Q2, Q2_ITEMS, 200 + L, 1, 0, 1, K, 1, n_instr=L)
    rk = P.ranker(Q2, Q2_ITEMS)
    p, po, b, co = wl.packed()
    rk.prepare(p, po, b, co, 1)
    T = wl.n_tokens
    w = W.model_weights(Q2)
    rng = np.random.default_rng(L)
    for layer in [0, 1]:
        base = 1 + 11 * layer
        mats = {
            0: np.concatenate([bf16_to_f32(w[base + 1]), bf16_to_f32(w[base + 2]), bf16_to_f32(w[base + 3])]),
            1: bf16_to_f32(w[base + 6]),
            2: np.concatenate([np.concatenate([bf16_to_f32(w[base + 8])[i:i + 128], bf16_to_f32(w[base + 9])[i:i + 128]])
                               for i in range(0, Q2.ffn, 128)]),
            3: bf16_to_f32(w[base + 10]),
        }
        for which, Wm in mats.items():
            A = (rng.normal(size=(T, Wm.shape[1])) * 0.5).astype(np.float16)
            ref = A.astype(np.float64) @ Wm.astype(np.float64).T
            # whole-K tiles (which) and the split-K form small batches use for
            # the O and down projections (which + 4: four K-slices summed in order)
            for split in (0, 4):
                got = rk.debug_gemm(layer, which + split, A, Wm.shape[0])
                # fp32 accumulation of K products: far inside 1e-5 of the row scale
                assert np.abs(got - ref).max() <= 1e-5 * np.abs(ref).max(), (layer, which, split)


def test_q2_layout_mask_gather_bit_exact():
    wl = W.custom(Q2, Q2_ITEMS, 301, 3, (1, 6), (3, 20), (5, 40), 1, n_instr=7, n_header=4)
    _check_layout_mask_gather(P.ranker(Q2, Q2_ITEMS), Q2, wl, P.oracle_table(Q2, Q2_ITEMS)[0])


@pytest.mark.parametrize("seed,n_req,n_hist,fb,K,b,n_instr", [
    (311, 1, 0, 1, 1, 1, 1),            # L = 1, K = 1
    (312, 3, (1, 6), (3, 20), (5, 40), 1, 7),
    (313, 2, (0, 4), (1, 30), (1, 20), 4, 3),
    (314, 2, 2, 28, 33, 1, 1),          # L = 63: prefix one short of a query sub-tile
    (315, 1, 1, 60, 64, 1, 0),          # L = 64, K = 64: every item fills sub-tile A only
    (316, 2, 3, (40, 45), (30, 70), 2, 5),  # L > 128: several key tiles, ragged tail
    (317, 1, 1, 60, 9, 32, 2),          # b = 32: a quarter of an attention item
    (318, 1, 1, 70, 2, 128, 2),         # b = 128: the longest branch the kernel takes
    (3101, 1, 1, 122, 200, 1, 2),       # L = 128 (one full item), branch rows span two items
    (3105, 4, 1, (120, 125), (60, 70), 1, 2),  # L in {126, ..., 129}: item and key-tile edges
    (3112, 1, 1, 60, 3, 96, 2),         # b = 96: one candidate per item, split across sub-tiles
])
def test_q2_ragged_scores(seed, n_req, n_hist, fb, K, b, n_instr):
    wl = W.custom(Q2, Q2_ITEMS, seed, n_req, n_hist, fb, K, b, n_instr=n_instr, n_header=2)
    rk = P.ranker(Q2, Q2_ITEMS)
    otab = P.oracle_table(Q2, Q2_ITEMS)[0]
    got = P.split_scores(wl, rk.score_workload(wl))
    got_ind = P.split_scores(wl, rk.score_workload(wl, 1))
    om = P.oracle_model(Q2)
    for q, r in enumerate(wl.requests):
        ref = R.score_mis(om, otab, r)
        if r.K == 1:  # std of a single score is 0: the spread of the oracle's scores on this prefix
            tol = P.single_candidate_tolerance(Q2, om, otab, r, Q2_ITEMS)
            assert abs(got[q][0] - ref[0]) <= tol
            assert abs(got_ind[q][0] - ref[0]) <= tol
            continue
        P.assert_scores_match(Q2, got[q], ref, f"req {q}")
        P.assert_scores_match(Q2, got_ind[q], ref, f"req {q} independent")


def test_q2_multivector_items():
    # items of m = 8 table rows: a history item is the marker and its 8 VIDs,
    # a candidate branch is its 8 VIDs (b = 8), scored at the last one
    wl = W.custom_fir(Q2, Q2_ITEMS // 8, 901, 2, 3, 6, 12, 8)
    assert wl.n_items == Q2_ITEMS
    rk = P.ranker(Q2, Q2_ITEMS)
    otab = P.oracle_table(Q2, Q2_ITEMS)[0]
    om = P.oracle_model(Q2)
    got = P.split_scores(wl, rk.score_workload(wl))
    got_ind = P.split_scores(wl, rk.score_workload(wl, 1))
    for q, r in enumerate(wl.requests):
        ref = R.score_mis(om, otab, r)
        P.assert_scores_match(Q2, got[q], ref, f"req {q}")
        P.assert_scores_match(Q2, got_ind[q], ref, f"req {q} independent")


def test_graph_replay_matches_eager_and_is_deterministic():
    wl = W.custom(Q2, Q2_ITEMS, 321, 3, (1, 6), (3, 20), (5, 40), 1, n_instr=7)
    rk = P.ranker(Q2, Q2_ITEMS)
    rk.set_graph(True)
    a = rk.score_workload(wl)
    b = rk.score_workload(wl)
    rk.set_graph(False)
    c = rk.score_workload(wl)
    rk.set_graph(True)
    assert np.array_equal(a, b) and np.array_equal(a, c)
    # gather, then per layer QKV, attention, O, gate/up, down (the norms are
    # folded into the projections), then the score head; with the split-K O
    # and down projections of small capacities, each adds its reduction
    assert rk.launches_per_execute() in (1 + 5 * Q2.n_layers + 1, 1 + 7 * Q2.n_layers + 1)


def test_programmatic_dependent_launch_changes_no_result():
    # each kernel after the first may start while its predecessor finishes
    # and waits for its data itself: bit-identical scores with it on and off,
    # graph and eager, over batches that use both tile widths
    for seed, n_req in ((322, 3), (323, 24)):
        wl = W.custom(Q2, Q2_ITEMS, seed, n_req, (1, 6), (3, 20), (5, 40), 1, n_instr=7)
        rk = P.ranker(Q2, Q2_ITEMS)
        out = []
        for pdl in (True, False):
            rk.set_pdl(pdl)
            for graph in (True, False):
                rk.set_graph(graph)
                out.append(rk.score_workload(wl))
        rk.set_pdl(True)
        rk.set_graph(True)
        for o in out[1:]:
            assert np.array_equal(out[0], o)


def test_host_validation_errors():
    import shared_prefix_item_b200 as S
    rk = P.ranker(Q2, Q2_ITEMS)
    wl = W.custom(Q2, Q2_ITEMS, 331, 2, 2, 5, 4, 1, n_instr=2)
    p, po, b, co = wl.packed()
    bad = p.copy()
    bad[3] = Q2.vocab + Q2_ITEMS  # one past the last table row
    with pytest.raises(S.DuolmError) as e:
        rk.score(bad, po, b, co, 1)
    assert e.value.code == -2
    with pytest.raises(S.DuolmError) as e:
        rk.score(p, po, b, np.array([0, 4, 4]), 1)  # second request has K = 0
    assert e.value.code == -4
    with pytest.raises(S.DuolmError) as e:
        rk.score(p, np.array([1, 5, len(p)]), b, co, 1)
    assert e.value.code == -3
    with pytest.raises(S.DuolmError) as e:
        rk.score(p, po, np.zeros(8 * 129, np.int32), co, 129)  # branch longer than an item
    assert e.value.code == -1
    # the context is still usable
    ref = rk.score_workload(wl)
    assert np.isfinite(ref).all()


def test_bounded_wait_reports_timeout_and_context_survives():
    import shared_prefix_item_b200 as S
    rk = P.ranker(Q2, Q2_ITEMS)
    with pytest.raises(S.DuolmError) as e:
        rk.debug_wait_timeout()
    assert e.value.code == -7 and "wait-timeout" in str(e.value)
    wl = W.custom(Q2, Q2_ITEMS, 341, 1, 2, 5, 4, 1, n_instr=2)
    assert np.isfinite(rk.score_workload(wl)).all()


def test_fp16_range_guard():
    """Activations beyond fp16 range raise the device flag instead of
    silently turning into inf: gate and up weights scaled by 2^8 (exact)
    make silu(g) * u reach ~1e5 in layer 0."""
    import shared_prefix_item_b200 as S
    from synth.rng import bf16_round
    w = list(W.model_weights(Q2))
    for i in (9, 10):  # layer 0 w_gate, w_up
        w[i] = bf16_round(bf16_to_f32(w[i]) * 256.0)
    rk = S.Ranker(Q2, w)
    try:
        rk.vid_table_build(W.item_vectors(Q2_ITEMS, Q2.d), 0.0, 0.02)
        wl = W.custom(Q2, Q2_ITEMS, 351, 1, 2, 5, 4, 1, n_instr=2)
        with pytest.raises(S.DuolmError) as e:
            rk.score_workload(wl)
        assert e.value.code == -7 and "fp16-out-of-range" in str(e.value)
        # the flag is cleared once reported
        rk.debug_residual(0, wl.n_tokens)
    finally:
        rk.close()
