"""Prefix KV reuse (incremental history append) against the oracle.

A causal prefix's K/V at every layer depend only on the tokens before them,
so a call that starts from the K/V an earlier call stored for the first c
prefix tokens must score like a call over the whole sequence (DuoLM summary
page, 未来方向 (3): new history items add only their own vectors and K/V).
Every expected score here is the oracle's score of the whole prefix; the
cached lengths cross the 128-key tiles of the tensor-core attention (exactly
128, one past, ragged) and the store slots are reused, rolled back and
shared read-only."""
import dataclasses

import numpy as np
import pytest

from oracle import ranker as R
from synth import workloads as W

import parity as P

pytestmark = pytest.mark.gpu

TINY = W.TINY
Q2 = dataclasses.replace(W.QWEN3_06B, n_layers=2, vocab=4096, name="qwen3-shape-2layer")
Q2_ITEMS = 1000
ITEMS = {TINY: 64, Q2: Q2_ITEMS}


@pytest.fixture
def store_ranker(request):
    shape = request.param
    rk = P.ranker(shape, ITEMS[shape])
    rk.kv_store_reserve(6, 640)
    yield shape, rk
    rk.kv_store_reserve(0, 0)  # the cached ranker goes back to its plain state


def _oracle(shape, prefix, branch):
    return R.score_mis(P.oracle_model(shape), P.oracle_table(shape, ITEMS[shape])[0], W.Request(prefix, branch))


def _long_request(shape, seed, L, K, b):
    wl = W.custom(shape, ITEMS[shape], seed, 1, 0, 1, K, b, n_instr=L)
    r = wl.requests[0]
    assert r.L == L
    return r.prefix_ids, r.branch_ids


def _one(rk, prefix_new, branch, b, slot, cached, keep):
    return rk.score_cached(prefix_new, [0, len(prefix_new)], branch.reshape(-1), [0, branch.shape[0]], b, [slot],
                           [cached], [keep])


@pytest.mark.parametrize("store_ranker", [TINY, Q2], indirect=True, ids=["fp32", "bf16"])
def test_append_in_steps_rescore_and_roll_back(store_ranker):
    shape, rk = store_ranker
    b = 2
    prefix, branch = _long_request(shape, 301, 300, 24, b)
    _, branch2 = _long_request(shape, 302, 1, 17, b)
    # 1: the first 37 tokens from scratch, all kept
    got = _one(rk, prefix[:37], branch, b, 3, 0, 37)
    P.assert_scores_match(shape, got, _oracle(shape, prefix[:37], branch), "37 from scratch")
    assert rk.kv_slot_length(3) == 37
    # 2: append up to 128 (the store's first tile exactly full), keep them
    got = _one(rk, prefix[37:128], branch, b, 3, 37, 91)
    P.assert_scores_match(shape, got, _oracle(shape, prefix[:128], branch), "append to 128")
    assert rk.kv_slot_length(3) == 128
    # 3: append to 300 keeping only up to 129: one row into the second tile
    got = _one(rk, prefix[128:300], branch, b, 3, 128, 1)
    P.assert_scores_match(shape, got, _oracle(shape, prefix[:300], branch), "append to 300")
    assert rk.kv_slot_length(3) == 129
    # 4: continue from 129 and keep everything
    got = _one(rk, prefix[129:300], branch, b, 3, 129, 171)
    P.assert_scores_match(shape, got, _oracle(shape, prefix[:300], branch), "append from 129")
    assert rk.kv_slot_length(3) == 300
    # 5: new candidates for the unchanged prefix: no new prefix token
    got = _one(rk, prefix[:0], branch2, b, 3, 300, 0)
    P.assert_scores_match(shape, got, _oracle(shape, prefix, branch2), "rescore")
    assert rk.kv_slot_length(3) == 300
    # 6: roll back to 200 and continue with other tokens
    other = prefix[::-1][:60].copy()
    seq = np.concatenate([prefix[:200], other])
    got = _one(rk, other, branch, b, 3, 200, 60)
    P.assert_scores_match(shape, got, _oracle(shape, seq, branch), "roll back to 200")
    assert rk.kv_slot_length(3) == 260
    # the uncached call on the same context still agrees
    got = rk.score(seq, [0, len(seq)], branch.reshape(-1), [0, branch.shape[0]], b)
    P.assert_scores_match(shape, got, _oracle(shape, seq, branch), "uncached")


@pytest.mark.parametrize("store_ranker", [TINY, Q2], indirect=True, ids=["fp32", "bf16"])
def test_mixed_batch(store_ranker):
    """One batch: requests on their own slots with cached lengths 1, 127, 128,
    129 and 255, one without a slot, two sharing a slot read-only."""
    shape, rk = store_ranker
    b = 3
    cuts = [1, 127, 128, 129, 255]
    reqs = [_long_request(shape, 400 + i, c + 20 + 7 * i, 5 + 3 * i, b) for i, c in enumerate(cuts)]
    # warm the slots: each request's first `cut` tokens, stored
    pre = [p[:c] for (p, _), c in zip(reqs, cuts)]
    brs = [br for _, br in reqs]
    poff = np.cumsum([0] + [len(x) for x in pre])
    coff = np.cumsum([0] + [x.shape[0] for x in brs])
    got = rk.score_cached(np.concatenate(pre), poff, np.concatenate([x.reshape(-1) for x in brs]), coff, b,
                          list(range(5)), [0] * 5, cuts)
    for q, (c, (p, br)) in enumerate(zip(cuts, reqs)):
        P.assert_scores_match(shape, got[coff[q]:coff[q + 1]], _oracle(shape, p[:c], br), f"warm {q}")
    # the batch: the five continue their prefixes (slot 4 shared by request 6,
    # which reads 100 of its tokens), request 5 has no slot
    plain_p, plain_b = _long_request(shape, 450, 77, 9, b)
    shared_new = np.array([5, 6, 7, 8, 9], np.int32)
    news = [p[c:] for (p, _), c in zip(reqs, cuts)] + [plain_p, shared_new]
    brs = brs + [plain_b, brs[4][:4]]
    slots = [0, 1, 2, 3, 4, -1, 4]
    cached = cuts + [0, 100]
    keep = [0] * 7
    poff = np.cumsum([0] + [len(x) for x in news])
    coff = np.cumsum([0] + [x.shape[0] for x in brs])
    got = rk.score_cached(np.concatenate(news), poff, np.concatenate([x.reshape(-1) for x in brs]), coff, b, slots,
                          cached, keep)
    full = [p for p, _ in reqs] + [plain_p, np.concatenate([reqs[4][0][:100], shared_new])]
    for q in range(7):
        P.assert_scores_match(shape, got[coff[q]:coff[q + 1]], _oracle(shape, full[q], brs[q]), f"request {q}")
    for s, c in enumerate(cuts):
        assert rk.kv_slot_length(s) == c  # keep = 0 leaves the slots as they were


@pytest.mark.parametrize("store_ranker", [Q2], indirect=True, ids=["bf16"])
def test_graph_eager_and_repeated_execute(store_ranker):
    """The appending batch runs three times (the append rewrites the same
    rows), with the CUDA graph and with eager launches."""
    shape, rk = store_ranker
    p, br = _long_request(shape, 500, 260, 30, 1)
    ref = _oracle(shape, p, br)
    try:
        for graph in (True, False):
            rk.set_graph(graph)
            rk.prepare_cached(p[:140], [0, 140], br.reshape(-1), [0, 30], 1, [0], [0], [140])
            for _ in range(3):
                rk.execute()
            rk.sync()
            assert rk.kv_slot_length(0) == 140
            got = _one(rk, p[140:], br, 1, 0, 140, 0)
            P.assert_scores_match(shape, got, ref, f"graph={graph}")
    finally:
        rk.set_graph(True)


def test_errors():
    import shared_prefix_item_b200 as S
    rk = P.ranker(Q2, Q2_ITEMS)
    p, br = _long_request(Q2, 600, 50, 4, 1)
    brf = br.reshape(-1)

    def code(slot, cached, keep, prefix=p):
        with pytest.raises(S.DuolmError) as e:
            rk.score_cached(prefix, [0, len(prefix)], brf, [0, 4], 1, [slot], [cached], [keep])
        return e.value.code

    rk.kv_store_reserve(0, 0)
    assert code(0, 0, 0) == -8                  # no store reserved
    rk.kv_store_reserve(2, 64)
    try:
        assert code(2, 0, 0) == -1              # slot out of range
        assert code(0, 1, 0) == -8              # the slot holds nothing yet
        assert code(0, 0, 51) == -1             # keep above the new tokens
        assert code(0, 0, -1) == -1
        assert code(-1, 3, 0) == -1             # cached without a slot
        assert code(0, 0, 0, prefix=p[:0]) == -4  # nothing at all before the branches
        rk.score_cached(p, [0, 50], brf, [0, 4], 1, [0], [0], [50])
        assert rk.kv_slot_length(0) == 50
        assert code(0, 20, 45) == -5            # 65 rows in a 64-row slot
        with pytest.raises(S.DuolmError) as e:  # a slot written by one request and read by another
            rk.score_cached(np.concatenate([p[:5], p[:5]]), [0, 5, 10], np.concatenate([brf, brf]), [0, 4, 8], 1,
                            [1, 1], [0, 0], [5, 0])
        assert e.value.code == -1
        with pytest.raises(S.DuolmError):
            rk.kv_slot_length(5)
        # a failed call left the slot as it was
        assert rk.kv_slot_length(0) == 50
    finally:
        rk.kv_store_reserve(0, 0)


def test_c64_history_append_matches_full_recompute():
    """The 64-request batch at full size: every request's history minus its
    last item and header is stored first; the timed-path call appends the
    rest.  Against the uncached scores of the same batch (and the oracle on
    two sampled requests)."""
    Q = W.QWEN3_06B
    wl = W.c64()
    rk = P.ranker(Q, wl.n_items)
    try:
        full = rk.score_workload(wl)
        rk.kv_store_reserve(64, 1536)
        cuts = [wl.history_offsets(q)[-1] for q in range(64)]  # before each last history item
        p, po, b, co = wl.packed()
        warm = np.concatenate([r.prefix_ids[:c] for r, c in zip(wl.requests, cuts)])
        wpo = np.cumsum([0] + cuts)
        rk.score_cached(warm, wpo, b, co, wl.branch_len, np.arange(64), np.zeros(64), cuts)
        rest = np.concatenate([r.prefix_ids[c:] for r, c in zip(wl.requests, cuts)])
        rpo = np.cumsum([0] + [r.L - c for r, c in zip(wl.requests, cuts)])
        got = rk.score_cached(rest, rpo, b, co, wl.branch_len, np.arange(64), cuts, np.zeros(64))
        gs, fs = P.split_scores(wl, got), P.split_scores(wl, full)
        for q in range(64):
            P.assert_scores_match(Q, gs[q], fs[q].astype(np.float64), f"request {q} cached vs uncached")
        om, otab = P.oracle_model(Q), P.oracle_table(Q, wl.n_items)[0]
        Ls = [r.L for r in wl.requests]
        for q in sorted({int(np.argmax(Ls)), 17}):
            P.assert_scores_match(Q, gs[q], R.score_mis(om, otab, wl.requests[q]), f"request {q} vs oracle")
    finally:
        rk.kv_store_reserve(0, 0)



@pytest.mark.parametrize("store_ranker", [TINY, Q2], indirect=True, ids=["fp32", "bf16"])
def test_every_request_reads_one_shared_template_slot(store_ranker):
    # the instruction every prompt of a recipe starts with, stored once and
    # read by all requests of a batch (the exact part of cross-request prefix
    # sharing, Summary page 未来方向 (5)): every score equals the oracle's over
    # the whole prefix
    shape, rk = store_ranker
    wl = W.custom(shape, ITEMS[shape], 341, 5, (1, 6), (3, 20), (5, 40), 1, n_instr=40, n_header=3)
    n = 40
    r0 = wl.requests[0]
    for r in wl.requests:
        assert np.array_equal(r.prefix_ids[:n], r0.prefix_ids[:n])
    # store the instruction in slot 3 (scoring request 0's candidates once)
    _one(rk, r0.prefix_ids[:n], r0.branch_ids, 1, 3, 0, n)
    assert rk.kv_slot_length(3) == n
    new = np.concatenate([r.prefix_ids[n:] for r in wl.requests])
    off = np.cumsum([0] + [r.L - n for r in wl.requests])
    _, _, b, co = wl.packed()
    R_ = len(wl.requests)
    got = P.split_scores(wl, rk.score_cached(new, off, b, co, 1, [3] * R_, [n] * R_, [0] * R_))
    assert rk.kv_slot_length(3) == n  # read only
    for q, r in enumerate(wl.requests):
        ref = _oracle(shape, r.prefix_ids, r.branch_ids)
        P.assert_scores_match(shape, got[q], ref, f"request {q}")
