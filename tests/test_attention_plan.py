"""The tensor-core attention's work list and CTA schedule (host logic, CPU).

Every (request, KV head) must have its query rows covered exactly once: the
prefix rows from the request's cached length c to L by kind-0 items, the
branch rows by kind-1 items that hold whole candidates (a candidate's keys
are its own branch rows, so it cannot be split across items).  The CTA
ranges partition the list, and the greedy list schedule leaves no CTA more
than one item's estimated cost above the least loaded one."""
import numpy as np
import pytest

from synth import workloads as W


@pytest.fixture(scope="module")
def S():
    import shared_prefix_item_b200 as S
    return S


def _cost(L, K, c, b, Rw, kind, row0):
    """The schedule's per-item estimate: key tiles, +20% with the second
    sub-tile in use, +half a tile to start."""
    per = (Rw // b) * b
    nrows = min(per, K * b - row0) if kind else min(Rw, L - row0)
    kend = L if kind else min(row0 + Rw, L)
    tiles = -(-c // 128) + -(-(kend - c) // 128) + (-(-nrows // 128) if kind else 0)
    return 10 * tiles + (2 * tiles if nrows > Rw // 2 else 0) + 5


def _check(S, L, K, cached, b, H, Rw, n_ctas):
    items, cta = S.attention_plan(L, K, cached, b, H, Rw, n_ctas)
    per = (Rw // b) * b
    n = len(items)
    assert cta[0] == 0 and cta[-1] == n and np.all(np.diff(cta) >= 0)
    seen_prefix = {}
    seen_branch = {}
    for r_, h, kind, row0 in items:
        assert 0 <= h < H
        if kind == 0:
            assert cached[r_] <= row0 < L[r_]
            rows = range(row0, min(row0 + Rw, L[r_]))
            seen_prefix.setdefault((r_, h), []).extend(rows)
        else:
            assert kind == 1 and row0 % b == 0 and 0 <= row0 < K[r_] * b
            end = min(row0 + per, K[r_] * b)
            assert (end - row0) % b == 0  # whole candidates
            seen_branch.setdefault((r_, h), []).extend(range(row0, end))
    for r_ in range(len(L)):
        for h in range(H):
            assert sorted(seen_prefix.get((r_, h), [])) == list(range(cached[r_], L[r_]))
            assert sorted(seen_branch[(r_, h)]) == list(range(K[r_] * b))
    loads = []
    for c in range(n_ctas):
        loads.append(sum(_cost(L[i[0]], K[i[0]], cached[i[0]], b, Rw, i[2], i[3]) for i in items[cta[c]:cta[c + 1]]))
    max_item = max(_cost(L[i[0]], K[i[0]], cached[i[0]], b, Rw, i[2], i[3]) for i in items)
    assert max(loads) - min(loads) <= max_item
    return items, cta


def test_c64_batch_on_148_ctas(S):
    wl = W.c64()
    L = [r.L for r in wl.requests]
    K = [r.K for r in wl.requests]
    items, _ = _check(S, L, K, [0] * 64, 1, 8, 128, 148)
    # per (request, KV head): ceil(L / 128) prefix items and one branch item of 100 rows
    assert len(items) == 8 * sum(-(-l // 128) + 1 for l in L)


def test_cached_prefixes_and_empty_new_prefix(S):
    wl = W.c64(n_requests=12)
    L = [r.L for r in wl.requests]
    K = [r.K for r in wl.requests]
    cached = [0, 1, 127, 128, 129, L[5], L[6] - 1, 300 if L[7] > 300 else 0, 64, 0, 255 if L[10] > 255 else 3, 2]
    _check(S, L, K, cached, 1, 8, 128, 148)


@pytest.mark.parametrize("b,H,Rw,n_ctas", [(3, 8, 128, 148), (4, 8, 128, 7), (8, 8, 128, 148), (1, 16, 256, 148),
                                           (5, 4, 64, 3), (64, 2, 64, 148)])
def test_branch_lengths_groupings_and_cta_counts(S, b, H, Rw, n_ctas):
    rng = np.random.default_rng(b * 1000 + Rw)
    R = 9
    L = [int(x) for x in rng.integers(1, 700, R)]
    K = [int(x) for x in rng.integers(1, 300, R)]
    cached = [int(rng.integers(0, l + 1)) if i % 2 else 0 for i, l in enumerate(L)]
    cached = [c if c < l else l for c, l in zip(cached, L)]
    _check(S, L, K, cached, b, H, Rw, n_ctas)


def test_capacity_and_arguments(S):
    from shared_prefix_item_b200 import _lib
    L = np.array([300, 40], np.int32)
    K = np.array([100, 3], np.int32)
    c = np.zeros(2, np.int32)
    items, _ = S.attention_plan(L, K, c, 1, 8, 128, 148)
    need = len(items)
    buf = np.zeros((need, 4), np.int32)
    cta = np.zeros(149, np.int32)
    f = _lib.lib.duolm_debug_attention_plan
    assert f(2, _lib._p(L), _lib._p(K), _lib._p(c), 1, 8, 128, 148, _lib._p(buf), need - 1, _lib._p(cta)) == -5
    assert f(2, _lib._p(L), _lib._p(K), _lib._p(c), 1, 8, 128, 148, _lib._p(buf), need, _lib._p(cta)) == need
    assert np.array_equal(buf, items)
    bad = np.array([301, 40], np.int32)  # cached above L
    assert f(2, _lib._p(L), _lib._p(K), _lib._p(bad), 1, 8, 128, 148, _lib._p(buf), need, _lib._p(cta)) == -1
    assert f(2, _lib._p(L), _lib._p(K), _lib._p(c), 129, 8, 128, 148, _lib._p(buf), need, _lib._p(cta)) == -1
