"""duolm_compile, the host-side request compiler: request records (item ids,
feedback tokens) in, the packed ranker sequences out.  Runs on CPU.

The expected arrays are the ones the seeded request generator writes while
it draws each request (the prefix and branch ids every parity test and the
bench feed the kernels), so the compiler must reproduce them exactly from
the records alone: instruction, per history item the marker, the item's
VIDs and its feedback tokens, the header; per candidate the branch header
and the candidate's VIDs (DuoLM summary page, 方法步骤详情 steps 3-4)."""
import numpy as np
import pytest

from synth import workloads as W


@pytest.fixture(scope="module")
def S():
    import shared_prefix_item_b200 as S
    return S


def _compile(S, wl, n_threads=0, **over):
    t = wl.template
    hist, hoff, fb, foff, cand, coff = wl.records()
    args = dict(vocab=wl.model.vocab, marker=t.marker, m=wl.m, instr=t.instr, header=t.header,
                branch_header=t.branch_header[: wl.branch_len - wl.m], hist_items=hist, hist_offsets=hoff,
                feedback=fb, feedback_offsets=foff, cand_items=cand, cand_offsets=coff,
                n_items=wl.n_items // wl.m, n_threads=n_threads)
    args.update(over)
    return S.compile_requests(**args)


def _check(S, wl, n_threads=0):
    prefix, poff, branch, coff, b = _compile(S, wl, n_threads)
    want = wl.packed()
    assert b == wl.branch_len
    assert np.array_equal(poff, want[1])
    assert np.array_equal(prefix, want[0])
    assert np.array_equal(coff, want[3])
    assert np.array_equal(branch, want[2])


@pytest.mark.parametrize("name", ["tiny", "c1", "c64", "stress"])
def test_compiled_requests_match_the_generated_sequences(S, name):
    _check(S, W.CONFIGS[name]())


def test_multi_vector_items(S):
    _check(S, W.fir(m=8, n_requests=16))


def test_zipf_catalog_and_shards(S):
    _check(S, W.catalog(8, shard=1))
    _check(S, W.c64(n_requests=9, shard=3))


@pytest.mark.parametrize("n_threads", [1, 2, 3, 64, 1000])
def test_thread_count_does_not_change_the_output(S, n_threads):
    _check(S, W.c64(n_requests=23), n_threads)


def test_ragged_with_branch_header_and_empty_history(S):
    wl = W.custom(W.QWEN3_06B, 5000, 77, 12, (0, 6), (0, 9), (1, 40), 3, n_header=2,
                  random_branch_header=False)
    assert any(len(r.history_items) == 0 for r in wl.requests)
    _check(S, wl)


def _code(S, wl, **over):
    with pytest.raises(S.DuolmError) as e:
        _compile(S, wl, **over)
    return e.value.code


def test_errors(S):
    wl = W.c64(n_requests=4)
    hist, hoff, fb, foff, cand, coff = wl.records()
    bad = cand.copy()
    bad[7] = wl.n_items
    assert _code(S, wl, cand_items=bad) == -2            # item id one past the table
    bad = hist.copy()
    bad[-1] = -1
    assert _code(S, wl, hist_items=bad) == -2
    bad = fb.copy()
    bad[3] = wl.model.vocab                              # a feedback token that is an item id
    assert _code(S, wl, feedback=bad) == -2
    assert _code(S, wl, marker=wl.model.vocab) == -2
    assert _code(S, wl, instr=np.array([1, -4])) == -2
    bad = coff.copy()
    bad[2] = bad[1] - 1
    assert _code(S, wl, cand_offsets=bad) == -3          # decreasing
    bad = foff.copy()
    bad[0] = 1
    assert _code(S, wl, feedback_offsets=bad) == -3      # not starting at 0
    bad = coff.copy()
    bad[2] = bad[1]
    assert _code(S, wl, cand_offsets=bad) == -4          # a request without candidates
    assert _code(S, wl, m=0) == -1


def test_capacity_is_checked_before_writing(S):
    import ctypes
    from shared_prefix_item_b200 import _lib
    wl = W.c64(n_requests=3)
    t = wl.template
    hist, hoff, fb, foff, cand, coff = wl.records()
    want = wl.packed()
    ins, hdr = np.ascontiguousarray(t.instr, np.int32), np.ascontiguousarray(t.header, np.int32)
    tpl = _lib.Template(wl.model.vocab, t.marker, 1, ins.ctypes.data, len(ins), hdr.ctypes.data, len(hdr), None, 0)
    L, C = len(want[0]), len(want[2])
    for pcap, bcap in [(L - 1, C), (L, C - 1)]:
        prefix = np.full(L, -9, np.int32)
        branch = np.full(C, -9, np.int32)
        poff = np.zeros(4, np.int64)
        rc = _lib.lib.duolm_compile(ctypes.byref(tpl), 3, _lib._p(hist), _lib._p(hoff), _lib._p(fb), _lib._p(foff),
                                    _lib._p(cand), _lib._p(coff), wl.n_items, 2, _lib._p(prefix), pcap,
                                    _lib._p(poff), _lib._p(branch), bcap)
        assert rc == -5
        assert b"capacity" in _lib.lib.duolm_last_error(None)
        assert np.all(prefix == -9) and np.all(branch == -9)
        # the append form leaves its cached / keep outputs untouched as well
        hc = np.zeros(3, np.int32)
        cached = np.full(3, -9, np.int32)
        keep = np.full(3, -9, np.int32)
        rc = _lib.lib.duolm_compile_append(ctypes.byref(tpl), 3, _lib._p(hist), _lib._p(hoff), _lib._p(fb),
                                           _lib._p(foff), _lib._p(cand), _lib._p(coff), wl.n_items, 2, _lib._p(hc),
                                           _lib._p(prefix), pcap, _lib._p(poff), _lib._p(branch), bcap,
                                           _lib._p(cached), _lib._p(keep))
        assert rc == -5
        assert np.all(cached == -9) and np.all(keep == -9)
        assert np.all(prefix == -9) and np.all(branch == -9)


def test_thread_count_above_the_host_threads_is_capped(S):
    # a caller asking for far more workers than the host has gets the same
    # output (the count is capped at the hardware threads, not honoured)
    wl = W.c64(n_requests=64)
    hist, hoff, fb, foff, cand, coff = wl.records()
    t = wl.template
    out = S.compile_requests(wl.model.vocab, t.marker, 1, t.instr, t.header, t.branch_header[:0], hist, hoff, fb,
                             foff, cand, coff, wl.n_items, 100000)
    want = wl.packed()
    assert np.array_equal(out[0], want[0]) and np.array_equal(out[2], want[2])


def _append_expected(wl, hc):
    """What the store already holds and what is left, from the generated
    sequences: with h > 0 items stored the slot holds everything before
    item h (the instruction and items 0..h-1); h = 0 is an empty slot."""
    n_header = len(wl.template.header)
    news, cached, keep = [], [], []
    for q, r in enumerate(wl.requests):
        h = hc[q]
        offs = wl.history_offsets(q) + [r.L - n_header]
        c = offs[h] if h > 0 else 0
        news.append(r.prefix_ids[c:])
        cached.append(c)
        keep.append(0 if h < 0 else r.L - n_header - c)
    return np.concatenate(news), cached, keep


@pytest.mark.parametrize("recipe", ["c64", "fir"])
def test_compile_append_matches_the_generated_sequences(S, recipe):
    wl = W.c64(n_requests=16) if recipe == "c64" else W.fir(m=8, n_requests=16)
    n_hist = [len(r.history_items) for r in wl.requests]
    rng = np.random.default_rng(5)
    hc = [-1, 0] + [int(rng.integers(0, n + 1)) for n in n_hist[2:]]
    hc[2] = n_hist[2]          # every item stored: only the header is new
    hc[3] = n_hist[3] - 1      # the next item arrives
    hist, hoff, fb, foff, cand, coff = wl.records()
    t = wl.template
    prefix, poff, branch, coff2, b, cached, keep = S.compile_requests(
        wl.model.vocab, t.marker, wl.m, t.instr, t.header, t.branch_header[: wl.branch_len - wl.m], hist, hoff, fb,
        foff, cand, coff, wl.n_items // wl.m, 3, hist_cached=hc)
    want_ids, want_cached, want_keep = _append_expected(wl, hc)
    assert np.array_equal(prefix, want_ids)
    assert list(cached) == want_cached and list(keep) == want_keep
    assert np.array_equal(branch, wl.packed()[2])
    # the whole prefix is the stored part followed by the compiled part
    for q, r in enumerate(wl.requests):
        assert poff[q + 1] - poff[q] + cached[q] == r.L


def test_compile_append_rejects_bad_counts(S):
    wl = W.c64(n_requests=3)
    hist, hoff, fb, foff, cand, coff = wl.records()
    t = wl.template
    n0 = len(wl.requests[0].history_items)
    for bad in ([n0 + 1, 0, 0], [-2, 0, 0]):
        with pytest.raises(S.DuolmError) as e:
            S.compile_requests(wl.model.vocab, t.marker, 1, t.instr, t.header, t.branch_header[:0], hist, hoff, fb,
                               foff, cand, coff, wl.n_items, 1, hist_cached=bad)
        assert e.value.code == -1
