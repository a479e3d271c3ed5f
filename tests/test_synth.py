"""Seeded synthetic input generators (no method arithmetic here)."""
import numpy as np

from synth import workloads as W


def test_zipf_lookup_stream_is_seeded_and_zipf_shaped():
    # the standalone gather's id stream: deterministic, in range, and its top
    # ranks appear with the Zipf(1.1) probabilities k^-1.1 / H
    n, rows = 400_000, 100_000
    a = W.zipf_lookups(n, rows)
    assert np.array_equal(a, W.zipf_lookups(n, rows))
    assert a.min() >= 0 and a.max() < rows
    H = np.sum(np.arange(1, rows + 1, dtype=np.float64) ** -1.1)
    counts = np.bincount(a, minlength=rows)
    for k in (1, 2, 10):
        p = k ** -1.1 / H
        assert abs(counts[k - 1] / n - p) < 5 * np.sqrt(p / n), k


def test_item_vector_rows_do_not_depend_on_the_draw_length():
    # the GPU parity tests draw only the rows up to the largest one a request
    # touches: the stream is counter-based, so those rows equal the full draw's
    assert np.array_equal(W.item_vectors(300, 64), W.item_vectors(1000, 64)[:300])
