"""Pins for the oracle's routing metadata (CPU only).

A hand-worked example, the defining invariants (offsets are the cumulative
expert counts, rows of one expert are contiguous and in (token, slot) order,
every kept pair appears exactly once with its own weight), dropped slots, an
independent stable sort (numpy's lexsort), and the grouped product it feeds:
gathering x rows through row_token reproduces the per-token, per-slot product.
"""
import numpy as np

from oracle import routing as RO
from synth import generators as G


def test_hand_worked_example():
    ids = np.array([[2, 0], [0, 1], [2, 2]])            # T=3, k=2, E=3 (token 2 picks expert 2 twice)
    w = np.array([[0.5, 0.25], [1.0, 2.0], [3.0, 4.0]], np.float32)
    off, tok, wt, dst = RO.routing_metadata(ids, w, 3)
    assert off.tolist() == [0, 2, 3, 6]
    assert tok.tolist() == [0, 1, 1, 0, 2, 2]           # expert 0: (0,1), (1,0); expert 1: (1,1); expert 2: (0,0), (2,0), (2,1)
    assert dst.tolist() == [1, 2, 3, 0, 4, 5]
    assert wt.tolist() == [0.25, 1.0, 2.0, 0.5, 3.0, 4.0]


def test_invariants_on_random_routing():
    T, E, k = 300, 16, 4
    ids, w = G.route_softmax_topk(3, T, E, k)
    off, tok, wt, dst = RO.routing_metadata(ids, w, E)
    counts = np.bincount(ids.reshape(-1), minlength=E)
    assert np.array_equal(np.diff(off), counts)
    assert off[0] == 0 and off[-1] == T * k
    assert sorted(dst.tolist()) == list(range(T * k))    # every pair exactly once
    for r in range(T * k):
        t, s = divmod(int(dst[r]), k)
        assert tok[r] == t and wt[r] == w[t, s]
        e = int(np.searchsorted(off, r, side="right") - 1)
        assert ids[t, s] == e
    for e in range(E):                                   # (token, slot) order inside a group
        seg = dst[off[e]:off[e + 1]]
        assert np.all(np.diff(seg) > 0)


def test_matches_an_independent_stable_sort():
    T, E, k = 257, 64, 8
    ids, w = G.route_zipf_topk(5, T, E, k)
    off, tok, wt, dst = RO.routing_metadata(ids, w, E)
    flat = ids.reshape(-1)
    order = np.lexsort((np.arange(T * k), flat))         # by expert, then by pair index t*k + s
    assert np.array_equal(dst, order.astype(np.int32))
    assert np.array_equal(tok, (order // k).astype(np.int32))
    assert np.array_equal(wt, w.reshape(-1)[order])


def test_dropped_slots_get_no_row():
    ids = np.array([[0, -1], [5, 1], [1, 0]])            # E = 2: -1 and 5 are dropped
    w = np.ones((3, 2), np.float32)
    off, tok, wt, dst = RO.routing_metadata(ids, w, 2)
    assert off.tolist() == [0, 2, 4]
    assert dst.tolist() == [0, 5, 3, 4]


def test_feeds_the_grouped_product():
    """x gathered through row_token, weighted and scattered to row_dest gives, per
    (token, slot), the weighted product with that slot's expert."""
    T, E, k, K, N = 20, 5, 3, 8, 4
    ids, w = G.route_softmax_topk(7, T, E, k)
    off, tok, wt, dst = RO.routing_metadata(ids, w, E)
    rng = np.random.default_rng(8)
    x = rng.standard_normal((T, K))
    Ws = rng.standard_normal((E, N, K))
    out = np.zeros((T * k, N))
    for e in range(E):
        r = np.arange(off[e], off[e + 1])
        out[dst[r]] = (x[tok[r]] @ Ws[e].T) * wt[r][:, None]
    for t in range(T):
        for s in range(k):
            want = w[t, s] * (Ws[ids[t, s]] @ x[t])
            assert np.allclose(out[t * k + s], want)


def test_empty():
    off, tok, wt, dst = RO.routing_metadata(np.zeros((0, 4), np.int64), np.zeros((0, 4), np.float32), 3)
    assert off.tolist() == [0, 0, 0, 0] and len(tok) == 0
