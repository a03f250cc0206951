"""Plain CPU oracle for the routing metadata of a grouped call.

TEST INFRASTRUCTURE ONLY, like ``gnf4_oracle``: only the tests and the bench's
CPU baseline leg use it, and it shares no code with the CUDA path.

Passages: the solution page, "Supported scope" (the grouped call takes the
routed rows grouped by expert -- ``a_cat`` "group-sorted" -- and "sort and
scatter live outside the kernel"; ``build_group_tiles_device`` builds the
call's tile table on the device so that it can be captured), and the same
page's "Smallest correct example" (``sizes`` per expert, rows of one expert
contiguous).

Definition (reading 20): from the router's choices ``ids [T, k]`` (expert of
slot s of token t) and ``weights [T, k]``, the routed rows are the T*k pairs
(t, s) ordered by expert, and within one expert by t, then s (the order in
which the pairs appear in ``ids`` read row by row: a stable counting sort).
Routed row r of that order has ``row_token[r] = t``, ``row_weight[r] =
weights[t, s]``, ``row_dest[r] = t*k + s``, and expert e owns the rows
``[expert_offsets[e], expert_offsets[e+1])``. An id outside ``[0, E)`` is a
dropped slot: it gets no row.
"""
from __future__ import annotations

import numpy as np


def routing_metadata(ids: np.ndarray, weights: np.ndarray, E: int):
    """Counting sort written out: returns (expert_offsets int64 [E+1], row_token int32 [R],
    row_weight float32 [R], row_dest int32 [R])."""
    ids = np.asarray(ids, dtype=np.int64)
    weights = np.asarray(weights, dtype=np.float32)
    T, k = ids.shape
    counts = [0] * E
    for t in range(T):
        for s in range(k):
            e = int(ids[t, s])
            if 0 <= e < E:
                counts[e] += 1
    offsets = np.zeros(E + 1, dtype=np.int64)
    for e in range(E):
        offsets[e + 1] = offsets[e] + counts[e]
    R = int(offsets[E])
    row_token = np.zeros(R, dtype=np.int32)
    row_weight = np.zeros(R, dtype=np.float32)
    row_dest = np.zeros(R, dtype=np.int32)
    fill = [int(offsets[e]) for e in range(E)]
    for t in range(T):                      # pairs in (t, s) order: stable within each expert
        for s in range(k):
            e = int(ids[t, s])
            if 0 <= e < E:
                r = fill[e]
                fill[e] += 1
                row_token[r] = t
                row_weight[r] = weights[t, s]
                row_dest[r] = t * k + s
    return offsets, row_token, row_weight, row_dest
