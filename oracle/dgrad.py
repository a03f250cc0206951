"""Plain CPU oracle for the input gradient of the grouped 4-bit GEMM.

TEST INFRASTRUCTURE ONLY, like ``gnf4_oracle``: only the tests,
``__graft_entry__.smoke()`` and the bench's CPU baseline leg use it, and it
shares no code with the CUDA path.

Passage: the grouped-nf4-gemm README (0.11.0), "Training: the backward is a
kernel too (0.7.0)": ``dgrad_4bit_grouped`` is the input gradient
``grad_out @ dequant(B)`` of every group in one launch, with the same on-chip
decode as the forward and nothing materialised; its fp32 accumulation lands
near 2.9e-3 of the exact per-expert loop. The solution page, "Supported scope",
lists ``dgrad_4bit_grouped(grad_out, B, absmax, sizes, expert_ids)`` as the
training entry point.

For a forward ``y[dest(r)] = w(r) * x[tok(r)] @ What[e(r)].T`` (``What[e]`` of
shape ``[N, K]``), the gradient of the routed input row r is

    dx[r, k] = w(r) * sum_n g[src(r), n] * What[e(r), n, k]

with ``src(r)`` the row of ``grad_out`` that belongs to routed row r (``dest(r)``
of the forward; ``r`` when the gradient is already in routed order) and ``w(r)``
the forward's routing weight (1 when none). Exact arithmetic (fp64), one bf16
rounding at the end.

Reading 19 (the pages print no formula for the scale's place): the contraction
runs over N, across the rows that carry different block scales, so the scale
cannot be applied to finished block sums as in the forward; the oracle simply
uses the exact dequantized weights.
"""
from __future__ import annotations

import numpy as np

from .gnf4_oracle import bf16_bits, bf16_to_f64, decode_expert


def dgrad_rows_f64(fmt, g_bits, W, S, offsets, row_src, row_weight, rows):
    """Unrounded fp64 gradients of the routed rows listed in ``rows`` (any order):
    ``[len(rows), K]``."""
    rows = np.asarray(rows, dtype=np.int64)
    offsets = np.asarray(offsets, dtype=np.int64)
    g = bf16_to_f64(g_bits)
    K = W.shape[2] * 2
    out = np.empty((len(rows), K), dtype=np.float64)
    experts = np.searchsorted(offsets, rows, side="right") - 1
    for e in np.unique(experts):
        sel = np.nonzero(experts == e)[0]
        r = rows[sel]
        src = r if row_src is None else np.asarray(row_src, dtype=np.int64)[r]
        acc = g[src] @ decode_expert(fmt, W, S, int(e), K)      # [m, N] @ [N, K]
        if row_weight is not None:
            acc = acc * np.asarray(row_weight, dtype=np.float64)[r][:, None]
        out[sel] = acc
    return out


def dgrad(fmt, g_bits, W, S, offsets, row_src=None, row_weight=None):
    """The whole input gradient, bf16 bit patterns ``[R, K]`` in routed order."""
    R = int(np.asarray(offsets)[-1])
    if R == 0:
        return np.zeros((0, W.shape[2] * 2), dtype=np.uint16)
    return bf16_bits(dgrad_rows_f64(fmt, g_bits, W, S, offsets, row_src, row_weight, np.arange(R)))
