"""Seeded generators for weights, activations and routed token groups.

Every draw is keyed by an explicit seed (and, for expert weights, by the
expert index), so any single expert can be regenerated without drawing the
whole stack. Recipes (they follow the workloads the grouped-nf4-gemm pages
measure on; no checkpoint or dataset is used):

* expert weights: fp32 N(0, 0.02), one ``[N, K]`` matrix per expert;
* activations: N(0, 1) drawn in fp32, stored as bf16 (round to nearest even);
* routing: top-k of softmax(N(0, 1) logits) per token, or a Zipf(s)-skewed
  draw of k distinct experts per token (Gumbel top-k of log p);
* routing metadata: the T*k routed rows sorted by (expert, token, slot), with
  per-expert int64 offsets, the token each row reads, its routing weight and
  the slot-major destination row ``t*k + slot``.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Optional

import numpy as np

_TAGS = {"w": 1, "x": 2, "route": 3, "w_down": 4, "x_down": 5, "h": 6, "y": 7, "misc": 9}


def _rng(*key: int) -> np.random.Generator:
    return np.random.default_rng([int(k) for k in key])


# --------------------------------------------------------------------------
# bf16 storage helpers (input preparation only)
# --------------------------------------------------------------------------
def bf16_bits_from_f32(a: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 bit patterns (uint16), round to nearest even; NaN stays NaN."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    u = a.view(np.uint32).astype(np.uint64)
    bias = ((u >> 16) & 1) + 0x7FFF
    r = ((u + bias) >> 16).astype(np.uint16)
    nan = np.isnan(a)
    if nan.any():
        r[nan] = ((u[nan] >> 16) | 0x40).astype(np.uint16)
    return r


def f32_from_bf16_bits(b: np.ndarray) -> np.ndarray:
    """bf16 bit patterns (uint16) -> fp32 values (exact widening)."""
    b = np.ascontiguousarray(b, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32)


# --------------------------------------------------------------------------
# weights and activations
# --------------------------------------------------------------------------
def expert_weights(seed: int, e: int, N: int, K: int, tag: str = "w",
                   std: float = 0.02) -> np.ndarray:
    """One expert's fp32 ``[N, K]`` weight matrix, N(0, std), keyed by (seed, tag, e)."""
    g = _rng(seed, _TAGS[tag], e)
    w = g.standard_normal((N, K), dtype=np.float32)
    w *= np.float32(std)
    return w


def activations_bf16(seed: int, T: int, K: int, tag: str = "x") -> np.ndarray:
    """``[T, K]`` activations N(0, 1), returned as bf16 bit patterns (uint16)."""
    g = _rng(seed, _TAGS[tag], T, K)
    return bf16_bits_from_f32(g.standard_normal((T, K), dtype=np.float32))


# --------------------------------------------------------------------------
# routing
# --------------------------------------------------------------------------
def route_softmax_topk(seed: int, T: int, E: int, k: int):
    """Top-k of softmax over N(0,1) logits. Ties go to the lower expert id.

    Returns (ids int32 [T, k], weights float32 [T, k]); the weights are the
    selected softmax probabilities, not renormalised.
    """
    g = _rng(seed, _TAGS["route"], T, E, k)
    logits = g.standard_normal((T, E))
    z = logits - logits.max(axis=1, keepdims=True)
    p = np.exp(z)
    p /= p.sum(axis=1, keepdims=True)
    order = np.argsort(-p, axis=1, kind="stable")[:, :k]
    w = np.take_along_axis(p, order, axis=1)
    return order.astype(np.int32), w.astype(np.float32)


def route_zipf_topk(seed: int, T: int, E: int, k: int, s: float = 1.2):
    """k distinct experts per token from a Zipf(s) popularity over a seeded
    permutation of expert ids (Gumbel top-k of log p).

    Returns (ids int32 [T, k], weights float32 [T, k]); a row's weight is its
    expert's Zipf probability.
    """
    g = _rng(seed, _TAGS["route"], T, E, k, int(round(s * 1000)))
    perm = g.permutation(E)
    ranks = np.arange(1, E + 1, dtype=np.float64)
    pr = ranks ** (-s)
    pr /= pr.sum()
    p = np.empty(E)
    p[perm] = pr
    gumbel = -np.log(-np.log(g.random((T, E))))
    score = np.log(p)[None, :] + gumbel
    order = np.argsort(-score, axis=1, kind="stable")[:, :k]
    return order.astype(np.int32), p[order].astype(np.float32)


def routing_metadata(ids: np.ndarray, weights: np.ndarray, E: int):
    """Sort the T*k routed rows by (expert, token, slot).

    Returns (expert_offsets int64 [E+1], row_token int32 [R],
    row_weight float32 [R], row_dest int32 [R]) where row_dest = t*k + slot.
    """
    T, k = ids.shape
    t = np.repeat(np.arange(T), k)
    slot = np.tile(np.arange(k), T)
    ex = ids.reshape(-1).astype(np.int64)
    order = np.lexsort((slot, t, ex))
    counts = np.bincount(ex, minlength=E)
    offsets = np.zeros(E + 1, dtype=np.int64)
    offsets[1:] = np.cumsum(counts)
    row_token = t[order].astype(np.int32)
    row_weight = weights.reshape(-1)[order].astype(np.float32)
    row_dest = (t * k + slot)[order].astype(np.int32)
    return offsets, row_token, row_weight, row_dest


@dataclass
class RoutedBatch:
    """One routed batch: tokens, their expert choices and the sorted rows."""
    T: int
    E: int
    k: int
    ids: np.ndarray          # int32 [T, k]
    weights: np.ndarray      # float32 [T, k]
    offsets: np.ndarray      # int64 [E+1]
    row_token: np.ndarray    # int32 [R]
    row_weight: np.ndarray   # float32 [R]
    row_dest: np.ndarray     # int32 [R]

    @property
    def R(self) -> int:
        return int(self.offsets[-1])

    def counts(self) -> np.ndarray:
        return np.diff(self.offsets)

    def active_experts(self) -> np.ndarray:
        return np.nonzero(self.counts() > 0)[0]


def make_routed_batch(seed: int, T: int, E: int, k: int, routing: str = "softmax",
                      zipf_s: float = 1.2) -> RoutedBatch:
    if routing == "softmax":
        ids, w = route_softmax_topk(seed, T, E, k)
    elif routing == "zipf":
        ids, w = route_zipf_topk(seed, T, E, k, zipf_s)
    else:
        raise ValueError(f"unknown routing {routing!r}")
    off, tok, rw, dst = routing_metadata(ids, w, E)
    return RoutedBatch(T, E, k, ids, w, off, tok, rw, dst)


def explicit_batch(counts, E: Optional[int] = None, seed: int = 0) -> RoutedBatch:
    """A batch with the given per-expert row counts (empty experts allowed):
    token t of expert e's rows is drawn uniformly, weights uniform in [0.5, 1.5)."""
    counts = np.asarray(counts, dtype=np.int64)
    E = len(counts) if E is None else E
    g = _rng(seed, _TAGS["misc"], len(counts), int(counts.sum()))
    R = int(counts.sum())
    offsets = np.zeros(E + 1, dtype=np.int64)
    offsets[1:len(counts) + 1] = np.cumsum(counts)
    offsets[len(counts) + 1:] = offsets[len(counts)]
    T = max(R, 1)
    row_token = g.integers(0, T, R).astype(np.int32)
    row_weight = (0.5 + g.random(R)).astype(np.float32)
    row_dest = g.permutation(R).astype(np.int32)
    ids = np.zeros((0, 1), np.int32)
    return RoutedBatch(T, E, 1, ids, np.zeros((0, 1), np.float32), offsets, row_token,
                       row_weight, row_dest)


def groups_to_routing(sizes, expert_ids, E: int):
    """Translate the pages' group description -- a_cat rows grouped in the order
    of ``expert_ids`` with ``sizes`` rows each -- into per-expert offsets over
    rows sorted by expert id, the a_cat row each sorted row reads, and the a_cat
    row it writes back to. Returns (offsets int64 [E+1], row_token int32,
    row_dest int32)."""
    sizes = [int(s) for s in sizes]
    expert_ids = [int(e) for e in expert_ids]
    starts = np.concatenate([[0], np.cumsum(sizes)[:-1]]).astype(np.int64)
    counts = np.zeros(E, dtype=np.int64)
    for s, e in zip(sizes, expert_ids):
        counts[e] += s
    offsets = np.zeros(E + 1, dtype=np.int64)
    offsets[1:] = np.cumsum(counts)
    src = []
    for e in range(E):
        for s0, s, ee in zip(starts, sizes, expert_ids):
            if ee == e:
                src.extend(range(s0, s0 + s))
    src = np.asarray(src, dtype=np.int32)
    return offsets, src, src.copy()
