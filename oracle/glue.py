"""Plain CPU oracle for the two steps either side of the grouped GEMM in a routed
MoE layer: the SwiGLU between gate_up and down, and the top-k combine of the
down outputs back into one row per token.

TEST INFRASTRUCTURE ONLY, like ``gnf4_oracle``: only the tests,
``__graft_entry__.smoke()`` and the bench's CPU baseline leg use it, and it
shares no code with the CUDA path.

Passages:

* The status page "MoE Software Status & Known Limits", section
  "grouped-nf4-gemm", "Correctness contracts": the decode glue is a SwiGLU over
  rows (``swiglu_rows``), a top-k combine (``combine_rows``) and a partial
  reduction (``reduce_partials``); the combine carries an accuracy contract,
  the partial reduction is bitwise the slot-order sum, and a token's combined
  row has the same bits whether it is combined alone or inside a larger call
  (row-count invariance). The consumer compatibility record of the same
  project names the three as the decode glue the MoE layer integrates.
* The experts4bit-qlora 0.6.5 README, "Scope" (and the lead paragraph above
  "Which door?"): the MoE architectures served are fused SwiGLU ones; gpt-oss
  adds per-expert biases and a clamped-GLU epilogue, whose formula the pages
  do not print (not built here).

Readings (the pages name these steps but print no formula for them):

17. SwiGLU: the gate_up output row is ``[gate | up]`` (the first I columns are
    the gate projection, the next I the up projection, the fused layout of the
    SwiGLU MoE checkpoints), and ``act = silu(gate) * up`` with
    ``silu(g) = g / (1 + exp(-g))``. Exact arithmetic (fp64 here), one rounding
    to bf16 at the end.
18. Combine: ``out[t] = sum over slots s = 0..k-1 of w[t, s] * y[src(t, s)]``
    with ``src(t, s) = row_of_slot[t*k + s]`` (or ``t*k + s`` when no index is
    given: the down GEMM already scattered slot s of token t to that row) and
    ``w`` the routing weight (1 when none is given: the down GEMM's epilogue
    already applied it). "Bitwise the slot-order sum" is read as: an fp32
    accumulator that starts at +0 and, for s = 0, 1, ..., k-1 in that order,
    adds the fp32-rounded product ``w * y`` (one rounding for the product, one
    for each addition, no fused multiply-add), then one rounding to bf16.
    A source index outside ``[0, R)`` contributes nothing (a dropped slot).
"""
from __future__ import annotations

import numpy as np

from .gnf4_oracle import bf16_bits, bf16_to_f64


# --------------------------------------------------------------------------
# SwiGLU (reading 17)
# --------------------------------------------------------------------------
def silu_f64(g: np.ndarray) -> np.ndarray:
    """``g * sigmoid(g)`` in fp64, written as ``g / (1 + exp(-g))``.

    For g below about -709 ``exp(-g)`` overflows to inf and the quotient is -0,
    the limit of the function."""
    g = np.asarray(g, dtype=np.float64)
    with np.errstate(over="ignore"):
        return g / (1.0 + np.exp(-g))


def swiglu_rows_f64(h_bits: np.ndarray) -> np.ndarray:
    """Unrounded SwiGLU of gate_up rows: bf16 bits ``[R, 2I]`` -> fp64 ``[R, I]``."""
    h = bf16_to_f64(h_bits)
    if h.ndim != 2 or h.shape[1] % 2:
        raise ValueError("gate_up rows must be [R, 2I]")
    I = h.shape[1] // 2
    gate, up = h[:, :I], h[:, I:]
    with np.errstate(over="ignore", invalid="ignore"):
        return silu_f64(gate) * up


def swiglu_rows(h_bits: np.ndarray) -> np.ndarray:
    """SwiGLU of gate_up rows, rounded once to bf16: bits ``[R, 2I]`` -> bits ``[R, I]``."""
    return bf16_bits(swiglu_rows_f64(h_bits))


# --------------------------------------------------------------------------
# top-k combine (reading 18)
# --------------------------------------------------------------------------
def _sources(T: int, k: int, R: int, row_of_slot):
    if row_of_slot is None:
        src = np.arange(T * k, dtype=np.int64).reshape(T, k)
    else:
        src = np.asarray(row_of_slot, dtype=np.int64).reshape(T, k)
    valid = (src >= 0) & (src < R)
    return np.where(valid, src, 0), valid


def combine_topk(y_bits: np.ndarray, T: int, k: int, row_of_slot=None, slot_weight=None) -> np.ndarray:
    """Top-k combine as the fp32 slot-order sum: bf16 bits ``[R, N]`` -> bits ``[T, N]``.

    The loop over slots is the definition itself: one fp32 product and one fp32
    addition per slot, in slot order, starting from +0."""
    y = np.ascontiguousarray(y_bits, dtype=np.uint16)
    R, N = y.shape
    if R == 0:
        return np.zeros((T, N), dtype=np.uint16)
    src, valid = _sources(T, k, R, row_of_slot)
    w = (np.ones((T, k), dtype=np.float32) if slot_weight is None
         else np.asarray(slot_weight, dtype=np.float32).reshape(T, k))
    yf = bf16_to_f64(y).astype(np.float32)            # exact: bf16 values are fp32 values
    acc = np.zeros((T, N), dtype=np.float32)
    for s in range(k):
        term = w[:, s:s + 1] * yf[src[:, s]]          # fp32 product, rounded once
        acc = np.where(valid[:, s:s + 1], acc + term, acc)   # fp32 sum, rounded once
    return bf16_bits(acc.astype(np.float64))


def combine_topk_f64(y_bits: np.ndarray, T: int, k: int, row_of_slot=None, slot_weight=None) -> np.ndarray:
    """The same combine in exact arithmetic (fp64), unrounded: the accuracy reference."""
    y = bf16_to_f64(y_bits)
    R, N = y.shape
    if R == 0:
        return np.zeros((T, N))
    src, valid = _sources(T, k, R, row_of_slot)
    w = (np.ones((T, k)) if slot_weight is None
         else np.asarray(slot_weight, dtype=np.float32).astype(np.float64).reshape(T, k))
    out = np.zeros((T, N))
    for s in range(k):
        out += np.where(valid[:, s:s + 1], w[:, s:s + 1] * y[src[:, s]], 0.0)
    return out
