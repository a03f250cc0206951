"""Storage variants of the grouped 4-bit product: bf16 absmax and fp16 activations.

TEST INFRASTRUCTURE ONLY. Like the rest of ``oracle``, nothing in the product
path imports, calls or links this module; only the tests, ``smoke()`` and the
bench's CPU legs use it, and it shares no code with the CUDA path.

What it computes, and from which passage:

* ``absmax_to_bf16`` -- the grouped-nf4-gemm README (0.11.0 PKG-INFO), "Which
  entry point? Pick by where the weights live", the ``--absmax-dtype bf16``
  paragraph: the NF4 absmax may be stored as bf16, which is lossless when the
  source weights are bf16 (a block's absmax is one of its magnitudes, and the
  largest of a set of bf16 values is a bf16 value); the cast refuses instead of
  rounding when a value is not exactly representable. Plain definition used
  here: an fp32 value is a bf16 value exactly when its low 16 bits are zero,
  and then its bf16 pattern is its high 16 bits.
* ``dequant_nf4_bf16`` -- the NF4 decode with the stored bf16 absmax widened
  back to fp32 (exact): codebook value times absmax, in fp64.
* ``packed_bytes_bf16`` -- byte accounting of an NF4 matrix whose absmax is
  stored as bf16 (2 bytes a block instead of 4).
* ``round_to_f16`` / ``f16_bits`` -- fp64 to IEEE binary16, one rounding to
  nearest even (11 significant bits, subnormal spacing 2^-24, overflow to inf
  from 65520 up), for the fp16-activation variant of the solution page "How do I
  run a grouped GEMM directly on NF4 packed MoE expert weights, without
  dequantizing to bf16 first?", "Supported scope" (``a_cat [T, K]`` bf16/fp16).
* ``grouped_rows_f64_x`` -- the grouped product of the solution page's "Smallest
  correct example" with the activations given as fp64 values (decoded by the
  caller from bf16 or fp16 bits) and the NF4 absmax in either storage type.

Reading taken where the pages are silent: the output of an fp16-activation call
is fp16 (the op's result type follows its activations, as for the bf16 example
the pages print); the fp32 accumulation and the single final rounding are the
same as for bf16.
"""
from __future__ import annotations

import numpy as np

from .gnf4_oracle import (MXFP4_BLOCK, NF4_BLOCK, NF4_CODEBOOK, bf16_to_f64, dequant_mxfp4,
                          nf4_codes)


# --------------------------------------------------------------------------
# bf16 absmax
# --------------------------------------------------------------------------
def absmax_to_bf16(absmax: np.ndarray) -> np.ndarray:
    """fp32 absmax -> bf16 bit patterns (uint16); ValueError if any value is not
    exactly a bf16 value (the cast never rounds)."""
    a = np.ascontiguousarray(absmax, dtype=np.float32)
    u = a.view(np.uint32)
    if np.any(u & np.uint32(0xFFFF)):
        bad = int(np.count_nonzero(u & np.uint32(0xFFFF)))
        raise ValueError(f"{bad} absmax values are not exactly representable in bf16")
    return (u >> np.uint32(16)).astype(np.uint16)


def dequant_nf4_bf16(packed: np.ndarray, absmax_bits: np.ndarray, K: int) -> np.ndarray:
    """Exact decode to fp64 ``[rows, K]`` with the absmax stored as bf16 bits."""
    codes = nf4_codes(packed, K)
    vals = NF4_CODEBOOK.astype(np.float64)[codes]
    scale = np.repeat(bf16_to_f64(absmax_bits), NF4_BLOCK, axis=1)
    return vals * scale


def packed_bytes_bf16(N: int, K: int) -> dict:
    """Nibble and scale bytes of one ``[N, K]`` NF4 matrix with bf16 absmax."""
    return {"nibbles": N * K // 2, "scales": N * (K // NF4_BLOCK) * 2}


# --------------------------------------------------------------------------
# fp16 (IEEE binary16)
# --------------------------------------------------------------------------
def round_to_f16(v: np.ndarray) -> np.ndarray:
    """Round fp64 values to the nearest binary16 value (ties to even), as fp64.

    11 significant bits; below 2^-14 the spacing stays 2^-24 (subnormals); a
    magnitude that rounds to 2^16 or beyond is inf (the largest finite value is
    65504, and 65520, halfway to 65536, rounds to the even neighbour 65536)."""
    v = np.asarray(v, dtype=np.float64)
    out = np.array(v, copy=True)
    fin = np.isfinite(v) & (v != 0)
    _, e = np.frexp(v[fin])                       # |v| = m * 2^e, m in [0.5, 1)
    q = np.maximum(e - 11, -24)                   # exponent of one unit in the last place
    r = np.ldexp(np.round(np.ldexp(v[fin], -q)), q)
    big = np.abs(r) >= 2.0 ** 16
    r[big] = np.inf * np.sign(r[big])
    out[fin] = r
    return out


def f16_bits(v: np.ndarray) -> np.ndarray:
    """fp64 -> binary16 bit patterns (uint16), one round-to-nearest-even step."""
    r = round_to_f16(v)
    return r.astype(np.float16).view(np.uint16)   # exact: r is on the binary16 grid


def f16_to_f64(bits: np.ndarray) -> np.ndarray:
    return np.ascontiguousarray(bits, dtype=np.uint16).view(np.float16).astype(np.float64)


# --------------------------------------------------------------------------
# the grouped product with either activation type and either absmax type
# --------------------------------------------------------------------------
def decode_expert_x(fmt: str, W: np.ndarray, S: np.ndarray, e: int, K: int) -> np.ndarray:
    """Expert e in fp64. NF4 scales may be fp32 (float32 array) or bf16 (uint16 bits)."""
    if fmt == "nf4":
        if S.dtype == np.uint16:
            return dequant_nf4_bf16(W[e], S[e], K)
        codes = nf4_codes(W[e], K)
        return NF4_CODEBOOK.astype(np.float64)[codes] * np.repeat(
            np.asarray(S[e], dtype=np.float64), NF4_BLOCK, axis=1)
    if fmt == "mxfp4":
        return dequant_mxfp4(W[e], S[e], K)
    raise ValueError(f"unknown format {fmt!r}")


def grouped_rows_f64_x(fmt, x_f64, W, S, offsets, row_token, row_weight, K, rows):
    """Unrounded fp64 results ``w(r) * sum_k x[tok(r), k] * What[e(r), :, k]`` for
    the routed rows in ``rows``; ``x_f64`` holds the activations' exact values."""
    rows = np.asarray(rows, dtype=np.int64)
    offsets = np.asarray(offsets, dtype=np.int64)
    x = np.asarray(x_f64, dtype=np.float64)
    N = W.shape[1]
    out = np.empty((len(rows), N), dtype=np.float64)
    experts = np.searchsorted(offsets, rows, side="right") - 1
    for e in np.unique(experts):
        sel = np.nonzero(experts == e)[0]
        r = rows[sel]
        tok = r if row_token is None else np.asarray(row_token, dtype=np.int64)[r]
        acc = x[tok] @ decode_expert_x(fmt, W, S, int(e), K).T
        if row_weight is not None:
            acc = acc * np.asarray(row_weight, dtype=np.float64)[r][:, None]
        out[sel] = acc
    return out


__all__ = ["absmax_to_bf16", "dequant_nf4_bf16", "packed_bytes_bf16", "round_to_f16", "f16_bits",
           "f16_to_f64", "decode_expert_x", "grouped_rows_f64_x", "MXFP4_BLOCK"]
