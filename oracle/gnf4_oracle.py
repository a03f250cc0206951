"""Plain CPU oracle for the grouped 4-bit MoE GEMM (NF4 and MXFP4).

TEST INFRASTRUCTURE ONLY. Nothing in the product path imports, calls or links
this module: only the tests, ``__graft_entry__.smoke()`` and the bench's CPU
baseline leg use it. It shares no code with the CUDA path; the only thing
both sides consume is the seeded input generators in ``synth``.

What it computes, and from which passage:

* NF4 packing, ``quantize_nf4`` / ``dequant_nf4`` -- the grouped-nf4-gemm
  README (0.11.0 PKG-INFO), "Try it on CPU right now", block 1 (NF4
  round-trip: ``[N, K]`` fp32 -> ``[N, K//2]`` uint8 + ``[N, K//64]`` fp32,
  re-pack idempotent), and the solution page "How do I run a grouped GEMM
  directly on NF4 packed MoE expert weights, without dequantizing to bf16
  first?", "Supported scope" (bitsandbytes ``gemm_4bit`` layout, blocksize 64,
  ``K % 64 == 0``).
* MXFP4 packing, ``quantize_mxfp4`` / ``dequant_mxfp4`` -- the same README,
  block 2 (MXFP4 round-trip, K a multiple of 32, e8m0 per-32 scales) and "The
  NVMe tier" (kernel view ``[E, N, K//2]`` blocks + ``[E, N, K//32]`` scales).
* The grouped product, ``grouped_gemm`` -- the solution page, "Smallest
  correct example" (per group ``a.double() @ dequant_ref(B[e]).double().T``)
  and "Expected result" (the per-element decode is the kernel's; only the
  fp32 reduction order differs). The routing weight and the row scatter are
  the epilogue options of the op this library exports.

Arithmetic: products and sums are fp64 (exact decode, fp64 accumulation), the
result is rounded once to bf16 (round to nearest even). The two quantizers
work in fp32 on purpose: their bytes are compared bit for bit, so every
rounding step is fixed here (fp32 IEEE division for NF4 normalisation; exact
power-of-two scaling for MXFP4).

Readings taken where the pages are silent (each one is listed with its
reason in the design notes of the repository):

1. NF4 codebook: the 16 NF4 values of the QLoRA paper (Dettmers et al. 2023,
   appendix E), i.e. bitsandbytes' NF4 type, held as fp32.
2. NF4 nibble order: element 2j in the HIGH nibble of byte j, 2j+1 in the low.
3. NF4 normalisation: x = fl32(w / absmax); code = number of fp32 midpoints
   (c_i + c_{i+1})/2 strictly below x (nearest value, ties to the lower code).
   A block whose absmax is 0 gets code 7 (0.0) everywhere.
4. e2m1 and e8m0 decode: the OCP Microscaling v1.0 definitions; e8m0 255 is NaN.
5. MXFP4 quantizer: E = floor(log2 amax) - 2 from the fp32 exponent field,
   clamped to [-127, 127]; x = w * 2^-E (exact); x rounded to the e2m1 grid,
   ties to the even code, |x| > 6 saturates to 6; the sign nibble bit is set
   for w < 0. An all-zero block gets scale 127 and codes 0.
6. MXFP4 nibble order: element 2j in the LOW nibble, 2j+1 in the high.
"""
from __future__ import annotations

import numpy as np

# --------------------------------------------------------------------------
# NF4 codebook (reading 1) -- fp32 values, ascending
# --------------------------------------------------------------------------
NF4_CODEBOOK = np.array([
    -1.0, -0.6961928009986877, -0.5250730514526367, -0.39491748809814453,
    -0.28444138169288635, -0.18477343022823334, -0.09105003625154495, 0.0,
    0.07958029955625534, 0.16093020141124725, 0.24611230194568634,
    0.33791524171829224, 0.44070982933044434, 0.5626170039176941,
    0.7229568362236023, 1.0], dtype=np.float32)

NF4_BLOCK = 64
MXFP4_BLOCK = 32


def nf4_thresholds() -> np.ndarray:
    """fp32 midpoints between neighbouring NF4 values (15 of them)."""
    c = NF4_CODEBOOK
    return ((c[:-1] + c[1:]) / np.float32(2)).astype(np.float32)


def quantize_nf4(w: np.ndarray):
    """fp32 ``[rows, K]`` -> (packed uint8 ``[rows, K//2]``, absmax fp32 ``[rows, K//64]``)."""
    w = np.ascontiguousarray(w, dtype=np.float32)
    rows, K = w.shape
    if K % NF4_BLOCK:
        raise ValueError("K must be a multiple of 64")
    blk = w.reshape(rows, K // NF4_BLOCK, NF4_BLOCK)
    absmax = np.abs(blk).max(axis=2)
    with np.errstate(divide="ignore", invalid="ignore"):
        x = (blk / absmax[:, :, None]).astype(np.float32)
    x[absmax == 0] = np.float32(0.0)
    codes = np.searchsorted(nf4_thresholds(), x.reshape(-1), side="left")
    codes = codes.reshape(rows, K).astype(np.uint8)
    packed = (codes[:, 0::2] << 4) | codes[:, 1::2]
    return packed.astype(np.uint8), absmax.astype(np.float32)


def nf4_codes(packed: np.ndarray, K: int) -> np.ndarray:
    """uint8 ``[rows, K//2]`` -> codes ``[rows, K]`` (element 2j from the high nibble)."""
    packed = np.asarray(packed, dtype=np.uint8)
    rows = packed.shape[0]
    codes = np.empty((rows, K), dtype=np.uint8)
    codes[:, 0::2] = packed >> 4
    codes[:, 1::2] = packed & 0x0F
    return codes


def dequant_nf4(packed: np.ndarray, absmax: np.ndarray, K: int) -> np.ndarray:
    """Exact decode to fp64 ``[rows, K]``: codebook value times its block's absmax."""
    codes = nf4_codes(packed, K)
    vals = NF4_CODEBOOK.astype(np.float64)[codes]
    scale = np.repeat(np.asarray(absmax, dtype=np.float64), NF4_BLOCK, axis=1)
    return vals * scale


# --------------------------------------------------------------------------
# MXFP4 (readings 4-6)
# --------------------------------------------------------------------------
def e2m1_value(code: int) -> float:
    """OCP e2m1: 1 sign bit, 2 exponent bits (bias 1), 1 mantissa bit."""
    s = (code >> 3) & 1
    e = (code >> 1) & 3
    m = code & 1
    mag = (m * 0.5) if e == 0 else (2.0 ** (e - 1)) * (1.0 + m * 0.5)
    return -mag if s else mag


E2M1_TABLE = np.array([e2m1_value(c) for c in range(16)], dtype=np.float64)


def e8m0_value(s: int) -> float:
    """OCP e8m0 scale: 2^(s - 127); the pattern 255 is NaN."""
    return float("nan") if s == 255 else float(np.ldexp(1.0, int(s) - 127))


E8M0_TABLE = np.array([e8m0_value(s) for s in range(256)], dtype=np.float64)

# magnitudes of e2m1 codes 0..7 and the midpoints between neighbours
_E2M1_MAG = E2M1_TABLE[:8]
_E2M1_MID = (_E2M1_MAG[:-1] + _E2M1_MAG[1:]) / 2.0


def _e2m1_round(a: np.ndarray) -> np.ndarray:
    """Magnitudes (fp64, >= 0) -> nearest e2m1 magnitude code, ties to even code,
    saturating above 6."""
    code = np.zeros(a.shape, dtype=np.uint8)
    for i, m in enumerate(_E2M1_MID):          # m lies between codes i and i+1
        up = (a > m) | ((a == m) & (i % 2 == 1))
        code += up.astype(np.uint8)
    return code


def mxfp4_scale_exponent(amax: np.ndarray) -> np.ndarray:
    """Shared exponent E per block from the fp32 exponent field of amax (reading 5)."""
    amax = np.ascontiguousarray(amax, dtype=np.float32)
    ef = ((amax.view(np.uint32) >> 23) & 0xFF).astype(np.int64)
    E = np.where(ef > 0, ef - 127 - 2, -127)
    E = np.clip(E, -127, 127)
    return np.where(amax == 0, 0, E)


def quantize_mxfp4(w: np.ndarray):
    """fp32 ``[rows, K]`` -> (blocks uint8 ``[rows, K//2]``, scales uint8 ``[rows, K//32]``)."""
    w = np.ascontiguousarray(w, dtype=np.float32)
    rows, K = w.shape
    if K % MXFP4_BLOCK:
        raise ValueError("K must be a multiple of 32")
    blk = w.reshape(rows, K // MXFP4_BLOCK, MXFP4_BLOCK)
    amax = np.abs(blk).max(axis=2)
    E = mxfp4_scale_exponent(amax)
    xs = blk.astype(np.float64) * np.ldexp(1.0, -E)[:, :, None]   # exact
    code = _e2m1_round(np.abs(xs)) | (np.where(xs < 0, 8, 0).astype(np.uint8))
    code = code.reshape(rows, K)
    blocks = code[:, 0::2] | (code[:, 1::2] << 4)
    return blocks.astype(np.uint8), (E + 127).astype(np.uint8)


def mxfp4_codes(blocks: np.ndarray, K: int) -> np.ndarray:
    """uint8 ``[rows, K//2]`` -> codes ``[rows, K]`` (element 2j from the low nibble)."""
    blocks = np.asarray(blocks, dtype=np.uint8).reshape(-1, K // 2)
    codes = np.empty((blocks.shape[0], K), dtype=np.uint8)
    codes[:, 0::2] = blocks & 0x0F
    codes[:, 1::2] = blocks >> 4
    return codes


def dequant_mxfp4(blocks: np.ndarray, scales: np.ndarray, K: int) -> np.ndarray:
    """Exact decode to fp64 ``[rows, K]``: e2m1 value times 2^(s-127)."""
    codes = mxfp4_codes(blocks, K)
    sc = E8M0_TABLE[np.asarray(scales, dtype=np.uint8).reshape(codes.shape[0], -1)]
    return E2M1_TABLE[codes] * np.repeat(sc, MXFP4_BLOCK, axis=1)


# --------------------------------------------------------------------------
# bf16 rounding (fp64 -> bf16, round to nearest even, one rounding)
# --------------------------------------------------------------------------
def round_to_bf16(v: np.ndarray) -> np.ndarray:
    """Round fp64 values to the nearest bf16 value (ties to even), returned as fp64.

    bf16 keeps 8 significant bits; below 2^-126 the spacing stays 2^-133
    (subnormals); magnitudes that round past the largest finite value give inf.
    """
    v = np.asarray(v, dtype=np.float64)
    out = np.array(v, copy=True)
    fin = np.isfinite(v) & (v != 0)
    _, e = np.frexp(v[fin])                       # |v| = m * 2^e, m in [0.5, 1)
    q = np.maximum(e - 8, -133)                   # exponent of one unit in the last place
    r = np.ldexp(np.round(np.ldexp(v[fin], -q)), q)
    r[np.abs(r) >= 2.0 ** 128] = np.inf * np.sign(r[np.abs(r) >= 2.0 ** 128])
    out[fin] = r
    return out


def bf16_bits(v: np.ndarray) -> np.ndarray:
    """fp64 -> bf16 bit patterns (uint16), one round-to-nearest-even step."""
    r = round_to_bf16(v).astype(np.float32)       # exact: r is on the bf16 grid
    return (r.view(np.uint32) >> 16).astype(np.uint16)


def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    bits = np.ascontiguousarray(bits, dtype=np.uint16)
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


# --------------------------------------------------------------------------
# the grouped product
# --------------------------------------------------------------------------
def decode_expert(fmt: str, W: np.ndarray, S: np.ndarray, e: int, K: int) -> np.ndarray:
    """Expert e of a packed stack (``W [E, N, K//2]``, scales ``S [E, N, K//b]``) in fp64."""
    if fmt == "nf4":
        return dequant_nf4(W[e], S[e], K)
    if fmt == "mxfp4":
        return dequant_mxfp4(W[e], S[e], K)
    raise ValueError(f"unknown format {fmt!r}")


def grouped_rows_f64(fmt, x_bits, W, S, offsets, row_token, row_weight, K, rows):
    """Unrounded fp64 results ``w(r) * sum_k x[tok(r), k] * What[e(r), :, k]`` for the
    routed rows listed in ``rows`` (any order). Returns fp64 ``[len(rows), N]``."""
    rows = np.asarray(rows, dtype=np.int64)
    offsets = np.asarray(offsets, dtype=np.int64)
    x = bf16_to_f64(x_bits)
    N = W.shape[1]
    out = np.empty((len(rows), N), dtype=np.float64)
    experts = np.searchsorted(offsets, rows, side="right") - 1
    for e in np.unique(experts):
        sel = np.nonzero(experts == e)[0]
        r = rows[sel]
        tok = r if row_token is None else np.asarray(row_token, dtype=np.int64)[r]
        acc = x[tok] @ decode_expert(fmt, W, S, int(e), K).T
        if row_weight is not None:
            acc = acc * np.asarray(row_weight, dtype=np.float64)[r][:, None]
        out[sel] = acc
    return out


def grouped_gemm(fmt, x_bits, W, S, offsets, row_token=None, row_weight=None,
                 row_dest=None, T_out=None, out_init=None):
    """The whole grouped product, bf16 bit patterns ``[T_out, N]``.

    ``out[dest(r), n] = bf16(w(r) * sum_k x[tok(r), k] * What[e(r), n, k])`` for
    every routed row r; e(r) is the expert whose offset range holds r; empty
    experts contribute nothing; rows of ``out`` that no routed row names keep
    ``out_init`` (zeros if not given).
    """
    offsets = np.asarray(offsets, dtype=np.int64)
    E = len(offsets) - 1
    N = W.shape[1]
    K = W.shape[2] * 2
    R = int(offsets[-1])
    if T_out is None:
        T_out = R
    out = (np.zeros((T_out, N), dtype=np.uint16) if out_init is None
           else np.array(out_init, dtype=np.uint16, copy=True))
    x = bf16_to_f64(x_bits)
    for e in range(E):
        r0, r1 = int(offsets[e]), int(offsets[e + 1])
        if r1 <= r0:
            continue
        r = np.arange(r0, r1)
        tok = r if row_token is None else np.asarray(row_token, dtype=np.int64)[r]
        acc = x[tok] @ decode_expert(fmt, W, S, e, K).T
        if row_weight is not None:
            acc = acc * np.asarray(row_weight, dtype=np.float64)[r][:, None]
        dest = r if row_dest is None else np.asarray(row_dest, dtype=np.int64)[r]
        out[dest] = bf16_bits(acc)
    return out


# --------------------------------------------------------------------------
# byte accounting (algorithmic bytes of a packed expert)
# --------------------------------------------------------------------------
def packed_bytes(fmt: str, N: int, K: int) -> dict:
    """Nibble and scale bytes of one ``[N, K]`` expert matrix."""
    if fmt == "nf4":
        return {"nibbles": N * K // 2, "scales": N * (K // NF4_BLOCK) * 4}
    if fmt == "mxfp4":
        return {"nibbles": N * K // 2, "scales": N * (K // MXFP4_BLOCK)}
    raise ValueError(fmt)
