"""Pins of the storage-variant oracle (bf16 absmax, fp16 activations) against what
the pages and the arithmetic fix: the lossless bf16 absmax of a bf16 source and the
refusal for an fp32 source, the printed 5.6 % byte saving, closed forms of the
binary16 rounding, and exact (rational) brute force on tiny products."""
import json
import os
from fractions import Fraction

import numpy as np
import pytest

from oracle import gnf4_oracle as O
from oracle import storage as S

GOLDEN = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "pages_printed_values.json")))


def _bf16_weights(seed, rows, K):
    """fp32 weights that are bf16 values (a bf16 checkpoint widened to fp32)."""
    w = np.random.default_rng(seed).normal(0, 0.02, (rows, K)).astype(np.float32)
    return (w.view(np.uint32) & np.uint32(0xFFFF0000)).view(np.float32)


def test_bf16_absmax_is_lossless_for_a_bf16_source():
    g = GOLDEN["nf4_bf16_absmax"]
    assert g["bitwise_identical_for_bf16_source"]
    w = _bf16_weights(1, 64, 512)
    p, a = O.quantize_nf4(w)
    bits = S.absmax_to_bf16(a)                       # must not raise
    assert np.array_equal(S.dequant_nf4_bf16(p, bits, 512), O.dequant_nf4(p, a, 512))
    # each absmax is one of its block's magnitudes
    blk = np.abs(w).reshape(64, 8, 64)
    assert np.array_equal(blk.max(axis=2), a)


def test_bf16_absmax_refuses_an_fp32_source():
    assert GOLDEN["nf4_bf16_absmax"]["fp32_source_refused"]
    w = np.random.default_rng(2).normal(0, 0.02, (16, 256)).astype(np.float32)
    _, a = O.quantize_nf4(w)
    with pytest.raises(ValueError):
        S.absmax_to_bf16(a)
    # a single non-bf16 value is enough to refuse
    ok = np.ones((2, 4), np.float32)
    S.absmax_to_bf16(ok)
    ok[1, 2] = np.float32(1.0 + 2.0 ** -20)
    with pytest.raises(ValueError):
        S.absmax_to_bf16(ok)


def test_bf16_absmax_bit_patterns():
    vals = np.array([0.0, 1.0, 0.5, 2.0 ** -120, 3.0, 0.0234375], np.float32)
    bits = S.absmax_to_bf16(vals)
    assert list(bits) == [0x0000, 0x3F80, 0x3F00, 0x0380, 0x4040, 0x3CC0]


def test_bf16_absmax_byte_saving_matches_the_printed_figure():
    g = GOLDEN["nf4_bf16_absmax"]
    share = GOLDEN["nf4_absmax_share_qwen3_expert"]
    f32 = sum(O.packed_bytes("nf4", N, K)["nibbles"] + O.packed_bytes("nf4", N, K)["scales"]
              for N, K in share["projections_NK"])
    b16 = sum(S.packed_bytes_bf16(N, K)["nibbles"] + S.packed_bytes_bf16(N, K)["scales"]
              for N, K in share["projections_NK"])
    assert f32 == share["row_bytes"]
    saving = 100.0 * (f32 - b16) / f32
    assert saving == pytest.approx(100.0 * share["absmax_bytes"] / 2 / share["row_bytes"])
    assert abs(saving - g["saving_percent_printed"]) < 0.05


@pytest.mark.parametrize("v,want", [
    (1.0 + 2.0 ** -11, 1.0),                        # halfway, even neighbour below
    (1.0 + 3 * 2.0 ** -11, 1.0 + 2.0 ** -9),        # halfway, even neighbour above
    (1.0 + 2.0 ** -11 + 2.0 ** -30, 1.0 + 2.0 ** -10),
    (65504.0, 65504.0),                             # largest finite
    (65519.99, 65504.0),
    (65520.0, np.inf),                              # halfway to 2^16: rounds to even, overflows
    (2.0 ** -24, 2.0 ** -24),                       # smallest subnormal
    (2.0 ** -25, 0.0),                              # halfway between 0 and 2^-24: even is 0
    (3 * 2.0 ** -26, 2.0 ** -24),
    (2.0 ** -14 - 2.0 ** -25, 2.0 ** -14),          # largest subnormal rounds up to min normal
    (-1.5, -1.5),
    (0.1, 0.0999755859375),
])
def test_round_to_f16_closed_forms(v, want):
    assert S.round_to_f16(np.array([v]))[0] == want


def test_f16_bits_round_trip_and_sign():
    v = np.array([1.0, -2.0, 0.5, -0.0, 65504.0, 2.0 ** -24], np.float64)
    bits = S.f16_bits(v)
    assert list(bits) == [0x3C00, 0xC000, 0x3800, 0x8000, 0x7BFF, 0x0001]
    assert np.array_equal(S.f16_to_f64(bits), v)


def test_grouped_product_fp16_activations_brute_force():
    """Exact rational arithmetic over every term on a tiny call (two experts, one empty
    group, a routing weight), NF4 with bf16 absmax and fp16 activations."""
    rng = np.random.default_rng(5)
    E, N, K = 3, 8, 128
    Wb = np.zeros((E, N, K // 2), np.uint8)
    Ab = np.zeros((E, N, K // 64), np.uint16)
    for e in range(E):
        p, a = O.quantize_nf4(_bf16_weights(10 + e, N, K))
        Wb[e], Ab[e] = p, S.absmax_to_bf16(a)
    T = 5
    xh = S.f16_bits(rng.normal(0, 1, (T, K)))
    x = S.f16_to_f64(xh)
    offsets = np.array([0, 2, 2, 5])
    tok = np.array([4, 0, 1, 3, 2])
    wt = np.array([0.5, 1.0, 0.25, 2.0, 1.0], np.float32)
    got = S.grouped_rows_f64_x("nf4", x, Wb, Ab, offsets, tok, wt, K, np.arange(5))
    codes = [O.nf4_codes(Wb[e], K) for e in range(E)]
    absv = O.bf16_to_f64(Ab)
    for r in range(5):
        e = 0 if r < 2 else 2
        for n in range(N):
            acc = Fraction(0)
            for k in range(K):
                c = Fraction(float(O.NF4_CODEBOOK[codes[e][n, k]]))
                am = Fraction(float(absv[e, n, k // 64]))
                acc += Fraction(float(x[tok[r], k])) * c * am
            acc *= Fraction(float(wt[r]))
            assert abs(float(acc) - got[r, n]) <= 1e-12 * max(1.0, abs(float(acc)))


def test_one_hot_fp16_row_reads_the_decoded_weight_column():
    E, N, K = 1, 16, 64
    p, a = O.quantize_nf4(_bf16_weights(3, N, K))
    Wb, Ab = p[None], S.absmax_to_bf16(a)[None]
    x = np.zeros((K, K))
    x[np.arange(K), np.arange(K)] = 1.0
    got = S.grouped_rows_f64_x("nf4", x, Wb, Ab, [0, K], None, None, K, np.arange(K))
    assert np.array_equal(got, S.dequant_nf4_bf16(p, Ab[0], K).T)


def test_fp16_and_bf16_activations_agree_on_common_values():
    """Values exact in both 16-bit types give the same fp64 product."""
    rng = np.random.default_rng(7)
    N, K = 16, 128
    p, a = O.quantize_nf4(rng.normal(0, 0.02, (N, K)).astype(np.float32))
    xv = rng.integers(-64, 64, (4, K)) / 32.0                 # exact in bf16 and fp16
    xb = O.bf16_bits(xv)
    xf = S.f16_bits(xv)
    rb = O.grouped_rows_f64("nf4", xb, p[None], a[None], [0, 4], None, None, K, np.arange(4))
    rf = S.grouped_rows_f64_x("nf4", S.f16_to_f64(xf), p[None], a[None], [0, 4], None, None, K, np.arange(4))
    assert np.array_equal(rb, rf)
