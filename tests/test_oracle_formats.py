"""Pins for the oracle's packing and decoding (CPU only).

Each check ties the oracle to something other than itself: values the
grouped-nf4-gemm pages print (tests/golden/pages_printed_values.json), the
closed-form construction of the NF4 codebook, the OCP e2m1/e8m0 definitions,
hand-worked bytes, and torch's own fp32->bf16 conversion.
"""
import json
import os

import numpy as np
import pytest
import torch

from oracle import gnf4_oracle as O

GOLDEN = json.load(open(os.path.join(os.path.dirname(__file__), "golden",
                                     "pages_printed_values.json")))


# --------------------------------------------------------------------------
# codebooks
# --------------------------------------------------------------------------
def test_nf4_codebook_matches_quantile_construction():
    """NF4 = normalised N(0,1) quantiles: 8 positive levels on an evenly spaced
    probability grid from 1-delta down to 1/2, 7 negative levels likewise, and 0,
    with 1-delta = (1 - 1/30)/2 + (1 - 1/32)/2 (QLoRA, appendix E)."""
    from scipy.stats import norm
    hi = 0.5 * (1 - 1 / 30) + 0.5 * (1 - 1 / 32)
    pos = norm.ppf(np.linspace(hi, 0.5, 9)[:-1])
    neg = -norm.ppf(np.linspace(hi, 0.5, 8)[:-1])
    v = np.sort(np.concatenate([pos, [0.0], neg]))
    v = v / v.max()
    np.testing.assert_allclose(O.NF4_CODEBOOK.astype(np.float64), v, atol=1e-6, rtol=0)


def test_nf4_codebook_invariants():
    c = O.NF4_CODEBOOK
    assert c.dtype == np.float32 and c.shape == (16,)
    assert np.all(np.diff(c) > 0)
    assert c[0] == -1.0 and c[7] == 0.0 and c[15] == 1.0
    assert (c < 0).sum() == 7 and (c > 0).sum() == 8


def test_e2m1_table_is_ocp_e2m1():
    # OCP MX v1.0: FP4 E2M1 magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6; bit 3 is the sign.
    mags = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    for code in range(8):
        assert O.E2M1_TABLE[code] == mags[code]
        assert O.E2M1_TABLE[code + 8] == -mags[code]
    assert np.signbit(O.E2M1_TABLE[8]) and O.E2M1_TABLE[8] == 0.0


def test_e8m0_table():
    for s in range(255):
        assert O.E8M0_TABLE[s] == 2.0 ** (s - 127)
    assert np.isnan(O.E8M0_TABLE[255])


# --------------------------------------------------------------------------
# NF4 packing: hand-worked bytes, ties, zero blocks, page pins
# --------------------------------------------------------------------------
def test_nf4_worked_bytes_and_nibble_order():
    w = np.zeros((1, 64), np.float32)
    w[0, :4] = [0.5, -0.5, 0.25, 0.0]          # absmax 0.5 -> x = 1, -1, 0.5, 0
    packed, absmax = O.quantize_nf4(w)
    assert absmax.tolist() == [[0.5]]
    # codes 15, 0, 12, 7: element 2j in the high nibble, 2j+1 in the low nibble
    assert packed[0, 0] == 0xF0 and packed[0, 1] == 0xC7
    assert np.all(packed[0, 2:] == 0x77)
    d = O.dequant_nf4(packed, absmax, 64)
    assert d[0, 0] == 0.5 and d[0, 1] == -0.5 and d[0, 3] == 0.0
    assert d[0, 2] == np.float64(np.float32(0.44070982933044434)) * 0.5


def test_nf4_ties_go_to_lower_code():
    m = O.nf4_thresholds()
    w = np.zeros((1, 64), np.float32)
    w[0, 0] = 1.0                               # absmax 1 -> x = w exactly
    w[0, 1] = m[7]                              # midpoint of codes 7 and 8
    w[0, 2] = np.nextafter(m[7], np.float32(1))
    w[0, 3] = m[0]                              # midpoint of codes 0 and 1
    packed, _ = O.quantize_nf4(w)
    codes = O.nf4_codes(packed, 64)[0]
    assert codes[:4].tolist() == [15, 7, 8, 0]


def test_nf4_zero_block_and_second_block_scale():
    w = np.zeros((2, 128), np.float32)
    w[1, 64:] = np.linspace(-3, 3, 64, dtype=np.float32)
    packed, absmax = O.quantize_nf4(w)
    assert absmax[0].tolist() == [0.0, 0.0] and absmax[1, 0] == 0.0 and absmax[1, 1] == 3.0
    assert np.all(packed[0] == 0x77) and np.all(packed[1, :32] == 0x77)
    d = O.dequant_nf4(packed, absmax, 128)
    assert np.all(d[0] == 0) and not np.isnan(d).any()
    assert d[1, 64] == -3.0 and d[1, 127] == 3.0


def test_nf4_page_roundtrip_pins():
    g = GOLDEN["nf4_roundtrip"]
    torch.manual_seed(0)
    w = torch.randn(*g["w_shape"]).numpy()
    packed, absmax = O.quantize_nf4(w)
    assert list(packed.shape) == g["packed_shape"] and packed.dtype == np.uint8
    assert list(absmax.shape) == g["absmax_shape"] and absmax.dtype == np.float32
    wq = O.dequant_nf4(packed, absmax, w.shape[1])
    rel = np.linalg.norm(wq - w) / np.linalg.norm(w)
    assert abs(rel - g["rel_err_printed"]) <= g["rel_err_tolerance"]
    p2, a2 = O.quantize_nf4(wq.astype(np.float32))
    assert np.array_equal(p2, packed) and np.array_equal(a2, absmax)


def test_nf4_idempotent_adversarial_blocks():
    rng = np.random.default_rng(3)
    w = rng.standard_normal((16, 256)).astype(np.float32)
    w[0, :64] = 0.0                                    # zero block
    w[1, :64] = 1e-30                                  # tiny constant block
    w[2, :64] = -7.5                                   # constant negative
    w[3, 64:128] = rng.standard_normal(64) * 1e30      # huge values
    w[4, :64] *= 1e-20
    packed, absmax = O.quantize_nf4(w)
    wq = O.dequant_nf4(packed, absmax, 256).astype(np.float32)
    p2, a2 = O.quantize_nf4(wq)
    assert np.array_equal(p2, packed) and np.array_equal(a2, absmax)


# --------------------------------------------------------------------------
# MXFP4 packing
# --------------------------------------------------------------------------
def test_mxfp4_worked_bytes_ties_and_nibble_order():
    w = np.zeros((1, 32), np.float32)
    w[0, :4] = [1.0, -0.375, 0.0625, 0.1875]   # amax 1 -> E = -2, x = 4, -1.5, 0.25, 0.75
    blocks, scales = O.quantize_mxfp4(w)
    assert scales.tolist() == [[125]]
    # codes 6, 11 (=-1.5), 0 (0.25 ties to even code 0), 2 (0.75 ties to code 2)
    # element 2j in the low nibble, 2j+1 in the high nibble
    assert blocks[0, 0] == 0xB6 and blocks[0, 1] == 0x20
    d = O.dequant_mxfp4(blocks, scales, 32)
    assert d[0, :4].tolist() == [1.0, -0.375, 0.0, 0.25]


def test_mxfp4_rounding_grid_ties_even():
    # amax 1.5 -> E = -2; x = 4 w.  Midpoints of the grid and where they land:
    x = np.array([6.0, 0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 5.5, 0.2, 2.6], np.float32)
    w = np.zeros((1, 32), np.float32)
    w[0, :len(x)] = x / 4
    blocks, scales = O.quantize_mxfp4(w)
    codes = O.mxfp4_codes(blocks, 32)[0, :len(x)]
    assert codes.tolist() == [7, 0, 2, 2, 4, 4, 6, 6, 7, 0, 5]


def test_mxfp4_saturation_zero_block_and_sign():
    w = np.zeros((2, 64), np.float32)
    w[0, 0] = 1.9                      # E = -2 -> x = 7.6, saturates to 6 -> 1.5
    w[0, 1] = -0.01
    blocks, scales = O.quantize_mxfp4(w)
    assert scales[0, 0] == 125 and scales[0, 1] == 127 and scales[1].tolist() == [127, 127]
    codes = O.mxfp4_codes(blocks, 64)
    assert codes[0, 0] == 7 and codes[0, 1] == 8          # -0.04 rounds to -0
    assert np.all(codes[1] == 0) and np.all(codes[0, 32:] == 0)
    d = O.dequant_mxfp4(blocks, scales, 64)
    assert d[0, 0] == 1.5 and d[0, 1] == 0.0


def test_mxfp4_page_roundtrip_pins():
    g = GOLDEN["mxfp4_roundtrip"]
    torch.manual_seed(0)
    w = torch.randn(*g["w_shape"]).numpy()
    blocks, scales = O.quantize_mxfp4(w)
    assert list(blocks.reshape(w.shape[0], -1, 16).shape) == g["blocks_shape"]
    assert list(scales.shape) == g["scales_shape"] and scales.dtype == np.uint8
    wq = O.dequant_mxfp4(blocks, scales, w.shape[1])
    rel = np.linalg.norm(wq - w) / np.linalg.norm(w)
    assert abs(rel - g["rel_err_printed"]) <= g["rel_err_tolerance"]
    # exact decode: re-quantizing the decode reproduces the values, and the
    # bytes up to -0 (code 8), which re-quantizes as +0 (code 0)
    b2, s2 = O.quantize_mxfp4(wq.astype(np.float32))
    assert np.array_equal(s2, scales)
    assert np.array_equal(O.dequant_mxfp4(b2, s2, w.shape[1]), wq)
    c1, c2 = O.mxfp4_codes(blocks, w.shape[1]), O.mxfp4_codes(b2, w.shape[1])
    assert np.array_equal(np.where(c1 == 8, 0, c1), c2)


def test_mxfp4_scale_exponent_examples():
    amax = np.array([1.0, 1.5, 2.0, 0.02, 6.0, 0.0, 1e-45, 3e38], np.float32)
    E = O.mxfp4_scale_exponent(amax)
    # floor(log2 amax) - 2, clamped to [-127, 127]; zero block E = 0
    assert E.tolist() == [-2, -2, -1, -8, 0, 0, -127, 125]


# --------------------------------------------------------------------------
# bf16 rounding
# --------------------------------------------------------------------------
def test_bf16_rounding_matches_torch_on_fp32_inputs():
    rng = np.random.default_rng(7)
    v = np.concatenate([
        rng.standard_normal(20000).astype(np.float32),
        (rng.standard_normal(2000) * 1e-39).astype(np.float32),      # subnormals
        np.array([3.3895314e38, -3.3961776e38, 1e-45, 0.0, -0.0], np.float32),
    ])
    # exact ties: bf16 value + half an ulp
    base = rng.standard_normal(2000).astype(np.float32)
    bits = (base.view(np.uint32) & 0xFFFF0000) | 0x8000
    v = np.concatenate([v, bits.view(np.float32)])
    ours = O.bf16_bits(v.astype(np.float64))
    ref = torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)


def test_bf16_rounding_single_step_from_fp64():
    # 1 + 2^-8 + 2^-30 is above the tie: one rounding gives 1 + 2^-7; rounding to
    # fp32 first would land on the tie and go to even (1.0).
    v = np.array([1 + 2.0 ** -8 + 2.0 ** -30, 1 + 2.0 ** -8, -(1 + 3 * 2.0 ** -8)])
    r = O.round_to_bf16(v)
    assert r.tolist() == [1 + 2.0 ** -7, 1.0, -(1 + 4 * 2.0 ** -8)]


# --------------------------------------------------------------------------
# byte accounting
# --------------------------------------------------------------------------
def test_byte_accounting_closed_forms():
    g = GOLDEN["nf4_absmax_share_qwen3_expert"]
    nib = sc = 0
    for N, K in g["projections_NK"]:
        b = O.packed_bytes("nf4", N, K)
        nib += b["nibbles"]
        sc += b["scales"]
    assert sc == g["absmax_bytes"] and nib + sc == g["row_bytes"]
    assert round(100 * sc / (nib + sc), 1) == g["share_percent_printed"]
    bpw = (nib + sc) / (sum(N * K for N, K in g["projections_NK"]))
    assert round(2.0 / bpw, 2) == GOLDEN["nf4_vs_bf16_bytes"]["ratio_printed"]
    m = O.packed_bytes("mxfp4", 2880, 2880)
    assert m["nibbles"] == 2880 * 1440 and m["scales"] == 2880 * 90
