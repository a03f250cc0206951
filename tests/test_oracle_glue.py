"""Pins for the oracle's SwiGLU and top-k combine (CPU only).

SwiGLU: closed forms of the logistic function (sigmoid(0) = 1/2,
sigmoid(ln 3) = 3/4), the identity silu(x) - silu(-x) = x, the library logistic
(scipy.special.expit), its limits, and which half of the row is the gate.
Combine: identity for k = 1, cancellation cases whose slot-order fp32 result
differs from both the exact sum and the reversed order, a brute-force fp32
re-implementation with struct rounding and integer bf16 rounding, the accuracy
bound of an fp32 running sum, dropped slots and row-count invariance.
"""
import math
import struct

import numpy as np
import pytest
from scipy.special import expit

from oracle import gnf4_oracle as O
from oracle import glue as GL
from synth import generators as G


def _bits(vals):
    """Exact bf16 values -> bits (asserts they are on the bf16 grid)."""
    v = np.asarray(vals, dtype=np.float64)
    b = O.bf16_bits(v)
    assert np.array_equal(O.bf16_to_f64(b), v), "test value is not a bf16 value"
    return b


# --------------------------------------------------------------------------
# SwiGLU
# --------------------------------------------------------------------------
def test_silu_closed_forms():
    ln3 = math.log(3.0)
    got = GL.silu_f64(np.array([0.0, ln3, -ln3]))
    assert got[0] == 0.0
    assert got[1] == pytest.approx(0.75 * ln3, rel=1e-15)
    assert got[2] == pytest.approx(-0.25 * ln3, rel=1e-15)


def test_silu_odd_part_identity():
    # sigmoid(x) + sigmoid(-x) = 1, hence silu(x) - silu(-x) = x
    x = np.random.default_rng(1).standard_normal(1000) * 8
    d = GL.silu_f64(x) - GL.silu_f64(-x)
    assert np.allclose(d, x, rtol=1e-13, atol=1e-13)


def test_silu_matches_library_logistic():
    x = np.concatenate([np.linspace(-40, 40, 4001), [-700.0, -1000.0, 1000.0]])
    ref = x * expit(x)
    assert np.allclose(GL.silu_f64(x), ref, rtol=1e-14, atol=1e-300)
    # limits: silu(x) -> x above, -> -0 far below
    assert GL.silu_f64(np.array([1000.0]))[0] == 1000.0
    far = GL.silu_f64(np.array([-1000.0]))[0]
    assert far == 0.0 and math.copysign(1.0, far) == -1.0


def test_swiglu_gate_is_first_half():
    ln3_b = float(O.bf16_to_f64(O.bf16_bits(np.array([math.log(3.0)])))[0])
    I = 4
    gate = np.array([0.0, ln3_b, 2.0, -3.0])
    up = np.array([123.0, 2.0, 0.0, 1.0])
    h = _bits(np.concatenate([gate, up]).reshape(1, 2 * I))
    got = GL.swiglu_rows_f64(h)[0]
    exp = gate * expit(gate) * up
    assert got[0] == 0.0                      # silu(0) = 0 whatever the up value
    assert got[2] == 0.0                      # up = 0
    assert np.allclose(got, exp, rtol=1e-14)
    # swapping the halves gives a different row (the pin would catch a transposed layout)
    swapped = up * expit(up) * gate
    assert not np.allclose(got, swapped)


def test_swiglu_rounds_once_to_bf16():
    h = G.activations_bf16(3, 16, 64, tag="h")
    exact = GL.swiglu_rows_f64(h)
    got = O.bf16_to_f64(GL.swiglu_rows(h))
    nz = exact != 0
    # one round-to-nearest step: within half a bf16 unit in the last place (8 significant bits)
    assert np.all(np.abs(got[nz] - exact[nz]) <= np.abs(exact[nz]) * 2.0 ** -8)
    # and it is the nearest bf16: the neighbours on either side are no closer
    bits = GL.swiglu_rows(h).astype(np.int32)
    for d in (-1, 1):
        nb = O.bf16_to_f64((bits + d).astype(np.uint16))
        assert np.all(np.abs(nb - exact) >= np.abs(got - exact))


# --------------------------------------------------------------------------
# combine
# --------------------------------------------------------------------------
def _f32(v: float) -> float:
    return struct.unpack("<f", struct.pack("<f", v))[0]


def _bf16_rne_from_f32(v: float) -> int:
    u = struct.unpack("<I", struct.pack("<f", v))[0]
    return ((u + 0x7FFF + ((u >> 16) & 1)) >> 16) & 0xFFFF


def _brute_combine(y_bits, T, k, src, w):
    """Scalar loops, fp32 rounding by struct, bf16 rounding on the integer bits."""
    R, N = y_bits.shape
    y = O.bf16_to_f64(y_bits)
    out = np.zeros((T, N), np.uint16)
    for t in range(T):
        for n in range(N):
            acc = 0.0
            for s in range(k):
                r = int(src[t * k + s])
                if 0 <= r < R:
                    acc = _f32(acc + _f32(float(w[t * k + s]) * float(y[r, n])))
            out[t, n] = _bf16_rne_from_f32(acc)
    return out


def test_combine_k1_is_identity():
    y = G.activations_bf16(1, 9, 24, tag="y")
    assert np.array_equal(GL.combine_topk(y, 9, 1), y)


def test_combine_is_slot_order_not_exact_nor_reversed():
    big = 2.0 ** 30
    # slots (1, 2^30, -2^30): slot order 1 + 2^30 rounds to 2^30 in fp32, then 0;
    # the exact sum is 1, and the reversed order gives 1 as well
    y = _bits(np.array([[1.0], [big], [-big]]))
    got = O.bf16_to_f64(GL.combine_topk(y, 1, 3))[0, 0]
    assert got == 0.0
    assert GL.combine_topk_f64(y, 1, 3)[0, 0] == 1.0
    rev = GL.combine_topk(y, 1, 3, row_of_slot=np.array([2, 1, 0]))
    assert O.bf16_to_f64(rev)[0, 0] == 1.0


def test_combine_rounds_product_then_sum_no_fma():
    # slot 0 gives -(1 + 2^-7); slot 1 the product (1 + 2^-23)(1 + 2^-7), whose 2^-30 term
    # the fp32 product drops: the sum is 2^-23. A fused multiply-add would keep it and give
    # 2^-23 (1 + 2^-7), a different bf16 value.
    w = np.array([1.0, 1.0 + 2.0 ** -23], np.float32)
    y = _bits(np.array([[-(1.0 + 2.0 ** -7)], [1.0 + 2.0 ** -7]]))
    got = O.bf16_to_f64(GL.combine_topk(y, 1, 2, slot_weight=w))[0, 0]
    assert got == 2.0 ** -23
    assert GL.combine_topk_f64(y, 1, 2, slot_weight=w)[0, 0] == 2.0 ** -23 * (1 + 2.0 ** -7)


def test_combine_brute_force_with_gather_weights_and_dropped_slot():
    T, k, N, R = 3, 4, 5, 13
    y = G.activations_bf16(5, R, N, tag="y")
    rng = np.random.default_rng(2)
    src = rng.permutation(R)[:T * k].astype(np.int32)
    src[5] = -1                                # a dropped slot
    src[10] = R                                # out of range: dropped as well
    w = rng.random(T * k).astype(np.float32)
    got = GL.combine_topk(y, T, k, row_of_slot=src, slot_weight=w)
    assert np.array_equal(got, _brute_combine(y, T, k, src, w))
    got_plain = GL.combine_topk(y[:T * k], T, k)
    assert np.array_equal(got_plain, _brute_combine(y[:T * k], T, k, np.arange(T * k), np.ones(T * k)))


def test_combine_accuracy_bound():
    T, k, N = 64, 8, 32
    y = G.activations_bf16(6, T * k, N, tag="y")
    w = np.random.default_rng(3).random(T * k).astype(np.float32)
    got = O.bf16_to_f64(GL.combine_topk(y, T, k, slot_weight=w))
    exact = GL.combine_topk_f64(y, T, k, slot_weight=w)
    # running fp32 sum of k rounded products: |err| <= (k+1) u sum|w y| (u = 2^-24),
    # then one bf16 rounding: half a unit of 8 significant bits
    yv = O.bf16_to_f64(y).reshape(T, k, N)
    mag = np.sum(np.abs(w.reshape(T, k, 1).astype(np.float64) * yv), axis=1)
    bound = (k + 1) * 2.0 ** -24 * mag + 2.0 ** -8 * (np.abs(exact) + (k + 1) * 2.0 ** -24 * mag)
    assert np.all(np.abs(got - exact) <= bound)


def test_combine_row_count_invariance():
    T, k, N = 40, 8, 16
    y = G.activations_bf16(7, T * k, N, tag="y")
    full = GL.combine_topk(y, T, k)
    for t in (0, 17, 39):
        alone = GL.combine_topk(y[t * k:(t + 1) * k], 1, k)
        assert np.array_equal(alone[0], full[t])


def test_combine_empty():
    y = np.zeros((0, 8), np.uint16)
    assert GL.combine_topk(y, 3, 2).shape == (3, 8)
    assert not GL.combine_topk(y, 3, 2).any()
    assert GL.combine_topk(np.zeros((4, 8), np.uint16), 0, 2).shape == (0, 8)
