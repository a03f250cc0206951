"""Parity of the MoE glue kernels (SwiGLU, top-k combine) with the oracle, through the C ABI.

SwiGLU: every element within one bf16 rounding of the fp64 value (plus fp32
rounding: (2^-8 + 2^-16) relative, 2^-118 absolute below the fp32 normal range).
Combine: bit for bit the oracle's fp32 slot-order sum. Both at small ragged sizes
and at the full widths of the three workloads, every element. Then one whole MoE
layer (gate_up -> SwiGLU -> down with routing weights and scatter -> combine)
against the oracle's own chain, per-row tolerance.
"""
import numpy as np
import pytest
import torch

import synth
from oracle import glue as GL
from oracle import gnf4_oracle as O
from synth import generators as G
from synth.workloads import WORKLOADS

from gpu_support import bf16_dev, bf16_host_bits, build_stack, check_rows, run_gemm, to_dev

pytestmark = pytest.mark.gpu

SWIGLU_REL = 2.0 ** -8 + 2.0 ** -16
SWIGLU_ABS = 2.0 ** -118


def run_swiglu(h_bits):
    import bit_grouped_moe_gnf4_b200 as g
    out = g.swiglu(bf16_dev(h_bits))
    g.device_status()
    return bf16_host_bits(out)


def run_combine(y_bits, T, k, row_of_slot=None, slot_weight=None):
    import bit_grouped_moe_gnf4_b200 as g
    out = g.combine_topk(bf16_dev(y_bits), T, k, row_of_slot=to_dev(row_of_slot),
                         slot_weight=to_dev(slot_weight))
    g.device_status()
    return bf16_host_bits(out)


def check_swiglu(got_bits, h_bits, what="", max_mismatch=1e-3):
    exact = GL.swiglu_rows_f64(h_bits)
    got = O.bf16_to_f64(got_bits)
    err = np.abs(got - exact)
    bad = err > SWIGLU_REL * np.abs(exact) + SWIGLU_ABS
    assert not bad.any(), f"{what}: {int(bad.sum())} elements off, e.g. got {got[bad][:4]} want {exact[bad][:4]}"
    # the fp32 arithmetic is far finer than bf16: the rounded value almost always matches
    mism = np.mean(got_bits != GL.swiglu_rows(h_bits))
    assert mism < max_mismatch, f"{what}: {mism:.2e} of the elements round differently from the oracle"


def _wide_range_rows(I):
    """Gate values from -120 to 120 (both exp regimes, gradual underflow) against up values."""
    g = np.linspace(-120.0, 120.0, I, dtype=np.float32)
    u = np.resize(np.array([1.0, -3.5, 0.25, 100.0], np.float32), I)
    rows = [np.concatenate([g, u]), np.concatenate([-g, u]), np.concatenate([np.zeros(I, np.float32), u])]
    return G.bf16_bits_from_f32(np.stack(rows))


# --------------------------------------------------------------------------
# SwiGLU
# --------------------------------------------------------------------------
@pytest.mark.parametrize("R,I", [(1, 8), (7, 24), (33, 264)])
def test_swiglu_small(R, I):
    h = G.activations_bf16(1, R, 2 * I, tag="h")
    check_swiglu(run_swiglu(h), h, f"swiglu R={R} I={I}")


def test_swiglu_wide_range_and_zero_rows():
    h = _wide_range_rows(1024)
    # |g| up to 120: the fp32 error grows with |g| (up to 2^-17 relative), so more
    # elements sit near a bf16 rounding boundary; the bound itself is unchanged
    check_swiglu(run_swiglu(h), h, "wide range", max_mismatch=2e-2)
    assert run_swiglu(np.zeros((0, 64), np.uint16)).shape == (0, 32)


@pytest.mark.parametrize("name", ["olmoe_decode_nf4", "qwen3_prefill_nf4", "gptoss_mxfp4"])
def test_swiglu_full_width(name):
    wl = WORKLOADS[name]
    gu = wl.projections[0]
    R = max(wl.T) * wl.top_k[0]
    h = G.activations_bf16(2, R, gu.N, tag="h")
    check_swiglu(run_swiglu(h), h, f"swiglu {name} R={R}")


# --------------------------------------------------------------------------
# combine
# --------------------------------------------------------------------------
@pytest.mark.parametrize("k", [1, 3, 8, 10, 17])
def test_combine_small_bitwise(k):
    T, N = 5, 24
    R = T * k + 3
    y = G.activations_bf16(3, R, N, tag="y")
    rng = np.random.default_rng(k)
    src = rng.integers(0, R, T * k).astype(np.int32)
    src[::7] = -1                                   # dropped slots
    src[1::11] = R + 5                              # out of range: dropped as well
    w = rng.random(T * k).astype(np.float32)
    assert np.array_equal(run_combine(y, T, k, src, w), GL.combine_topk(y, T, k, src, w))
    assert np.array_equal(run_combine(y, T, k, src), GL.combine_topk(y, T, k, src))
    assert np.array_equal(run_combine(y, T, k, None, w), GL.combine_topk(y, T, k, None, w))
    assert np.array_equal(run_combine(y, T, k), GL.combine_topk(y, T, k))


def test_combine_cancellation_is_slot_order():
    y = G.bf16_bits_from_f32(np.array([[1.0] * 8, [2.0 ** 30] * 8, [-(2.0 ** 30)] * 8], np.float32))
    got = run_combine(y, 1, 3)
    assert np.array_equal(got, GL.combine_topk(y, 1, 3))
    assert not got.any()                             # slot order gives 0, the exact sum 1


@pytest.mark.parametrize("name", ["olmoe_decode_nf4", "qwen3_prefill_nf4", "gptoss_mxfp4"])
def test_combine_full_width_bitwise(name):
    wl = WORKLOADS[name]
    dn = wl.projections[1]
    T, k = max(wl.T), wl.top_k[0]
    b = synth.make_routed_batch(4, T, wl.E, k)
    y = G.activations_bf16(4, T * k, dn.N, tag="y")
    # scattered rows (row_dest = t*k + slot), weights already applied
    assert np.array_equal(run_combine(y, T, k), GL.combine_topk(y, T, k))
    # expert-sorted rows: the row of each (token, slot) and its routing weight
    row_of_slot = np.empty(T * k, np.int32)
    row_of_slot[b.row_dest] = np.arange(b.R, dtype=np.int32)
    w = b.weights.reshape(-1).astype(np.float32)
    assert np.array_equal(run_combine(y, T, k, row_of_slot, w), GL.combine_topk(y, T, k, row_of_slot, w))


def test_combine_row_count_invariance():
    T, k, N = 160, 8, 2048
    y = G.activations_bf16(5, T * k, N, tag="y")
    full = run_combine(y, T, k)
    for t in (0, 77, 159):
        alone = run_combine(y[t * k:(t + 1) * k], 1, k)
        assert np.array_equal(alone[0], full[t])
    seventeen = run_combine(y[:17 * k], 17, k)
    assert np.array_equal(seventeen, full[:17])


# --------------------------------------------------------------------------
# one MoE layer end to end
# --------------------------------------------------------------------------
@pytest.mark.parametrize("fmt,T,k", [("nf4", 12, 2), ("nf4", 300, 8), ("mxfp4", 40, 4)])
def test_moe_layer_chain(fmt, T, k):
    """gate_up (gathers token rows) -> SwiGLU -> down (routing weight, scatter to
    t*k + slot) -> combine, on the GPU and in the oracle (bf16 between steps, as
    the method stores them); per-row tolerance on the combined rows."""
    import bit_grouped_moe_gnf4_b200 as g
    E, H, I = 8, 256, 128
    Wg, Sg, Wgh, Sgh = build_stack(fmt, E, 2 * I, H, seed=6, tag="w")
    Wdn, Sdn, Wdh, Sdh = build_stack(fmt, E, H, I, seed=6, tag="w_down")
    b = synth.make_routed_batch(6, T, E, k)
    x = synth.activations_bf16(6, T, H)
    # oracle chain
    h_ref = O.grouped_gemm(fmt, x, Wgh, Sgh, b.offsets, row_token=b.row_token)
    a_ref = GL.swiglu_rows(h_ref)
    y_ref = O.grouped_gemm(fmt, a_ref, Wdh, Sdh, b.offsets, row_weight=b.row_weight,
                           row_dest=b.row_dest, T_out=T * k)
    ref = GL.combine_topk_f64(y_ref, T, k)
    # CUDA chain, device buffers only
    off, tok = to_dev(b.offsets), to_dev(b.row_token)
    h = g.grouped_gemm(fmt, bf16_dev(x), Wg, Sg, off, row_token=tok, T_out=b.R)
    a = g.swiglu(h)
    y = g.grouped_gemm(fmt, a, Wdn, Sdn, off, row_weight=to_dev(b.row_weight),
                       row_dest=to_dev(b.row_dest), T_out=T * k)
    out = g.combine_topk(y, T, k)
    g.device_status()
    check_rows(bf16_host_bits(out), ref, f"layer {fmt} T={T} k={k}")
