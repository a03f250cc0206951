"""Parity of the grouped input gradient (dgrad) with the oracle, through the C ABI.

Per-row tolerance 2e-2 * max|row| against the oracle's exact fp64 gradient: small
ragged cases on every element (both row-tile shapes of the kernel, gathered
gradient rows, routing weights, empty experts), the three workloads' full shapes
on sampled rows, one-hot gradients (MXFP4: exactly the dequantized weight row),
determinism, the GNF4_CHECK path and the empty call.
"""
import numpy as np
import pytest
import torch

import synth
from oracle import dgrad as D
from oracle import gnf4_oracle as O
from synth import generators as G
from synth.workloads import WORKLOADS

from gpu_support import (bf16_dev, bf16_host_bits, build_stack, check_group_frobenius, check_rows,
                         sample_rows, to_dev)

pytestmark = pytest.mark.gpu


def run_dgrad(fmt, g_bits, Wd, Sd, offsets, row_src=None, row_weight=None, flags=0):
    import bit_grouped_moe_gnf4_b200 as g
    R = int(offsets[-1])
    out = g.dgrad(fmt, bf16_dev(g_bits), Wd, Sd, to_dev(np.asarray(offsets, np.int64)),
                  row_src=to_dev(row_src), row_weight=to_dev(row_weight), R=R, flags=flags)
    g.device_status()
    return bf16_host_bits(out)


@pytest.mark.parametrize("fmt", ["nf4", "mxfp4"])
@pytest.mark.parametrize("counts", [[1, 0, 17, 40], [50, 0, 70, 33], [3], [0, 0, 130, 0, 1]])
def test_small_ragged_all_elements(fmt, counts):
    E, N, K = len(counts), 144, 320                       # 9 steps of 16; 5 column tiles of 64
    Wd, Sd, Wh, Sh = build_stack(fmt, E, N, K, seed=21)
    b = G.explicit_batch(counts, seed=22)
    T_in = b.R + 5
    g = synth.activations_bf16(23, T_in, N, tag="y")
    src = np.random.default_rng(24).permutation(T_in)[:b.R].astype(np.int32)
    got = run_dgrad(fmt, g, Wd, Sd, b.offsets, src, b.row_weight)
    ref = D.dgrad_rows_f64(fmt, g, Wh, Sh, b.offsets, src, b.row_weight, np.arange(b.R))
    check_rows(got, ref, f"dgrad {fmt} {counts}")
    check_group_frobenius(got, ref, b.offsets, f"dgrad {fmt} {counts}")
    # rows already in routed order, no weight
    got2 = run_dgrad(fmt, g[:b.R], Wd, Sd, b.offsets)
    ref2 = D.dgrad_rows_f64(fmt, g[:b.R], Wh, Sh, b.offsets, None, None, np.arange(b.R))
    check_rows(got2, ref2, f"dgrad {fmt} {counts} plain")


@pytest.mark.parametrize("fmt", ["nf4", "mxfp4"])
def test_two_row_tiles_with_split_contraction(fmt):
    """Groups averaging 66 rows over a narrow K: the host picks two 16-row tiles per item
    and an 8-way split of the contraction (partial sums added through shared memory)."""
    counts, N, K = [100, 0, 60, 40], 512, 128
    Wd, Sd, Wh, Sh = build_stack(fmt, len(counts), N, K, seed=34)
    b = G.explicit_batch(counts, seed=35)
    g = synth.activations_bf16(36, b.R, N, tag="y")
    got = run_dgrad(fmt, g, Wd, Sd, b.offsets, None, b.row_weight)
    ref = D.dgrad_rows_f64(fmt, g, Wh, Sh, b.offsets, None, b.row_weight, np.arange(b.R))
    check_rows(got, ref, f"dgrad {fmt} RT=2 split")


def test_one_hot_mxfp4_reads_the_weight_row_exactly():
    E, N, K = 2, 64, 256
    Wd, Sd, Wh, Sh = build_stack("mxfp4", E, N, K, seed=25)
    offsets = np.array([0, N, 2 * N], np.int64)
    g = np.zeros((2 * N, N), np.uint16)
    for r in range(2 * N):
        g[r, r % N] = 0x3F80
    got = O.bf16_to_f64(run_dgrad("mxfp4", g, Wd, Sd, offsets))
    for e in range(E):
        want = O.bf16_to_f64(O.bf16_bits(O.decode_expert("mxfp4", Wh, Sh, e, K)))
        assert np.array_equal(got[e * N:(e + 1) * N], want)


def _projection_case(name, proj_index, seed):
    wl = WORKLOADS[name]
    proj = wl.projections[proj_index]
    T, k = max(wl.T), wl.top_k[0]
    b = synth.make_routed_batch(seed, T, wl.E, k)
    rows, experts = sample_rows(b.offsets, max_rows=48, max_experts=5, seed=seed)
    Wd, Sd, Wh, Sh = build_stack(wl.fmt, wl.E, proj.N, proj.K, seed=seed, oracle_experts=experts,
                                 tag="w" if proj.name == "gate_up" else "w_down")
    return wl, proj, b, rows, Wd, Sd, Wh, Sh


@pytest.mark.parametrize("name", ["olmoe_decode_nf4", "qwen3_prefill_nf4", "gptoss_mxfp4"])
def test_full_shapes_sampled_rows(name):
    for pi in (0, 1):
        wl, proj, b, rows, Wd, Sd, Wh, Sh = _projection_case(name, pi, seed=26 + pi)
        if proj.name == "down":
            # the forward scattered row r to t*k + slot with weight w(r): gather the
            # gradient from there and weight it
            g = synth.activations_bf16(27, b.T * b.k, proj.N, tag="y")
            src, wt = b.row_dest, b.row_weight
        else:
            g = synth.activations_bf16(27, b.R, proj.N, tag="y")
            src, wt = None, None
        got = run_dgrad(wl.fmt, g, Wd, Sd, b.offsets, src, wt)
        ref = D.dgrad_rows_f64(wl.fmt, g, Wh, Sh, b.offsets, src, wt, rows)
        check_rows(got[rows], ref, f"dgrad {name} {proj.name}")


def test_olmoe_t1_all_rows():
    wl = WORKLOADS["olmoe_decode_nf4"]
    dn = wl.projections[1]
    b = synth.make_routed_batch(28, 1, wl.E, 8)
    Wd, Sd, Wh, Sh = build_stack("nf4", wl.E, dn.N, dn.K, seed=28, oracle_experts=b.active_experts(),
                                 tag="w_down")
    g = synth.activations_bf16(29, b.T * b.k, dn.N, tag="y")
    got = run_dgrad("nf4", g, Wd, Sd, b.offsets, b.row_dest, b.row_weight)
    ref = D.dgrad_rows_f64("nf4", g, Wh, Sh, b.offsets, b.row_dest, b.row_weight, np.arange(b.R))
    check_rows(got, ref, "dgrad OLMoE T=1 down")


def test_deterministic_over_calls():
    E, N, K = 8, 512, 512
    Wd, Sd, _, _ = build_stack("nf4", E, N, K, seed=30, oracle_experts=[])
    b = synth.make_routed_batch(31, 200, E, 2)
    g = synth.activations_bf16(32, b.R, N, tag="y")
    first = run_dgrad("nf4", g, Wd, Sd, b.offsets)
    for _ in range(20):
        assert np.array_equal(run_dgrad("nf4", g, Wd, Sd, b.offsets), first)


def test_check_flag_and_empty_call():
    import bit_grouped_moe_gnf4_b200 as gg
    E, N, K = 2, 64, 128
    Wd, Sd, _, _ = build_stack("nf4", E, N, K, seed=33, oracle_experts=[])
    offsets = to_dev(np.array([0, 2, 4], np.int64))
    g = torch.zeros((4, N), dtype=torch.bfloat16, device="cuda")
    bad = to_dev(np.array([0, 1, 9, 2], np.int32))        # 9 >= T_in
    with pytest.raises(gg.Gnf4Error) as ei:
        gg.dgrad("nf4", g, Wd, Sd, offsets, row_src=bad, flags=gg.GNF4_CHECK)
    assert ei.value.status == 5
    out = gg.dgrad("nf4", g[:0], Wd, Sd, to_dev(np.zeros(E + 1, np.int64)), R=0)
    assert out.shape == (0, K)
