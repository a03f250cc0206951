"""Grouped GEMM parity: the CUDA path through the C ABI against the oracle.

Small cases are compared on every output element; the full-size workloads on
sampled routed rows (each sample keeps the first and last row of its groups);
bands are exercised one at a time with the FORCE flags and together.
"""
import numpy as np
import pytest
import torch

import synth
from oracle import gnf4_oracle as O
from synth import generators as G
from synth.workloads import WORKLOADS

from gpu_support import (bf16_dev, bf16_host_bits, build_stack, check_group_frobenius, check_rows,
                         run_gemm, sample_rows, to_dev)

pytestmark = pytest.mark.gpu

BANDS = {"auto": 0, "decode": 0x2, "prefill": 0x4}


def _ref_rows(fmt, x, Wh, Sh, b, rows, weighted=True):
    return O.grouped_rows_f64(fmt, x, Wh, Sh, b.offsets, b.row_token,
                              b.row_weight if weighted else None, Wh.shape[2] * 2, rows)


# --------------------------------------------------------------------------
# tiny workload, every element
# --------------------------------------------------------------------------
@pytest.mark.parametrize("fmt", ["nf4", "mxfp4"])
@pytest.mark.parametrize("band", list(BANDS))
def test_tiny_all_elements(fmt, band):
    E, k, T, K, N = 4, 2, 8, 256, 128
    Wd, Sd, Wh, Sh = build_stack(fmt, E, N, K)
    b = synth.make_routed_batch(0, T, E, k)
    x = synth.activations_bf16(0, T, K)
    out = run_gemm(fmt, x, Wd, Sd, b.offsets, b.row_token, b.row_weight, b.row_dest,
                   T_out=T * k, flags=BANDS[band])
    ref = O.grouped_rows_f64(fmt, x, Wh, Sh, b.offsets, b.row_token, b.row_weight, K, np.arange(b.R))
    check_rows(out[b.row_dest], ref, f"tiny {fmt} {band}")
    check_group_frobenius(out[b.row_dest], ref, b.offsets, f"tiny {fmt} {band}")


@pytest.mark.parametrize("fmt", ["nf4", "mxfp4"])
@pytest.mark.parametrize("band", list(BANDS))
def test_ragged_groups_several_tiles(fmt, band):
    """N = 400 (25 row tiles of 16, 3 full tiles of 128 plus a ragged one), groups
    of 0..150 rows (token chunks with ragged tails), K = 640."""
    E, N, K = 7, 400, 640
    counts = [1, 0, 150, 9, 33, 0, 70]
    Wd, Sd, Wh, Sh = build_stack(fmt, E, N, K, seed=3)
    b = G.explicit_batch(counts, seed=5)
    x = synth.activations_bf16(9, b.T, K)
    out = run_gemm(fmt, x, Wd, Sd, b.offsets, b.row_token, b.row_weight, b.row_dest,
                   T_out=b.R, flags=BANDS[band])
    ref = O.grouped_rows_f64(fmt, x, Wh, Sh, b.offsets, b.row_token, b.row_weight, K, np.arange(b.R))
    check_rows(out[b.row_dest], ref, f"ragged {fmt} {band}")
    check_group_frobenius(out[b.row_dest], ref, b.offsets, f"ragged {fmt} {band}")


@pytest.mark.parametrize("fmt", ["nf4", "mxfp4"])
def test_decode_table_exhaustive_bitwise(fmt):
    """Every byte value 0..255 in every position: with x = identity the output is
    the decoded weight matrix (transposed) rounded to bf16, exactly."""
    N, K = 16, 512
    Wh = np.zeros((1, N, K // 2), np.uint8)
    for n in range(N):
        Wh[0, n] = (np.arange(256) + 17 * n) % 256
    if fmt == "nf4":
        Sh = np.ones((1, N, K // 64), np.float32)
    else:
        Sh = np.full((1, N, K // 32), 127, np.uint8)
    x = np.zeros((K, K), np.uint16)
    x[np.arange(K), np.arange(K)] = 0x3F80                 # bf16 1.0
    offs = np.array([0, K], np.int64)
    for flags in (0x2, 0x4):
        out = run_gemm(fmt, x, to_dev(Wh), to_dev(Sh), offs, flags=flags)
        want = O.bf16_bits(O.decode_expert(fmt, Wh, Sh, 0, K).T)
        got_v, want_v = O.bf16_to_f64(out), O.bf16_to_f64(want)
        assert np.array_equal(got_v, want_v), f"flags {flags}"


@pytest.mark.parametrize("fmt", ["nf4", "mxfp4"])
def test_permutation_weights_bitwise(fmt):
    N = K = 256
    perm = np.random.default_rng(11).permutation(K)
    w = np.zeros((N, K), np.float32)
    w[np.arange(N), perm] = 1.0
    p, s = (O.quantize_nf4 if fmt == "nf4" else O.quantize_mxfp4)(w)
    T = 40
    x = synth.activations_bf16(12, T, K)
    for flags in (0x2, 0x4):
        out = run_gemm(fmt, x, to_dev(p[None]), to_dev(s[None]), np.array([0, T], np.int64), flags=flags)
        assert np.array_equal(out, x[:, perm])


# --------------------------------------------------------------------------
# full-size workloads
# --------------------------------------------------------------------------
@pytest.fixture(scope="module")
def olmoe_stacks():
    wl = WORKLOADS["olmoe_decode_nf4"]
    gu, dn = wl.projections
    return {
        "gate_up": build_stack("nf4", wl.E, gu.N, gu.K, seed=0, tag="w"),
        "down": build_stack("nf4", wl.E, dn.N, dn.K, seed=0, tag="w_down"),
    }


def _run_projection(fmt, proj, stack, b, rows=None, flags=0, seed=0):
    """gate_up reads token rows and writes sorted rows; down reads sorted rows,
    weights them and scatters to t*k + slot."""
    Wd, Sd, Wh, Sh = stack
    K = proj.K
    if proj.name == "gate_up":
        x = synth.activations_bf16(seed, b.T, K)
        out = run_gemm(fmt, x, Wd, Sd, b.offsets, row_token=b.row_token, T_out=b.R, flags=flags)
        rows = np.arange(b.R) if rows is None else rows
        ref = O.grouped_rows_f64(fmt, x, Wh, Sh, b.offsets, b.row_token, None, K, rows)
        got = out[rows]
    else:
        x = synth.activations_bf16(seed, b.R, K, tag="x_down")
        out = run_gemm(fmt, x, Wd, Sd, b.offsets, row_weight=b.row_weight, row_dest=b.row_dest,
                       T_out=b.T * b.k, flags=flags)
        rows = np.arange(b.R) if rows is None else rows
        ref = O.grouped_rows_f64(fmt, x, Wh, Sh, b.offsets, None, b.row_weight, K, rows)
        got = out[b.row_dest[rows]]
    return check_rows(got, ref, f"{proj.name} T={b.T}")


@pytest.mark.parametrize("T", [1, 16])
def test_olmoe_decode_full(olmoe_stacks, T):
    wl = WORKLOADS["olmoe_decode_nf4"]
    b = synth.make_routed_batch(0, T, wl.E, 8)
    for proj in wl.projections:
        _run_projection("nf4", proj, olmoe_stacks[proj.name], b)


@pytest.mark.parametrize("T,k", [(t, k) for k in (1, 8) for t in (1, 4, 16, 64, 256, 1024, 4096, 8192)])
def test_olmoe_zipf_sweep_sampled(olmoe_stacks, T, k):
    wl = WORKLOADS["olmoe_sweep_nf4"]
    b = synth.make_routed_batch(1, T, wl.E, k, routing="zipf")
    rows, _ = sample_rows(b.offsets, max_rows=48, seed=T + k)
    for proj in wl.projections:
        _run_projection("nf4", proj, olmoe_stacks[proj.name], b, rows=rows, seed=2)


def test_qwen3_prefill_sampled():
    wl = WORKLOADS["qwen3_prefill_nf4"]
    b = synth.make_routed_batch(0, 4096, wl.E, 8)
    rows, experts = sample_rows(b.offsets, max_rows=64, max_experts=4, seed=3)
    for proj, tag in zip(wl.projections, ("w", "w_down")):
        stack = build_stack("nf4", wl.E, proj.N, proj.K, seed=0, oracle_experts=experts, tag=tag)
        _run_projection("nf4", proj, stack, b, rows=rows)
        del stack
        torch.cuda.empty_cache()


def test_prefill_acat_matches_fused_gather():
    """The pages' interface passes a_cat (token rows already in routed order); the
    fused gather reads x[row_token[r]] itself. Same activation bytes, same decode and
    MMAs: the two must give identical bits, and both match the oracle."""
    E, T, k, K, N = 16, 512, 8, 2048, 512
    b = synth.make_routed_batch(2, T, E, k)
    assert np.diff(b.offsets).max() > 64            # the prefill band takes these groups
    rows, experts = sample_rows(b.offsets, max_rows=48, max_experts=3, seed=5)
    Wd, Sd, Wh, Sh = build_stack("nf4", E, N, K, seed=2, oracle_experts=experts)
    x = synth.activations_bf16(2, T, K)
    x_cat = np.ascontiguousarray(x[b.row_token])
    fused = run_gemm("nf4", x, Wd, Sd, b.offsets, row_token=b.row_token, T_out=b.R)
    acat = run_gemm("nf4", x_cat, Wd, Sd, b.offsets, T_out=b.R)
    assert np.array_equal(fused, acat)               # run_gemm returns the bf16 bits on the host
    ref = O.grouped_rows_f64("nf4", x, Wh, Sh, b.offsets, b.row_token, None, K, rows)
    check_rows(acat[rows], ref, "a_cat prefill")


@pytest.mark.parametrize("T", [1, 8, 64])
def test_gptoss_mxfp4(T):
    wl = WORKLOADS["gptoss_mxfp4"]
    b = synth.make_routed_batch(0, T, wl.E, 4)
    if T == 1:
        rows, experts = np.arange(b.R), [int(e) for e in b.active_experts()]
    else:
        rows, experts = sample_rows(b.offsets, max_rows=32, max_experts=4, seed=T)
    for proj, tag in zip(wl.projections, ("w", "w_down")):
        stack = build_stack("mxfp4", wl.E, proj.N, proj.K, seed=0, oracle_experts=experts, tag=tag)
        _run_projection("mxfp4", proj, stack, b, rows=rows)
        del stack
        torch.cuda.empty_cache()


# --------------------------------------------------------------------------
# properties
# --------------------------------------------------------------------------
@pytest.mark.parametrize("band", ["decode", "prefill"])
def test_deterministic_50_calls(olmoe_stacks, band):
    import bit_grouped_moe_gnf4_b200 as g
    Wd, Sd, _, _ = olmoe_stacks["gate_up"]
    b = synth.make_routed_batch(4, 64 if band == "decode" else 512, 64, 8)
    x = bf16_dev(synth.activations_bf16(4, b.T, 2048))
    off, tok = to_dev(b.offsets), to_dev(b.row_token)
    outs = set()
    for _ in range(50):
        out = g.grouped_gemm("nf4", x, Wd, Sd, off, row_token=tok, flags=BANDS[band])
        outs.add(bytes(out.view(torch.int16).cpu().numpy().tobytes()))
    assert len(outs) == 1


@pytest.mark.parametrize("band", ["decode", "prefill"])
def test_row_count_invariance(olmoe_stacks, band):
    """A token computed alone and inside 16-, 17- and 160-token calls to the same
    expert gets the same bits (within one band)."""
    import bit_grouped_moe_gnf4_b200 as g
    Wd, Sd, _, _ = olmoe_stacks["gate_up"]
    x_all = synth.activations_bf16(5, 160, 2048)
    x = bf16_dev(x_all)
    e = 9
    results = []
    for m in (1, 16, 17, 160):
        offs = np.zeros(65, np.int64)
        offs[e + 1:] = m
        tok = np.arange(m, dtype=np.int32)[::-1].copy()    # token 0 is the last row
        out = g.grouped_gemm("nf4", x, Wd, Sd, to_dev(offs), row_token=to_dev(tok), flags=BANDS[band])
        results.append(bf16_host_bits(out)[m - 1])
    for r in results[1:]:
        assert np.array_equal(r, results[0])


def test_empty_experts_scatter_and_canary(olmoe_stacks):
    """Rows no routed row names keep their (NaN canary) contents; guard rows before
    and after the written range are untouched."""
    Wd, Sd, Wh, Sh = olmoe_stacks["down"]
    counts = np.zeros(64, np.int64)
    counts[[3, 17, 40, 63]] = [5, 1, 90, 2]
    b = G.explicit_batch(counts, seed=7)
    T_out = b.R + 50
    rng = np.random.default_rng(8)
    dest = rng.permutation(T_out)[:b.R].astype(np.int32)
    canary = np.full((T_out, Wd.shape[1]), 0x7FC1, np.uint16)
    x = synth.activations_bf16(6, b.R, 1024)
    for band, flags in BANDS.items():
        out = run_gemm("nf4", x, Wd, Sd, b.offsets, row_weight=b.row_weight, row_dest=dest,
                       out_init_bits=canary, flags=flags)
        untouched = np.setdiff1d(np.arange(T_out), dest)
        assert np.all(out[untouched] == 0x7FC1), band
        ref = O.grouped_rows_f64("nf4", x, Wh, Sh, b.offsets, None, b.row_weight, 1024, np.arange(b.R))
        check_rows(out[dest], ref, f"canary {band}")


def test_expert_relabelling(olmoe_stacks):
    import bit_grouped_moe_gnf4_b200 as g
    Wd, Sd, _, _ = olmoe_stacks["gate_up"]
    b = synth.make_routed_batch(6, 40, 64, 8)
    x = bf16_dev(synth.activations_bf16(7, 40, 2048))
    out1 = g.grouped_gemm("nf4", x, Wd, Sd, to_dev(b.offsets), row_token=to_dev(b.row_token),
                          row_dest=to_dev(b.row_dest), T_out=b.R)
    perm = np.random.default_rng(3).permutation(64)
    W2, S2 = torch.empty_like(Wd), torch.empty_like(Sd)
    W2[torch.from_numpy(perm).cuda()] = Wd
    S2[torch.from_numpy(perm).cuda()] = Sd
    off2, tok2, _, dst2 = G.routing_metadata(perm[b.ids].astype(np.int32), b.weights, 64)
    out2 = g.grouped_gemm("nf4", x, W2, S2, to_dev(off2), row_token=to_dev(tok2),
                          row_dest=to_dev(dst2), T_out=b.R)
    assert torch.equal(out1.view(torch.int16), out2.view(torch.int16))


def test_int64_expert_offsets_past_2gib():
    """A stack of 2.4 GB: the only active expert starts past byte 2^31."""
    E, N, K = 72, 4096, 16384
    assert (E - 1) * N * (K // 2) > 2 ** 31
    e = E - 1
    p, s = O.quantize_nf4(G.expert_weights(0, e, N, K))
    Wd = torch.zeros((E, N, K // 2), dtype=torch.uint8, device="cuda")
    Sd = torch.zeros((E, N, K // 64), dtype=torch.float32, device="cuda")
    Wd[e] = torch.from_numpy(p).cuda()
    Sd[e] = torch.from_numpy(s).cuda()
    T = 3
    offs = np.zeros(E + 1, np.int64)
    offs[E] = T
    x = synth.activations_bf16(8, T, K)
    for flags in (0x2, 0x4):
        out = run_gemm("nf4", x, Wd, Sd, offs, flags=flags)
        Wh = np.zeros((1, N, K // 2), np.uint8)
        Wh[0] = p
        ref = O.grouped_rows_f64("nf4", x, Wh, s[None], np.array([0, T]), None, None, K, np.arange(T))
        check_rows(out, ref, "int64 boundary")
    del Wd, Sd
    torch.cuda.empty_cache()


def test_device_check_flags_bad_routing():
    import bit_grouped_moe_gnf4_b200 as g
    Wd, Sd, _, _ = build_stack("nf4", 4, 64, 128, seed=1)
    x = bf16_dev(synth.activations_bf16(1, 8, 128))
    bad_offsets = to_dev(np.array([0, 5, 3, 8, 8], np.int64))
    with pytest.raises(g.Gnf4Error) as ei:
        g.grouped_gemm("nf4", x, Wd, Sd, bad_offsets, flags=g.GNF4_CHECK, R=8)
    assert ei.value.status == 5
    tok = to_dev(np.array([0, 1, 2, 3, 4, 5, 6, 99], np.int32))
    with pytest.raises(g.Gnf4Error) as ei:
        g.grouped_gemm("nf4", x, Wd, Sd, to_dev(np.array([0, 2, 4, 6, 8], np.int64)), row_token=tok,
                       flags=g.GNF4_CHECK)
    assert ei.value.status == 5
    ok = g.grouped_gemm("nf4", x, Wd, Sd, to_dev(np.array([0, 2, 4, 6, 8], np.int64)),
                        flags=g.GNF4_CHECK, R=8)
    torch.cuda.synchronize()
    assert ok.shape == (8, 64)


def test_host_pointers_are_refused():
    import bit_grouped_moe_gnf4_b200 as g
    Wd, Sd, _, _ = build_stack("nf4", 2, 64, 128, seed=1)
    x_host = torch.zeros((4, 128), dtype=torch.bfloat16)
    with pytest.raises(g.Gnf4Error) as ei:
        g.grouped_gemm("nf4", x_host, Wd, Sd, to_dev(np.array([0, 2, 4], np.int64)), R=4)
    assert ei.value.status == 1


def test_bounded_wait_abort_path_reports_and_recovers():
    """GNF4_TEST_STALL: the decode band issues no weight copy, so every wait for a stage
    gives up after a short limit; the kernel records it, skips the math and drains
    nothing (nothing was issued). gnf4_device_status reports it once, and the next call
    on the same context returns correct results."""
    import bit_grouped_moe_gnf4_b200 as g
    E, k, T, K, N = 4, 2, 8, 256, 128
    Wd, Sd, Wh, Sh = build_stack("nf4", E, N, K)
    b = synth.make_routed_batch(0, T, E, k)
    x = synth.activations_bf16(0, T, K)
    args = dict(row_token=to_dev(b.row_token), row_weight=to_dev(b.row_weight), row_dest=to_dev(b.row_dest))
    for fused in (False, True):
        fn = g.grouped_gemm_swiglu if fused else g.grouped_gemm
        fn("nf4", bf16_dev(x), Wd, Sd, to_dev(b.offsets), T_out=T * k, flags=g.GNF4_TEST_STALL, **args)
        with pytest.raises(g.Gnf4Error) as ei:
            g.device_status()
        assert ei.value.status == 5
        g.device_status()                                # the record was cleared
    out = run_gemm("nf4", x, Wd, Sd, b.offsets, b.row_token, b.row_weight, b.row_dest, T_out=T * k)
    ref = O.grouped_rows_f64("nf4", x, Wh, Sh, b.offsets, b.row_token, b.row_weight, K, np.arange(b.R))
    check_rows(out[b.row_dest], ref, "after the stall test")


def test_default_mode_row_count_invariance():
    """A token's rows keep their bits whether it is routed alone or inside 16-, 17- and
    160-token calls with softmax top-8 routing, in the default band choice: every group
    of these calls has at most 64 rows, so every row runs in the decode band, whose fp32
    summation order depends on K alone."""
    import bit_grouped_moe_gnf4_b200 as g
    wl = WORKLOADS["olmoe_decode_nf4"]
    gu = wl.projections[0]
    E, k = wl.E, 8
    ids, w = G.route_softmax_topk(11, 160, E, k)
    x_all = synth.activations_bf16(12, 160, gu.K)
    Wd, Sd, _, _ = build_stack("nf4", E, gu.N, gu.K, seed=0, oracle_experts=[int(e) for e in ids[0]])
    rows0 = []
    for T in (1, 16, 17, 160):
        off, tok, wt, dst = G.routing_metadata(ids[:T].astype(np.int32), w[:T], E)
        assert np.diff(off).max() <= 64
        out = g.grouped_gemm("nf4", bf16_dev(x_all[:T]), Wd, Sd, to_dev(off), row_token=to_dev(tok),
                             row_dest=to_dev(dst), T_out=T * k)
        rows0.append(bf16_host_bits(out)[:k])             # token 0's k slots
    g.device_status()
    for r in rows0[1:]:
        assert np.array_equal(r, rows0[0])


@pytest.mark.parametrize("E", [1600, 2048])
@pytest.mark.parametrize("fmt", ["nf4", "mxfp4"])
def test_many_experts_decode_band(E, fmt):
    """The most experts a call allows (2048) and a count in between: the decode band's
    per-expert tables then take most of its shared memory, and the host shrinks the routing
    table and, past a point, the ring stages (scale boxes or not) to make room; every row
    against the oracle."""
    N, K = 64, 512
    counts = np.zeros(E, np.int64)
    rng = np.random.default_rng(E)
    active = np.sort(rng.choice(E, 24, replace=False))
    counts[active] = rng.integers(1, 12, len(active))
    counts[E - 1] = 3                                   # the last expert too
    active = np.nonzero(counts)[0]
    Wd, Sd, Wh, Sh = build_stack(fmt, E, N, K, seed=E + 1, oracle_experts=active)
    b = G.explicit_batch(counts, seed=E + 2)
    x = synth.activations_bf16(E + 3, b.T, K)
    out = run_gemm(fmt, x, Wd, Sd, b.offsets, b.row_token, b.row_weight, b.row_dest, flags=BANDS["decode"])
    ref = O.grouped_rows_f64(fmt, x, Wh, Sh, b.offsets, b.row_token, b.row_weight, K, np.arange(b.R))
    check_rows(out[b.row_dest], ref, f"{E} experts {fmt}")
