"""Pins for the oracle's grouped product (CPU only).

Brute force with plain Python loops on the tiny workload, permutation and
one-hot products whose exact answers are known, routing invariants (empty
experts, top_k = 1, expert relabelling, untouched rows), the routing-weight
epilogue and the pages' own group example.
"""
import math

import numpy as np
import pytest

import synth
from oracle import gnf4_oracle as O
from synth import generators as G


def _stack(fmt, E, N, K, seed=0, experts=None):
    q = O.quantize_nf4 if fmt == "nf4" else O.quantize_mxfp4
    Ws, Ss = [], []
    for e in range(E):
        w = G.expert_weights(seed, e, N, K)
        p, s = q(w)
        Ws.append(p)
        Ss.append(s)
    return np.stack(Ws), np.stack(Ss)


def _decode_one(fmt, W, S, e, n, k):
    """Scalar decode of one weight straight from the bytes (independent of the
    vectorised decoder)."""
    byte = int(W[e, n, k // 2])
    if fmt == "nf4":
        code = (byte >> 4) if k % 2 == 0 else (byte & 15)
        return float(O.NF4_CODEBOOK[code]) * float(S[e, n, k // 64])
    code = (byte & 15) if k % 2 == 0 else (byte >> 4)
    sign = -1.0 if code & 8 else 1.0
    ex, m = (code >> 1) & 3, code & 1
    mag = m * 0.5 if ex == 0 else 2.0 ** (ex - 1) * (1 + m / 2)
    return sign * mag * 2.0 ** (int(S[e, n, k // 32]) - 127)


@pytest.mark.parametrize("fmt", ["nf4", "mxfp4"])
def test_brute_force_tiny(fmt):
    E, k, T, K, N = 4, 2, 8, 256, 128
    W, S = _stack(fmt, E, N, K)
    b = synth.make_routed_batch(0, T, E, k)
    x = synth.activations_bf16(0, T, K)
    xf = G.f32_from_bf16_bits(x).astype(np.float64)
    out = O.grouped_gemm(fmt, x, W, S, b.offsets, b.row_token, b.row_weight, b.row_dest,
                         T_out=T * k)
    R = b.R
    for r in range(R):
        e = next(i for i in range(E) if b.offsets[i] <= r < b.offsets[i + 1])
        t = int(b.row_token[r])
        for n in range(0, N, 7):
            terms = [xf[t, kk] * _decode_one(fmt, W, S, e, n, kk) for kk in range(K)]
            v = math.fsum(terms) * float(b.row_weight[r])
            want = O.bf16_bits(np.array([v]))[0]
            assert out[b.row_dest[r], n] == want, (r, n)


def test_brute_force_fp32_orders_stay_inside_the_bound():
    """fp32 sums in two orders differ from the exact result by far less than the
    per-row bound 2e-2 * max|row| the kernels are held to."""
    E, k, T, K, N = 4, 2, 8, 256, 128
    W, S = _stack("nf4", E, N, K)
    b = synth.make_routed_batch(0, T, E, k)
    x = synth.activations_bf16(0, T, K)
    ref = O.grouped_rows_f64("nf4", x, W, S, b.offsets, b.row_token, None, K, np.arange(b.R))
    xf = G.f32_from_bf16_bits(x)
    worst = 0.0
    for r in range(b.R):
        e = int(np.searchsorted(b.offsets, r, side="right") - 1)
        wd = O.dequant_nf4(W[e], S[e], K).astype(np.float32)
        prod = (xf[b.row_token[r]][None, :] * wd).astype(np.float32)
        fwd = np.zeros(N, np.float32)
        bwd = np.zeros(N, np.float32)
        for kk in range(K):
            fwd += prod[:, kk]
            bwd += prod[:, K - 1 - kk]
        scale = np.abs(ref[r]).max()
        worst = max(worst, np.abs(fwd - ref[r]).max() / scale, np.abs(bwd - ref[r]).max() / scale)
    assert worst < 1e-4


@pytest.mark.parametrize("fmt", ["nf4", "mxfp4"])
def test_permutation_weights_give_permuted_x_bitwise(fmt):
    N = K = 128
    rng = np.random.default_rng(1)
    perm = rng.permutation(K)
    w = np.zeros((N, K), np.float32)
    w[np.arange(N), perm] = 1.0                  # W[n, k] = [k == perm[n]]
    q = O.quantize_nf4 if fmt == "nf4" else O.quantize_mxfp4
    p, s = q(w)
    W, S = p[None], s[None]
    T = 5
    x = synth.activations_bf16(2, T, K)
    offsets = np.array([0, T], np.int64)
    out = O.grouped_gemm(fmt, x, W, S, offsets)
    assert np.array_equal(out, x[:, perm])       # out[r, n] = x[r, perm[n]]


@pytest.mark.parametrize("fmt", ["nf4", "mxfp4"])
def test_one_hot_x_reads_one_weight_column(fmt):
    E, N, K = 2, 64, 128
    W, S = _stack(fmt, E, N, K, seed=5)
    kk = 77
    x = np.zeros((1, K), np.uint16)
    x[0, kk] = 0x3F80                            # bf16 1.0
    offsets = np.array([0, 0, 1], np.int64)      # the single row goes to expert 1
    out = O.grouped_gemm(fmt, x, W, S, offsets)
    col = np.array([_decode_one(fmt, W, S, 1, n, kk) for n in range(N)])
    # equal as values: a -0 weight (MXFP4 code 8) sums to +0 with the zero terms
    assert np.array_equal(O.bf16_to_f64(out[0]), O.round_to_bf16(col))


def test_empty_experts_and_untouched_rows():
    E, N, K = 6, 64, 128
    W, S = _stack("nf4", E, N, K, seed=2)
    counts = [0, 3, 0, 0, 2, 0]
    b = G.explicit_batch(counts, seed=4)
    x = synth.activations_bf16(3, b.T, K)
    T_out = 9
    dest = np.array([7, 1, 4, 0, 8], np.int32)
    init = np.full((T_out, N), 0x7FC1, np.uint16)          # NaN sentinel
    out = O.grouped_gemm("nf4", x, W, S, b.offsets, b.row_token, b.row_weight, dest,
                         T_out=T_out, out_init=init)
    untouched = sorted(set(range(T_out)) - set(dest.tolist()))
    assert np.all(out[untouched] == 0x7FC1)
    # each written row equals the single-expert product of its own expert
    for r, e in zip(range(5), [1, 1, 1, 4, 4]):
        one = O.grouped_gemm("nf4", x[b.row_token[r]][None], W[e:e + 1], S[e:e + 1],
                             np.array([0, 1], np.int64), row_weight=b.row_weight[r:r + 1])
        assert np.array_equal(out[dest[r]], one[0])


def test_top1_routing_is_per_token_product():
    E, N, K, T = 8, 64, 128, 12
    W, S = _stack("mxfp4", E, N, K, seed=6)
    b = synth.make_routed_batch(1, T, E, 1)
    x = synth.activations_bf16(4, T, K)
    out = O.grouped_gemm("mxfp4", x, W, S, b.offsets, b.row_token, None, b.row_dest, T_out=T)
    for t in range(T):
        e = int(b.ids[t, 0])
        ref = G.f32_from_bf16_bits(x[t]).astype(np.float64) @ O.dequant_mxfp4(W[e], S[e], K).T
        assert np.array_equal(out[t], O.bf16_bits(ref))


def test_routing_weight_two_doubles_exactly():
    E, N, K, T = 4, 64, 128, 6
    W, S = _stack("nf4", E, N, K, seed=7)
    b = synth.make_routed_batch(2, T, E, 2)
    x = synth.activations_bf16(5, T, K)
    one = O.grouped_gemm("nf4", x, W, S, b.offsets, b.row_token)
    two = O.grouped_gemm("nf4", x, W, S, b.offsets, b.row_token,
                         row_weight=np.full(b.R, 2.0, np.float32))
    assert np.array_equal(O.bf16_to_f64(two), 2.0 * O.bf16_to_f64(one))


def test_expert_relabelling_leaves_bytes_unchanged():
    E, N, K, T = 8, 64, 128, 10
    W, S = _stack("nf4", E, N, K, seed=8)
    b = synth.make_routed_batch(3, T, E, 3)
    x = synth.activations_bf16(6, T, K)
    out = O.grouped_gemm("nf4", x, W, S, b.offsets, b.row_token, b.row_weight, b.row_dest,
                         T_out=T * 3)
    perm = np.random.default_rng(9).permutation(E)   # new id of old expert e is perm[e]
    W2 = np.empty_like(W)
    S2 = np.empty_like(S)
    W2[perm] = W
    S2[perm] = S
    ids2 = perm[b.ids]
    off2, tok2, rw2, dst2 = G.routing_metadata(ids2.astype(np.int32), b.weights, E)
    out2 = O.grouped_gemm("nf4", x, W2, S2, off2, tok2, rw2, dst2, T_out=T * 3)
    assert np.array_equal(out, out2)


def test_pages_group_example_mapping():
    """The pages' example: 8 experts, groups of 3, 1, 4 rows for experts 5, 0, 2,
    output in the group order of a_cat. The offsets/row_token/row_dest form of
    the same call reproduces the per-group product in a_cat order."""
    import json
    import os
    g = json.load(open(os.path.join(os.path.dirname(__file__), "golden",
                                    "pages_printed_values.json")))["stack_fixture_shapes"]
    E, N, K = g["E"], 64, g["K"]
    W, S = _stack("nf4", E, N, K, seed=10)
    T = sum(g["sizes"])
    a_cat = synth.activations_bf16(7, T, K)
    off, tok, dst = G.groups_to_routing(g["sizes"], g["expert_ids"], E)
    out = O.grouped_gemm("nf4", a_cat, W, S, off, tok, None, dst, T_out=T)
    row = 0
    for m, e in zip(g["sizes"], g["expert_ids"]):
        ref = G.f32_from_bf16_bits(a_cat[row:row + m]).astype(np.float64) @ \
            O.dequant_nf4(W[e], S[e], K).T
        assert np.array_equal(out[row:row + m], O.bf16_bits(ref))
        row += m
