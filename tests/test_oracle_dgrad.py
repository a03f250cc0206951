"""Pins for the oracle's input gradient of the grouped GEMM (CPU only).

- A scalar brute force that decodes each weight straight from the bytes.
- The adjoint identity sum_r <dx[r], x[r]> = sum_r <g[src(r)], y(r)> against the
  forward oracle, which has its own pins. It catches a transposed operand, a wrong
  expert or row index, or a dropped routing weight.
- One-hot gradients read out one dequantized weight row.
- Torch autograd of the forward product in fp64 (a library routine).
- Empty experts and the empty call.
"""
import math

import numpy as np
import pytest
import torch

import synth
from oracle import dgrad as D
from oracle import gnf4_oracle as O
from synth import generators as G


def _stack(fmt, E, N, K, seed=0):
    q = O.quantize_nf4 if fmt == "nf4" else O.quantize_mxfp4
    Ws, Ss = zip(*(q(G.expert_weights(seed, e, N, K)) for e in range(E)))
    return np.stack(Ws), np.stack(Ss)


def _decode_one(fmt, W, S, e, n, k):
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
    E, N, K = 3, 48, 128
    W, S = _stack(fmt, E, N, K, seed=1)
    counts = [2, 0, 3]
    b = G.explicit_batch(counts, seed=2)
    g = synth.activations_bf16(3, b.R, N, tag="y")
    src = np.random.default_rng(4).permutation(b.R).astype(np.int32)
    got = D.dgrad(fmt, g, W, S, b.offsets, row_src=src, row_weight=b.row_weight)
    gf = O.bf16_to_f64(g)
    for r in range(b.R):
        e = next(i for i in range(E) if b.offsets[i] <= r < b.offsets[i + 1])
        for k in range(0, K, 5):
            v = math.fsum(gf[src[r], n] * _decode_one(fmt, W, S, e, n, k) for n in range(N))
            v *= float(b.row_weight[r])
            assert got[r, k] == O.bf16_bits(np.array([v]))[0], (r, k)


@pytest.mark.parametrize("fmt", ["nf4", "mxfp4"])
def test_adjoint_identity_with_the_forward(fmt):
    E, N, K = 5, 64, 192
    W, S = _stack(fmt, E, N, K, seed=5)
    b = G.explicit_batch([4, 1, 0, 7, 3], seed=6)
    R = b.R
    x = synth.activations_bf16(7, R, K)                       # routed rows, read in order
    g = synth.activations_bf16(8, R, N, tag="y")
    src = np.random.default_rng(9).permutation(R).astype(np.int32)
    # forward rows y(r) = w(r) x[r] What[e(r)].T, their gradient rows g[src(r)]
    y = O.grouped_rows_f64(fmt, x, W, S, b.offsets, None, b.row_weight, K, np.arange(R))
    dx = D.dgrad_rows_f64(fmt, g, W, S, b.offsets, src, b.row_weight, np.arange(R))
    lhs = float(np.sum(dx * O.bf16_to_f64(x)))
    rhs = float(np.sum(O.bf16_to_f64(g)[src] * y))
    assert lhs == pytest.approx(rhs, rel=1e-12, abs=1e-12)
    # a plausible slip (no permutation of the gradient rows) breaks it
    dx_wrong = D.dgrad_rows_f64(fmt, g, W, S, b.offsets, None, b.row_weight, np.arange(R))
    assert float(np.sum(dx_wrong * O.bf16_to_f64(x))) != pytest.approx(rhs, rel=1e-6)


@pytest.mark.parametrize("fmt", ["nf4", "mxfp4"])
def test_one_hot_gradient_reads_a_weight_row(fmt):
    E, N, K = 2, 32, 128
    W, S = _stack(fmt, E, N, K, seed=10)
    offsets = np.array([0, N, 2 * N], np.int64)               # N rows per expert
    g = np.zeros((2 * N, N), np.uint16)
    for r in range(2 * N):
        g[r, r % N] = 0x3F80                                  # bf16 1.0 at column n = r mod N
    got = D.dgrad(fmt, g, W, S, offsets)
    for e in range(E):
        What = O.decode_expert(fmt, W, S, e, K)
        # values, not bits: e2m1 code 8 is -0, and 1 * (-0) + 0 * (...) sums to +0
        assert np.array_equal(O.bf16_to_f64(got[e * N:(e + 1) * N]), O.bf16_to_f64(O.bf16_bits(What)))


def test_matches_torch_autograd_of_the_forward():
    fmt, E, N, K = "nf4", 3, 64, 128
    W, S = _stack(fmt, E, N, K, seed=11)
    b = G.explicit_batch([5, 2, 6], seed=12)
    x = torch.tensor(O.bf16_to_f64(synth.activations_bf16(13, b.R, K)), requires_grad=True)
    g = synth.activations_bf16(14, b.R, N, tag="y")
    w = torch.tensor(b.row_weight.astype(np.float64))
    ys = []
    for e in range(E):
        r0, r1 = int(b.offsets[e]), int(b.offsets[e + 1])
        What = torch.tensor(O.decode_expert(fmt, W, S, e, K))
        ys.append((x[r0:r1] @ What.T) * w[r0:r1, None])
    torch.cat(ys).backward(torch.tensor(O.bf16_to_f64(g)))
    want = x.grad.numpy()
    got = D.dgrad_rows_f64(fmt, g, W, S, b.offsets, None, b.row_weight, np.arange(b.R))
    assert np.allclose(got, want, rtol=1e-12, atol=1e-14)


def test_empty_experts_and_empty_call():
    E, N, K = 4, 32, 64
    W, S = _stack("nf4", E, N, K, seed=15)
    b = G.explicit_batch([0, 3, 0, 0], seed=16)
    g = synth.activations_bf16(17, b.R, N, tag="y")
    got = D.dgrad("nf4", g, W, S, b.offsets)
    assert got.shape == (3, K)
    want = O.bf16_bits(O.bf16_to_f64(g) @ O.decode_expert("nf4", W, S, 1, K))
    assert np.array_equal(got, want)
    assert D.dgrad("nf4", g[:0], W, S, np.zeros(E + 1, np.int64)).shape == (0, K)
