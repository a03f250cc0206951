"""Helpers for the GPU parity tests: build packed stacks with the oracle's own
quantizer on the host, upload them, run the CUDA path through the C ABI, and
compare with the oracle row by row.

The tolerance is the stated one: per output row, max_n |out - ref| <=
2e-2 * max_n |ref| with ref the oracle's fp64 value; a row whose reference is
all zero must come out exactly zero. Packed bytes and scales must match bit for
bit.
"""
from __future__ import annotations

import numpy as np
import torch

import synth
from oracle import gnf4_oracle as O
from synth import generators as G

ROW_TOL = 2e-2


def oracle_quantize(fmt, w):
    return O.quantize_nf4(w) if fmt == "nf4" else O.quantize_mxfp4(w)


def build_stack(fmt, E, N, K, seed=0, oracle_experts=None, tag="w", device="cuda"):
    """Packed stack on the device. Experts in ``oracle_experts`` (all if None) are
    quantized by the oracle on the host; the others get random bytes and scales
    (never compared). Returns (W_dev, S_dev, W_host, S_host) with host copies
    holding the oracle-quantized experts (zeros elsewhere)."""
    sdiv = 64 if fmt == "nf4" else 32
    Wh = np.zeros((E, N, K // 2), np.uint8)
    Sh = np.zeros((E, N, K // sdiv), np.float32 if fmt == "nf4" else np.uint8)
    experts = range(E) if oracle_experts is None else oracle_experts
    chosen = set(int(e) for e in experts)
    for e in range(E):
        if e in chosen:
            p, s = oracle_quantize(fmt, G.expert_weights(seed, e, N, K, tag=tag))
            Wh[e], Sh[e] = p, s
    Wd = torch.from_numpy(Wh).to(device)
    Sd = torch.from_numpy(Sh).to(device)
    others = [e for e in range(E) if e not in chosen]
    if others:
        # filler for experts no compared row reads (drawn on the device, seeded)
        gen = torch.Generator(device=device)
        gen.manual_seed(int(seed) * 7919 + 13)
        for e in others:
            Wd[e] = torch.randint(0, 256, (N, K // 2), dtype=torch.uint8, device=device, generator=gen)
            if fmt == "nf4":
                Sd[e] = torch.rand((N, K // sdiv), device=device, generator=gen) * 0.05
            else:
                Sd[e] = torch.randint(110, 125, (N, K // sdiv), dtype=torch.uint8, device=device,
                                      generator=gen)
    return Wd, Sd, Wh, Sh


def to_dev(a, device="cuda"):
    return None if a is None else torch.from_numpy(np.ascontiguousarray(a)).to(device)


def bf16_dev(bits, device="cuda"):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).to(device).view(torch.bfloat16)


def bf16_host_bits(t):
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


def check_rows(out_bits, ref_f64, what=""):
    """Per-row bound on bf16 output bits against fp64 references (rows aligned)."""
    got = O.bf16_to_f64(out_bits)
    assert got.shape == ref_f64.shape, (got.shape, ref_f64.shape)
    assert np.isfinite(got).all(), f"{what}: non-finite output"
    scale = np.abs(ref_f64).max(axis=1)
    err = np.abs(got - ref_f64).max(axis=1)
    zero = scale == 0
    assert np.all(err[zero] == 0), f"{what}: rows with all-zero reference are not zero"
    nz = ~zero
    rel = np.zeros_like(err)
    rel[nz] = err[nz] / scale[nz]
    worst = float(rel.max()) if rel.size else 0.0
    assert worst <= ROW_TOL, f"{what}: worst row error {worst:.3e} > {ROW_TOL}"
    return worst


GROUP_FROB_TOL = 1e-2


def check_group_frobenius(out_bits, ref_f64, offsets, what=""):
    """The pages' own bound beside the per-row one: per expert group, relative Frobenius
    error ||out - ref||_F / ||ref||_F <= 1e-2 (rows aligned with the routed order)."""
    got = O.bf16_to_f64(out_bits)
    worst = 0.0
    offsets = np.asarray(offsets)
    for e in range(len(offsets) - 1):
        r0, r1 = int(offsets[e]), int(offsets[e + 1])
        if r1 <= r0:
            continue
        den = np.linalg.norm(ref_f64[r0:r1])
        if den == 0:
            continue
        worst = max(worst, float(np.linalg.norm(got[r0:r1] - ref_f64[r0:r1]) / den))
    assert worst <= GROUP_FROB_TOL, f"{what}: group relative Frobenius error {worst:.3e} > {GROUP_FROB_TOL}"
    return worst


def run_gemm(fmt, x_bits, Wd, Sd, offsets, row_token=None, row_weight=None, row_dest=None,
             T_out=None, flags=0, out_init_bits=None):
    import bit_grouped_moe_gnf4_b200 as g
    x = bf16_dev(x_bits)
    R = int(offsets[-1])
    if out_init_bits is not None:
        out = bf16_dev(out_init_bits)
    else:
        out = torch.empty((R if T_out is None else T_out, Wd.shape[1]), dtype=torch.bfloat16, device="cuda")
    g.grouped_gemm(fmt, x, Wd, Sd, to_dev(np.asarray(offsets, np.int64)), row_token=to_dev(row_token),
                   row_weight=to_dev(row_weight), row_dest=to_dev(row_dest), out=out, flags=flags, R=R)
    g.device_status()          # synchronises; raises if a kernel gave up waiting on a barrier
    return bf16_host_bits(out)


def sample_rows(offsets, max_rows=64, max_experts=6, seed=0):
    """A sample of routed rows touching at most ``max_experts`` experts, including
    the first and last row of each chosen group."""
    offsets = np.asarray(offsets)
    counts = np.diff(offsets)
    active = np.nonzero(counts > 0)[0]
    rng = np.random.default_rng(seed)
    big = active[np.argsort(-counts[active], kind="stable")][:2]
    rest = np.setdiff1d(active, big)
    pick = list(big) + list(rng.choice(rest, size=min(len(rest), max_experts - len(big)), replace=False))
    rows = []
    per = max(2, max_rows // max(1, len(pick)))
    for e in pick:
        r0, r1 = int(offsets[e]), int(offsets[e + 1])
        rr = {r0, r1 - 1}
        if r1 - r0 > 2:
            rr |= set(rng.choice(np.arange(r0, r1), size=min(per, r1 - r0), replace=False).tolist())
        rows.extend(sorted(rr))
    return np.array(sorted(set(rows)), np.int64), sorted(int(e) for e in pick)
