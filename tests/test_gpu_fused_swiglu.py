"""gate_up grouped GEMM with the SwiGLU fused into its epilogue, through the C ABI,
against the glue oracle composed with the grouped oracle (silu(w G) * (w U) from the
exact fp64 gate and up sums, per-row bound), against the unfused chain (grouped GEMM
then the SwiGLU kernel), and for row-count invariance."""
import numpy as np
import pytest
import torch

import synth
from oracle import glue as GL
from oracle import gnf4_oracle as O
from oracle import storage as S
from synth import generators as G
from synth.workloads import WORKLOADS

from gpu_support import ROW_TOL, bf16_dev, build_stack, to_dev

pytestmark = pytest.mark.gpu


def _ref(fmt, x_f64, Wh, Sh, b, rows=None, weighted=True):
    K = Wh.shape[2] * 2
    I = Wh.shape[1] // 2
    rows = np.arange(b.R) if rows is None else rows
    gu = S.grouped_rows_f64_x(fmt, x_f64, Wh, Sh, b.offsets, b.row_token,
                              b.row_weight if weighted else None, K, rows)
    with np.errstate(over="ignore", invalid="ignore"):
        return GL.silu_f64(gu[:, :I]) * gu[:, I:]


def _f64(out):
    bits = out.view(torch.int16).cpu().numpy().view(np.uint16)
    return S.f16_to_f64(bits) if out.dtype == torch.float16 else O.bf16_to_f64(bits)


def _check(got, ref, what):
    assert np.isfinite(got).all(), what
    scale = np.abs(ref).max(axis=1)
    err = np.abs(got - ref).max(axis=1)
    assert np.all(err[scale == 0] == 0), what
    nz = scale > 0
    worst = float((err[nz] / scale[nz]).max()) if nz.any() else 0.0
    assert worst <= ROW_TOL, f"{what}: worst row error {worst:.3e}"
    return worst


@pytest.mark.parametrize("fmt", ["nf4", "mxfp4"])
def test_fused_swiglu_every_element(fmt):
    """I = 208 (a short last unit of 16 gate rows), groups of 0..150 rows (several passes),
    routing weights and a scatter."""
    import bit_grouped_moe_gnf4_b200 as g
    E, I, K = 7, 208, 640
    counts = [1, 0, 150, 9, 33, 0, 70]
    Wd, Sd, Wh, Sh = build_stack(fmt, E, 2 * I, K, seed=21)
    b = G.explicit_batch(counts, seed=22)
    xb = synth.activations_bf16(23, b.T, K)
    x = bf16_dev(xb)
    out = g.grouped_gemm_swiglu(fmt, x, Wd, Sd, to_dev(b.offsets), row_token=to_dev(b.row_token),
                                row_weight=to_dev(b.row_weight), row_dest=to_dev(b.row_dest), T_out=b.R)
    g.device_status()
    assert out.shape == (b.R, I)
    got = _f64(out)[b.row_dest]
    _check(got, _ref(fmt, O.bf16_to_f64(xb), Wh, Sh, b), f"fused {fmt}")
    # the unfused chain: grouped GEMM (bf16 gate_up rows) then the SwiGLU kernel
    h = g.grouped_gemm(fmt, x, Wd, Sd, to_dev(b.offsets), row_token=to_dev(b.row_token),
                       row_weight=to_dev(b.row_weight), row_dest=to_dev(b.row_dest), T_out=b.R)
    chain = _f64(g.swiglu(h))[b.row_dest]
    _check(got, chain, f"fused vs chain {fmt}")


def test_fused_swiglu_fp16_x_bf16_absmax():
    import bit_grouped_moe_gnf4_b200 as g
    E, I, K = 5, 256, 512
    W = np.zeros((E, 2 * I, K // 2), np.uint8)
    B = np.zeros((E, 2 * I, K // 64), np.uint16)
    for e in range(E):
        w = G.expert_weights(4, e, 2 * I, K)
        w = (w.view(np.uint32) & np.uint32(0xFFFF0000)).view(np.float32)
        p, a = O.quantize_nf4(w)
        W[e], B[e] = p, S.absmax_to_bf16(a)
    b = G.explicit_batch([3, 17, 0, 1, 40], seed=24)
    xh = S.f16_bits(np.random.default_rng(25).normal(0, 1, (b.T, K)))
    x = torch.from_numpy(xh.view(np.int16)).cuda().view(torch.float16)
    out = g.grouped_gemm_swiglu("nf4", x, to_dev(W), torch.from_numpy(B.view(np.int16)).cuda().view(torch.bfloat16),
                                to_dev(b.offsets), row_token=to_dev(b.row_token), R=b.R)
    g.device_status()
    assert out.dtype == torch.float16
    _check(_f64(out), _ref("nf4", S.f16_to_f64(xh), W, B, b, weighted=False), "fused fp16 bf16-absmax")


@pytest.mark.parametrize("T", [1, 16])
def test_fused_swiglu_olmoe_decode(T):
    """The OLMoE-shaped decode layer's gate_up (K 2048, 2I = 2048): every row."""
    import bit_grouped_moe_gnf4_b200 as g
    wl = WORKLOADS["olmoe_decode_nf4"]
    gu = wl.projections[0]
    b = synth.make_routed_batch(0, T, wl.E, 8)
    Wd, Sd, Wh, Sh = build_stack("nf4", wl.E, gu.N, gu.K, seed=0, oracle_experts=b.active_experts())
    xb = synth.activations_bf16(0, T, gu.K)
    out = g.grouped_gemm_swiglu("nf4", bf16_dev(xb), Wd, Sd, to_dev(b.offsets), row_token=to_dev(b.row_token),
                                R=b.R)
    g.device_status()
    _check(_f64(out), _ref("nf4", O.bf16_to_f64(xb), Wh, Sh, b, weighted=False), f"fused olmoe T={T}")


def test_fused_swiglu_row_count_invariance():
    import bit_grouped_moe_gnf4_b200 as g
    E, I, K = 64, 1024, 2048
    Wd, Sd, _, _ = build_stack("nf4", E, 2 * I, K, seed=0, oracle_experts=[9])
    x = bf16_dev(synth.activations_bf16(5, 160, K))
    results = []
    for m in (1, 16, 17, 160):
        offs = np.zeros(E + 1, np.int64)
        offs[10:] = m
        tok = np.arange(m, dtype=np.int32)[::-1].copy()
        out = g.grouped_gemm_swiglu("nf4", x, Wd, Sd, to_dev(offs), row_token=to_dev(tok))
        results.append(out.view(torch.int16).cpu().numpy()[m - 1])
    g.device_status()
    for r in results[1:]:
        assert np.array_equal(r, results[0])


def test_fused_swiglu_refuses_bad_shapes_and_prefill():
    import bit_grouped_moe_gnf4_b200 as g
    Wd, Sd, _, _ = build_stack("nf4", 2, 48, 128, seed=1)
    x = bf16_dev(synth.activations_bf16(1, 4, 128))
    off = to_dev(np.array([0, 2, 4], np.int64))
    with pytest.raises(g.Gnf4Error) as ei:
        g.grouped_gemm_swiglu("nf4", x, Wd, Sd, off, R=4)              # 2I = 48 is not a multiple of 32
    assert ei.value.status == 2
    Wd, Sd, _, _ = build_stack("nf4", 2, 64, 128, seed=1)
    with pytest.raises(g.Gnf4Error) as ei:
        g.grouped_gemm_swiglu("nf4", x, Wd, Sd, off, R=4, flags=g.GNF4_FORCE_PREFILL)
    assert ei.value.status == 1
