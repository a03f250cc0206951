"""Storage variants on the GPU, through the C ABI: NF4 absmax stored as bf16 and fp16
activations, in both bands, against the storage oracle (per-row bound, fp16 or bf16
output), and the lossless claim at kernel level: for a bf16 source the bf16-absmax
call returns the fp32-absmax call's bits."""
import numpy as np
import pytest
import torch

import synth
from oracle import gnf4_oracle as O
from oracle import storage as S
from synth import generators as G
from synth.workloads import WORKLOADS

from gpu_support import ROW_TOL, bf16_dev, bf16_host_bits, build_stack, to_dev

pytestmark = pytest.mark.gpu

BANDS = {"auto": 0, "decode": 0x2, "prefill": 0x4}


def _bf16_source_stack(E, N, K, seed=0, tag="w"):
    """NF4 stack quantized (by the oracle) from weights that are bf16 values: host
    packed bytes, fp32 absmax and the same absmax as bf16 bits (exact)."""
    W = np.zeros((E, N, K // 2), np.uint8)
    A = np.zeros((E, N, K // 64), np.float32)
    for e in range(E):
        w = G.expert_weights(seed, e, N, K, tag=tag)
        w = (w.view(np.uint32) & np.uint32(0xFFFF0000)).view(np.float32)
        W[e], A[e] = O.quantize_nf4(w)
    return W, A, S.absmax_to_bf16(A)


def _x(seed, T, K, f16):
    if f16:
        bits = S.f16_bits(np.random.default_rng(seed).normal(0, 1, (T, K)))
        return bits, S.f16_to_f64(bits), torch.from_numpy(bits.view(np.int16)).cuda().view(torch.float16)
    bits = synth.activations_bf16(seed, T, K)
    return bits, O.bf16_to_f64(bits), bf16_dev(bits)


def _out_f64(out):
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


@pytest.mark.parametrize("band", list(BANDS))
@pytest.mark.parametrize("absmax", ["f32", "bf16"])
@pytest.mark.parametrize("f16", [False, True])
def test_nf4_storage_variants_every_element(band, absmax, f16):
    import bit_grouped_moe_gnf4_b200 as g
    E, N, K = 7, 400, 640
    counts = [1, 0, 150, 9, 33, 0, 70]
    Wh, Ah, Bh = _bf16_source_stack(E, N, K, seed=3)
    Sh = Bh if absmax == "bf16" else Ah
    Sd = torch.from_numpy(Bh.view(np.int16)).cuda().view(torch.bfloat16) if absmax == "bf16" else to_dev(Ah)
    b = G.explicit_batch(counts, seed=5)
    _, xv, xd = _x(9, b.T, K, f16)
    out = torch.empty((b.R, N), dtype=xd.dtype, device="cuda")
    g.grouped_gemm("nf4", xd, to_dev(Wh), Sd, to_dev(b.offsets), row_token=to_dev(b.row_token),
                   row_weight=to_dev(b.row_weight), row_dest=to_dev(b.row_dest), out=out, flags=BANDS[band])
    g.device_status()
    ref = S.grouped_rows_f64_x("nf4", xv, Wh, Sh, b.offsets, b.row_token, b.row_weight, K, np.arange(b.R))
    _check(_out_f64(out)[b.row_dest], ref, f"nf4 {absmax} f16={f16} {band}")


@pytest.mark.parametrize("band", list(BANDS))
def test_mxfp4_fp16_activations_every_element(band):
    import bit_grouped_moe_gnf4_b200 as g
    E, N, K = 7, 400, 640
    counts = [1, 0, 150, 9, 33, 0, 70]
    Wd, Sd, Wh, Sh = build_stack("mxfp4", E, N, K, seed=4)
    b = G.explicit_batch(counts, seed=6)
    _, xv, xd = _x(10, b.T, K, True)
    out = g.grouped_gemm("mxfp4", xd, Wd, Sd, to_dev(b.offsets), row_token=to_dev(b.row_token),
                         row_weight=to_dev(b.row_weight), row_dest=to_dev(b.row_dest), flags=BANDS[band])
    g.device_status()
    assert out.dtype == torch.float16
    ref = S.grouped_rows_f64_x("mxfp4", xv, Wh, Sh, b.offsets, b.row_token, b.row_weight, K, np.arange(b.R))
    _check(_out_f64(out)[b.row_dest], ref, f"mxfp4 f16 {band}")


@pytest.mark.parametrize("band", list(BANDS))
@pytest.mark.parametrize("f16", [False, True])
def test_bf16_absmax_is_lossless_on_the_gpu(band, f16):
    """A bf16 source: the bf16-absmax call returns exactly the fp32-absmax call's bits."""
    import bit_grouped_moe_gnf4_b200 as g
    E, N, K = 16, 512, 1024
    Wh, Ah, Bh = _bf16_source_stack(E, N, K, seed=8)
    b = synth.make_routed_batch(3, 96, E, 4)
    _, _, xd = _x(11, b.T, K, f16)
    Wd, off, tok = to_dev(Wh), to_dev(b.offsets), to_dev(b.row_token)
    o32 = g.grouped_gemm("nf4", xd, Wd, to_dev(Ah), off, row_token=tok, flags=BANDS[band])
    o16 = g.grouped_gemm("nf4", xd, Wd, torch.from_numpy(Bh.view(np.int16)).cuda().view(torch.bfloat16), off,
                         row_token=tok, flags=BANDS[band])
    g.device_status()
    assert torch.equal(o32.view(torch.int16), o16.view(torch.int16))


def test_absmax_cast_matches_the_oracle_and_refuses_fp32_sources():
    import bit_grouped_moe_gnf4_b200 as g
    _, Ah, Bh = _bf16_source_stack(4, 256, 512, seed=12)
    got = g.absmax_to_bf16(to_dev(Ah))
    assert np.array_equal(got.view(torch.int16).cpu().numpy().view(np.uint16), Bh)
    _, a32 = O.quantize_nf4(G.expert_weights(0, 0, 64, 256))
    with pytest.raises(g.Gnf4Error) as ei:
        g.absmax_to_bf16(to_dev(a32))
    assert ei.value.status == 1
    # the library is still usable after a refusal
    again = g.absmax_to_bf16(to_dev(Ah))
    torch.cuda.synchronize()
    assert torch.equal(again.view(torch.int16), got.view(torch.int16))


@pytest.mark.parametrize("T", [1, 16])
def test_olmoe_decode_bf16_absmax_fp16_x(T):
    """The OLMoE-shaped decode step's gate_up on a bf16 source with bf16 absmax and fp16
    activations: every output row of the call against the oracle."""
    import bit_grouped_moe_gnf4_b200 as g
    wl = WORKLOADS["olmoe_decode_nf4"]
    gu = wl.projections[0]
    b = synth.make_routed_batch(0, T, wl.E, 8)
    experts = [int(e) for e in b.active_experts()]
    Wh = np.zeros((wl.E, gu.N, gu.K // 2), np.uint8)
    Bh = np.zeros((wl.E, gu.N, gu.K // 64), np.uint16)
    for e in experts:
        w = G.expert_weights(0, e, gu.N, gu.K)
        w = (w.view(np.uint32) & np.uint32(0xFFFF0000)).view(np.float32)
        p, a = O.quantize_nf4(w)
        Wh[e], Bh[e] = p, S.absmax_to_bf16(a)
    _, xv, xd = _x(13, T, gu.K, True)
    out = g.grouped_gemm("nf4", xd, to_dev(Wh), torch.from_numpy(Bh.view(np.int16)).cuda().view(torch.bfloat16),
                         to_dev(b.offsets), row_token=to_dev(b.row_token), R=b.R)
    g.device_status()
    ref = S.grouped_rows_f64_x("nf4", xv, Wh, Bh, b.offsets, b.row_token, None, gu.K, np.arange(b.R))
    _check(_out_f64(out), ref, f"olmoe T={T} bf16 absmax fp16")


def test_storage_type_checks_on_the_host():
    import bit_grouped_moe_gnf4_b200 as g
    from bit_grouped_moe_gnf4_b200._lib import lib
    Wd, Sd, _, _ = build_stack("nf4", 2, 64, 128, seed=1)
    x = bf16_dev(synth.activations_bf16(1, 4, 128))
    off = to_dev(np.array([0, 2, 4], np.int64))
    out = torch.empty((4, 64), dtype=torch.bfloat16, device="cuda")
    BF16, F16, F32 = g.GNF4_DTYPE_BF16, g.GNF4_DTYPE_F16, g.GNF4_DTYPE_F32

    def call(xdt, sdt, soff=0):
        return lib.gnf4_grouped_gemm_nf4_ex(x.data_ptr(), xdt, Wd.data_ptr(), Sd.data_ptr() + soff, sdt,
                                            off.data_ptr(), None, None, None, 2, 64, 128, 4, 4, 4,
                                            out.data_ptr(), 0, None)
    assert call(7, F32) == 1                              # unknown activation type
    assert call(F32, F32) == 1                            # fp32 activations are not a variant
    assert call(BF16, F16) == 1                           # NF4 absmax is fp32 or bf16
    assert call(BF16, BF16) == 0                          # bf16 absmax reading fp32 bytes: legal, meaningless
    g.device_status()
    assert call(BF16, BF16, soff=1) == 3                  # bf16 absmax off its 2-byte boundary
    assert call(BF16, F32, soff=2) == 3                   # fp32 absmax off its 4-byte boundary
