"""The decode band's two ways of bringing in the block scales give the same bits.

When a row of scales is TMA-able (a pitch of a multiple of 16 bytes and a 16-byte-aligned
array) the scales of a chunk ride in the ring stage with the packed weights; otherwise each
lane loads its rows' scales itself, a chunk ahead. The same call is run twice, once on an
aligned scale array and once on the same values at an offset that the C ABI allows (4 bytes
for fp32 absmax, 2 for bf16, 1 for e8m0) but TMA does not, and the outputs must match bit
for bit; the aligned run is also checked against the oracle (per-row bound)."""
import numpy as np
import pytest
import torch

from oracle import gnf4_oracle as O
from oracle import storage as S
from synth import activations_bf16
from synth import generators as G

from gpu_support import ROW_TOL, bf16_dev, build_stack, to_dev

pytestmark = pytest.mark.gpu

FORCE_DECODE = 0x2


def _offset_copy(t, elems):
    """The same values in a fresh buffer, starting `elems` elements past its start."""
    flat = t.reshape(-1)
    buf = torch.zeros(flat.numel() + elems, dtype=t.dtype, device=t.device)
    buf[elems:] = flat
    v = buf[elems:].view(t.shape)
    assert v.data_ptr() % 16 != 0
    return v


@pytest.mark.parametrize("case", ["nf4_f32", "nf4_bf16", "mxfp4"])
def test_scales_in_stage_match_scales_by_lanes(case):
    import bit_grouped_moe_gnf4_b200 as g
    fmt = "mxfp4" if case == "mxfp4" else "nf4"
    E, N, K = 6, 192, 1024                      # scale rows of 64, 32 and 32 bytes
    Wd, Sd, Wh, Sh = build_stack(fmt, E, N, K, seed=11)
    if case == "nf4_bf16":
        # absmax stored as bf16: the fp32 absmax cut to bf16 values (the oracle gets the same values)
        Sh = (Sh.view(np.uint32) & np.uint32(0xFFFF0000)).view(np.float32)
        bits = S.absmax_to_bf16(Sh)
        Sd = torch.from_numpy(bits.view(np.int16)).cuda().view(torch.bfloat16)
    counts = [1, 7, 20, 0, 40, 3]
    b = G.explicit_batch(counts, seed=12)
    x_bits = activations_bf16(14, b.T, K)
    xd = bf16_dev(x_bits)

    def run(scales):
        out = torch.empty((b.R, N), dtype=torch.bfloat16, device="cuda")
        g.grouped_gemm(fmt, xd, Wd, scales, to_dev(b.offsets), row_token=to_dev(b.row_token),
                       row_weight=to_dev(b.row_weight), row_dest=to_dev(b.row_dest), out=out, flags=FORCE_DECODE)
        g.device_status()
        return out.view(torch.int16).cpu().numpy()

    assert Sd.data_ptr() % 16 == 0
    aligned = run(Sd)
    shifted = run(_offset_copy(Sd, 1))
    assert np.array_equal(aligned, shifted), case

    ref_scales = Sh if case != "nf4_bf16" else bits
    if case == "nf4_bf16":
        ref = S.grouped_rows_f64_x("nf4", O.bf16_to_f64(x_bits), Wh, ref_scales, b.offsets, b.row_token,
                                   b.row_weight, K, np.arange(b.R))
    else:
        ref = O.grouped_rows_f64(fmt, x_bits, Wh, ref_scales, b.offsets, b.row_token, b.row_weight, K,
                                 np.arange(b.R))
    got = O.bf16_to_f64(aligned.view(np.uint16))[b.row_dest]
    scale = np.abs(ref).max(axis=1)
    err = np.abs(got - ref).max(axis=1)
    nz = scale > 0
    assert np.all(err[~nz] == 0)
    assert float((err[nz] / scale[nz]).max()) <= ROW_TOL, case
