"""GPU quantizers against the oracle's: packed bytes and scales bit for bit."""
import numpy as np
import pytest
import torch

import synth
from oracle import gnf4_oracle as O
from synth import generators as G

pytestmark = pytest.mark.gpu


def _adversarial(rows, K, seed):
    rng = np.random.default_rng(seed)
    w = (rng.standard_normal((rows, K)) * 0.02).astype(np.float32)
    w[0, :64] = 0.0                                   # all-zero block
    w[1, :64] = -3.5                                  # constant block
    w[2, 64:128] = rng.standard_normal(64).astype(np.float32) * 1e30
    w[3, :64] = rng.standard_normal(64).astype(np.float32) * 1e-38   # subnormal range
    w[4, :32] = 1.9                                   # MXFP4 saturation
    w[5, :64] = O.nf4_thresholds()[np.arange(64) % 15]  # exact NF4 midpoints (absmax < 1)
    w[5, 0] = 1.0                                     # absmax 1 so x = w exactly
    mids = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.0], np.float32) / 4
    w[6, :32] = np.resize(mids, 32) * np.where(np.arange(32) % 2, -1, 1)   # e2m1 ties
    w[7, :64] = -0.0
    return w


@pytest.mark.parametrize("rows,K", [(64, 256), (37, 2048), (512, 2880 * 2)])
def test_quantize_nf4_bit_exact(rows, K):
    import bit_grouped_moe_gnf4_b200 as g
    if K % 64:
        pytest.skip("NF4 needs K % 64 == 0")
    w = _adversarial(rows, K, rows + K)
    p_ref, a_ref = O.quantize_nf4(w)
    p, a = g.quantize_nf4(torch.from_numpy(w).cuda())
    torch.cuda.synchronize()
    assert np.array_equal(p.cpu().numpy(), p_ref)
    assert np.array_equal(a.cpu().numpy().view(np.uint32), a_ref.view(np.uint32))


@pytest.mark.parametrize("rows,K", [(64, 256), (37, 2880), (300, 5760)])
def test_quantize_mxfp4_bit_exact(rows, K):
    import bit_grouped_moe_gnf4_b200 as g
    w = _adversarial(rows, K, rows * 3 + K)
    b_ref, s_ref = O.quantize_mxfp4(w)
    b, s = g.quantize_mxfp4(torch.from_numpy(w).cuda())
    torch.cuda.synchronize()
    assert np.array_equal(b.cpu().numpy(), b_ref)
    assert np.array_equal(s.cpu().numpy(), s_ref)


def test_quantize_full_expert_shapes_match():
    """One full OLMoE gate_up expert (2048 x 2048) and one gpt-oss gate_up expert
    (5760 x 2880) from the synthetic weight recipe."""
    import bit_grouped_moe_gnf4_b200 as g
    w = G.expert_weights(0, 3, 2048, 2048)
    p, a = g.quantize_nf4(torch.from_numpy(w).cuda())
    p_ref, a_ref = O.quantize_nf4(w)
    assert np.array_equal(p.cpu().numpy(), p_ref) and np.array_equal(a.cpu().numpy(), a_ref)
    w = G.expert_weights(0, 5, 5760, 2880)
    b, s = g.quantize_mxfp4(torch.from_numpy(w).cuda())
    b_ref, s_ref = O.quantize_mxfp4(w)
    assert np.array_equal(b.cpu().numpy(), b_ref) and np.array_equal(s.cpu().numpy(), s_ref)
