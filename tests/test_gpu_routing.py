"""Parity of the on-device routing metadata with the oracle (bit for bit, integer
work), through the C ABI; and a grouped call fed by it equals the one fed by the
host-built metadata."""
import numpy as np
import pytest
import torch

import synth
from oracle import routing as RO
from synth import generators as G

from gpu_support import bf16_dev, bf16_host_bits, build_stack, to_dev

pytestmark = pytest.mark.gpu


def run_routing(ids, w, E):
    import bit_grouped_moe_gnf4_b200 as g
    off, tok, wt, dst = g.routing_metadata(to_dev(np.ascontiguousarray(ids, np.int32)),
                                           None if w is None else to_dev(np.ascontiguousarray(w, np.float32)), E)
    g.device_status()
    R = int(off[-1].item())
    return (off.cpu().numpy(), tok[:R].cpu().numpy(), None if wt is None else wt[:R].cpu().numpy(),
            dst[:R].cpu().numpy())


def check_same(got, want):
    for a, b, name in zip(got, want, ("offsets", "row_token", "row_weight", "row_dest")):
        if a is None:
            continue
        assert np.array_equal(a, b), name


@pytest.mark.parametrize("T,E,k,routing", [(1, 64, 8, "softmax"), (16, 64, 8, "softmax"),
                                           (4096, 128, 8, "zipf"), (64, 128, 4, "softmax"),
                                           (300, 2048, 4, "softmax"), (8192, 64, 1, "zipf")])
def test_matches_oracle_bitwise(T, E, k, routing):
    ids, w = (G.route_softmax_topk if routing == "softmax" else G.route_zipf_topk)(41, T, E, k)
    check_same(run_routing(ids, w, E), RO.routing_metadata(ids, w, E))


def test_dropped_slots_and_no_weights():
    rng = np.random.default_rng(42)
    T, E, k = 100, 16, 4
    ids = rng.integers(-3, E + 3, (T, k)).astype(np.int32)
    w = rng.random((T, k)).astype(np.float32)
    check_same(run_routing(ids, w, E), RO.routing_metadata(ids, w, E))
    off, tok, wt, dst = run_routing(ids, None, E)
    want = RO.routing_metadata(ids, w, E)
    assert wt is None
    assert np.array_equal(off, want[0]) and np.array_equal(tok, want[1]) and np.array_equal(dst, want[3])


def test_empty_and_deterministic():
    off, tok, wt, dst = run_routing(np.zeros((0, 8), np.int32), np.zeros((0, 8), np.float32), 32)
    assert np.array_equal(off, np.zeros(33, np.int64)) and len(tok) == 0
    ids, w = G.route_zipf_topk(43, 1000, 64, 8)
    first = run_routing(ids, w, 64)
    for _ in range(10):
        check_same(run_routing(ids, w, 64), first)


def test_grouped_call_fed_on_device_equals_host_metadata():
    import bit_grouped_moe_gnf4_b200 as g
    E, k, T, K, N = 16, 4, 48, 256, 128
    Wd, Sd, _, _ = build_stack("nf4", E, N, K, seed=44, oracle_experts=[])
    ids, w = G.route_softmax_topk(45, T, E, k)
    x = bf16_dev(synth.activations_bf16(46, T, K))
    off_h, tok_h, wt_h, dst_h = RO.routing_metadata(ids, w, E)
    host = g.grouped_gemm("nf4", x, Wd, Sd, to_dev(off_h), row_token=to_dev(tok_h), row_weight=to_dev(wt_h),
                          row_dest=to_dev(dst_h), T_out=T * k)
    off, tok, wt, dst = g.routing_metadata(to_dev(ids.astype(np.int32)), to_dev(w), E)
    dev = g.grouped_gemm("nf4", x, Wd, Sd, off, row_token=tok, row_weight=wt, row_dest=dst, T_out=T * k)
    g.device_status()
    assert np.array_equal(bf16_host_bits(host), bf16_host_bits(dev))
