"""Host-side checks of bench.py's multi-rank logic, on CPU: a world of two gloo
ranks for the max-over-ranks timing, and the reference arm's rank behaviour."""
import json
import os
import socket
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        got = bench.max_over_ranks([1.0 + rank, 5.0 - rank, 0.25 * rank], "cpu")
        q.put((rank, got))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_two_gloo_ranks():
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = dict(q.get(timeout=10) for _ in range(2))
    # every rank sees the maximum of each entry over both ranks
    for r in range(2):
        assert res[r] == [2.0, 5.0, 0.25]


def test_max_over_ranks_single_process_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks([3.0, 4.5], "cpu") == [3.0, 4.5]


def test_replica_rate_is_weak_scaling():
    sys.path.insert(0, ROOT)
    import bench
    one = bench.replica_rate(1, 100.0, 2.0)
    assert one == 50.0
    assert bench.replica_rate(4, 100.0, 2.0) == 4 * one          # same per-rank work and time


def _run_bench(env_extra, args):
    env = dict(os.environ, **env_extra)
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py")] + args, cwd=ROOT, env=env,
                          capture_output=True, text=True, timeout=600)


def test_reference_arm_other_ranks_exit_quietly():
    r = _run_bench({"RANK": "1", "WORLD_SIZE": "2", "LOCAL_RANK": "1"},
                   ["--impl", "reference", "--workload", "tiny_nf4", "--steps", "1", "--warmup", "1"])
    assert r.returncode == 0, r.stderr[-2000:]
    assert r.stdout.strip() == ""


def test_reference_arm_rank0_prints_one_line():
    r = _run_bench({"RANK": "0", "WORLD_SIZE": "1"},
                   ["--impl", "reference", "--workload", "tiny_nf4", "--steps", "1", "--warmup", "1"])
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference"
    assert d["unit"] == "GB/s" and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0


def test_glue_and_dgrad_accounting():
    """Byte counts of the glue legs and the inputs of the gradient leg, on the workload
    shapes (host arithmetic only)."""
    import bench
    import synth
    from synth.workloads import WORKLOADS
    wl = WORKLOADS["qwen3_prefill_nf4"]
    # SwiGLU: [32768, 1536] bf16 read, [32768, 768] written
    assert bench.glue_problem("swiglu", wl, 8, 4096) == (32768, 1536, 32768, 768,
                                                         32768 * 1536 * 2 + 32768 * 768 * 2)
    # combine: [32768, 2048] read, [4096, 2048] written
    assert bench.glue_problem("combine", wl, 8, 4096) == (32768, 2048, 4096, 2048,
                                                          32768 * 2048 * 2 + 4096 * 2048 * 2)
    # gradient of down: gathered from the forward's scatter rows with its weights;
    # gradient of gate_up: rows already in routed order, unweighted
    b = synth.make_routed_batch(0, 16, 64, 8)
    gu, dn = WORKLOADS["olmoe_decode_nf4"].projections
    src, wt, gb = bench.dgrad_call_inputs(dn, b, 0)
    assert src is b.row_dest and wt is b.row_weight and gb.shape == (16 * 8, dn.N)
    src, wt, gb = bench.dgrad_call_inputs(gu, b, 0)
    assert src is None and wt is None and gb.shape == (b.R, gu.N)
