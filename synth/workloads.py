"""The synthetic MoE shapes the grouped 4-bit GEMM is measured and checked on.

Model names only fix shapes (experts E, top-k, hidden and intermediate
widths); no checkpoint is read. Each projection is a grouped GEMM
``out[r, :] = x[tok(r), :] @ W[e(r)].T`` with ``W[e]`` of shape ``[N, K]``.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import Tuple


@dataclass(frozen=True)
class Projection:
    name: str      # "gate_up" (reads token rows, writes sorted rows) or "down"
    K: int         # reduction width
    N: int         # output width


@dataclass(frozen=True)
class Workload:
    name: str
    fmt: str                       # "nf4" | "mxfp4"
    E: int
    top_k: Tuple[int, ...]
    T: Tuple[int, ...]
    projections: Tuple[Projection, ...]
    routing: str = "softmax"       # "softmax" | "zipf"
    # how gate_up receives its activations: "gather" = x [T, K] plus row_token (the
    # kernel reads the token rows itself); "a_cat" = the rows already in routed order,
    # [R, K] (the pages' gemm_4bit_grouped(a_cat, ...) interface, sorted outside)
    gate_up_input: str = "gather"
    note: str = field(default="", compare=False)


WORKLOADS = {
    "tiny_nf4": Workload(
        "tiny_nf4", "nf4", E=4, top_k=(2,), T=(8,),
        projections=(Projection("gate_up", K=256, N=128),),
        note="E=4, top_k=2, T=8, K=256, N=128, blocksize 64"),
    "olmoe_decode_nf4": Workload(
        "olmoe_decode_nf4", "nf4", E=64, top_k=(8,), T=(1, 16),
        projections=(Projection("gate_up", K=2048, N=2048),
                     Projection("down", K=1024, N=2048)),
        note="OLMoE-1B-7B-shaped decode: hidden 2048, fused gate_up 2x1024"),
    "qwen3_prefill_nf4": Workload(
        "qwen3_prefill_nf4", "nf4", E=128, top_k=(8,), T=(4096,),
        projections=(Projection("gate_up", K=2048, N=1536),
                     Projection("down", K=768, N=2048)),
        gate_up_input="a_cat",
        note="Qwen3-30B-A3B-shaped prefill: hidden 2048, moe_intermediate 768; gate_up reads a_cat [R, K]"),
    "gptoss_mxfp4": Workload(
        "gptoss_mxfp4", "mxfp4", E=128, top_k=(4,), T=(1, 8, 64),
        projections=(Projection("gate_up", K=2880, N=5760),
                     Projection("down", K=2880, N=2880)),
        note="gpt-oss-120b-shaped: hidden 2880, intermediate 2880"),
    "olmoe_sweep_nf4": Workload(
        "olmoe_sweep_nf4", "nf4", E=64, top_k=(1, 8),
        T=(1, 4, 16, 64, 256, 1024, 4096, 8192),
        projections=(Projection("gate_up", K=2048, N=2048),
                     Projection("down", K=1024, N=2048)),
        routing="zipf", note="M-axis sweep, Zipf(1.2)-skewed routing"),
}


def expert_bytes(fmt: str, N: int, K: int) -> dict:
    """Algorithmic bytes of one packed ``[N, K]`` expert matrix: the 4-bit codes
    (K/2 bytes per row) plus one fp32 absmax per 64 K (NF4) or one e8m0 byte per
    32 K (MXFP4)."""
    if fmt == "nf4":
        return {"nibbles": N * K // 2, "scales": N * (K // 64) * 4}
    if fmt == "mxfp4":
        return {"nibbles": N * K // 2, "scales": N * (K // 32)}
    raise ValueError(fmt)
