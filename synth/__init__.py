"""Seeded synthetic inputs shared by the tests, the bench and the oracle checks.

This package draws inputs only: expert weights, activations and routing
metadata. It holds none of the grouped 4-bit GEMM's arithmetic (no codebook,
no packing, no scaling, no products), so the oracle and the CUDA path can both
consume its outputs without sharing any code of the method.
"""
from .generators import (  # noqa: F401
    bf16_bits_from_f32,
    f32_from_bf16_bits,
    expert_weights,
    activations_bf16,
    route_softmax_topk,
    route_zipf_topk,
    routing_metadata,
    RoutedBatch,
    make_routed_batch,
    explicit_batch,
    groups_to_routing,
)
from .workloads import WORKLOADS, Workload, Projection  # noqa: F401
