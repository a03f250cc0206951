"""gnf4 for B200: grouped MoE GEMM on NF4 / MXFP4-packed expert weights.

The computation lives in ``libgnf4.so`` (hand-written CUDA for sm_100a, C ABI
in ``include/gnf4.h``); this package holds the in-tree build script and a thin
torch-facing binding. Importing it without the built library raises.
"""
from .api import (  # noqa: F401
    quantize_nf4,
    quantize_mxfp4,
    grouped_gemm,
    grouped_gemm_nf4,
    grouped_gemm_mxfp4,
    launches_per_call,
    version,
)
from ._lib import Gnf4Error, GNF4_CHECK, GNF4_FORCE_DECODE, GNF4_FORCE_PREFILL  # noqa: F401
