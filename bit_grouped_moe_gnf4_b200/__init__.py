"""gnf4 for B200: grouped MoE GEMM on NF4 / MXFP4-packed expert weights.

The computation lives in ``libgnf4.so`` (hand-written CUDA for sm_100a, C ABI
in ``include/gnf4.h``); this package holds the in-tree build script and a thin
torch-facing binding. The binding loads the library on first use and raises if
it is missing -- there is no fallback implementation.
"""
_API = ("quantize_nf4", "quantize_mxfp4", "grouped_gemm", "grouped_gemm_nf4", "grouped_gemm_mxfp4",
        "launches_per_call", "device_status", "version", "swiglu", "combine_topk", "dgrad", "routing_metadata",
        "absmax_to_bf16", "grouped_gemm_swiglu")
_LIB = ("Gnf4Error", "GNF4_CHECK", "GNF4_FORCE_DECODE", "GNF4_FORCE_PREFILL", "GNF4_TEST_STALL", "GNF4_DTYPE_BF16", "GNF4_DTYPE_F16",
        "GNF4_DTYPE_F32")

__all__ = list(_API + _LIB)


def __getattr__(name):
    # load libgnf4.so only when the binding is used, so that the build script
    # (a submodule of this package) can run before the library exists
    if name in _API:
        from . import api
        return getattr(api, name)
    if name in _LIB:
        from . import _lib
        return getattr(_lib, name)
    raise AttributeError(name)
