"""The torch binding on a host without a GPU: argument checks raise before the
library is called, and host (CPU) tensors reach the C ABI only to be refused --
there is no CPU fallback anywhere in the product path."""
import pytest
import torch

import bit_grouped_moe_gnf4_b200 as g
from bit_grouped_moe_gnf4_b200 import _lib


def test_wrong_dtypes_and_shapes_raise_before_the_library():
    with pytest.raises(TypeError):
        g.swiglu(torch.zeros((4, 16), dtype=torch.float32))
    with pytest.raises(ValueError):
        g.swiglu(torch.zeros((4, 15), dtype=torch.bfloat16))          # not [R, 2I]
    with pytest.raises(ValueError):
        g.swiglu(torch.zeros((4, 16), dtype=torch.bfloat16), out=torch.zeros((4, 9), dtype=torch.bfloat16))
    with pytest.raises(ValueError):
        g.swiglu(torch.zeros((4, 32), dtype=torch.bfloat16)[:, ::2])  # not contiguous
    with pytest.raises(ValueError):
        g.combine_topk(torch.zeros((8, 16), dtype=torch.bfloat16), 2, 4,
                       row_of_slot=torch.zeros(5, dtype=torch.int32))  # not T*k entries
    with pytest.raises(TypeError):
        g.routing_metadata(torch.zeros((2, 4), dtype=torch.int64), None, 8)
    W = torch.zeros((2, 32, 64), dtype=torch.uint8)
    S = torch.zeros((2, 32, 2), dtype=torch.float32)
    off = torch.zeros(3, dtype=torch.int64)
    with pytest.raises(ValueError):
        g.dgrad("nf4", torch.zeros((4, 31), dtype=torch.bfloat16), W, S, off)  # grad width != N
    with pytest.raises(ValueError):
        g.dgrad("int4", torch.zeros((4, 32), dtype=torch.bfloat16), W, S, off)
    with pytest.raises(ValueError):
        g.grouped_gemm("nf4", torch.zeros((4, 100), dtype=torch.bfloat16), W, S, off, R=4)  # K mismatch


def test_host_tensors_are_refused_by_the_library():
    # well-formed calls with CPU tensors (stream 0: the raw legacy default stream, so that
    # no torch CUDA call is needed): the C ABI checks every pointer and refuses
    with pytest.raises(_lib.Gnf4Error) as ei:
        g.swiglu(torch.zeros((4, 16), dtype=torch.bfloat16), stream=0)
    assert ei.value.status == _lib.GNF4_ERR_INVALID_ARG
    assert "device memory" in str(ei.value)
    with pytest.raises(_lib.Gnf4Error):
        g.combine_topk(torch.zeros((8, 16), dtype=torch.bfloat16), 2, 4, stream=0)
    with pytest.raises(_lib.Gnf4Error):
        g.routing_metadata(torch.zeros((2, 4), dtype=torch.int32), torch.zeros((2, 4)), 8, stream=0)
    W = torch.zeros((2, 32, 64), dtype=torch.uint8)
    S = torch.zeros((2, 32, 2), dtype=torch.float32)
    off = torch.tensor([0, 2, 4], dtype=torch.int64)
    with pytest.raises(_lib.Gnf4Error):
        g.dgrad("nf4", torch.zeros((4, 32), dtype=torch.bfloat16), W, S, off, stream=0)
    with pytest.raises(_lib.Gnf4Error):
        g.grouped_gemm("nf4", torch.zeros((4, 128), dtype=torch.bfloat16), W, S, off, R=4, stream=0)
    with pytest.raises(_lib.Gnf4Error):
        g.quantize_nf4(torch.zeros((4, 128), dtype=torch.float32), stream=0)


def test_empty_calls_need_no_device():
    # no work: the library returns before looking at any pointer
    assert g.swiglu(torch.zeros((0, 16), dtype=torch.bfloat16), stream=0).shape == (0, 8)
    assert g.combine_topk(torch.zeros((0, 16), dtype=torch.bfloat16), 0, 4, stream=0).shape == (0, 16)
