"""Host-side checks of the C ABI (no GPU needed, no kernel launched).

The library loads, exports every symbol include/gnf4.h declares, and rejects
bad arguments with the documented status before touching the device.
"""
import ctypes
import os
import re

import pytest

from bit_grouped_moe_gnf4_b200 import _lib
from bit_grouped_moe_gnf4_b200._lib import lib

HEADER = os.path.join(os.path.dirname(os.path.dirname(__file__)), "include", "gnf4.h")


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(gnf4_[a-z0-9_]+)\s*\(", src)))


def test_header_declares_the_ops():
    names = declared_functions()
    for op in ("gnf4_quantize_nf4", "gnf4_quantize_mxfp4", "gnf4_grouped_gemm_nf4",
               "gnf4_grouped_gemm_mxfp4", "gnf4_swiglu", "gnf4_combine_topk"):
        assert op in names


def test_library_exports_every_declared_symbol():
    names = declared_functions()
    assert names, "no declarations parsed"
    for n in names:
        assert hasattr(lib, n), f"{n} declared in gnf4.h but not exported"
    assert set(_lib.EXPORTED) == set(names)


def test_version_and_launch_count():
    assert lib.gnf4_version() >= 100
    assert lib.gnf4_grouped_gemm_launches(0, 0) == 0
    assert lib.gnf4_grouped_gemm_launches(1, 0) == 1
    assert lib.gnf4_grouped_gemm_launches(1, _lib.GNF4_CHECK) == 2
    # calls of at most 128 routed rows run every group in the decode band: one launch
    assert lib.gnf4_grouped_gemm_launches(128, 0) == 1
    assert lib.gnf4_grouped_gemm_launches(129, 0) == 2
    assert lib.gnf4_grouped_gemm_launches(129, _lib.GNF4_FORCE_DECODE) == 1


FAKE = 0x7f0000001000          # 16-byte aligned, never dereferenced: validation fails first


def _gemm(**kw):
    a = dict(x=FAKE, W=FAKE, s=FAKE, off=FAKE, tok=None, wt=None, dst=None, E=4, N=128, K=256,
             R=8, T_in=8, T_out=8, out=FAKE, flags=0)
    a.update(kw)
    return lib.gnf4_grouped_gemm_nf4(a["x"], a["W"], a["s"], a["off"], a["tok"], a["wt"], a["dst"],
                                     a["E"], a["N"], a["K"], a["R"], a["T_in"], a["T_out"],
                                     a["out"], a["flags"], None)


@pytest.mark.parametrize("kw,status", [
    (dict(x=None), _lib.GNF4_ERR_INVALID_ARG),
    (dict(off=None), _lib.GNF4_ERR_INVALID_ARG),
    (dict(out=None), _lib.GNF4_ERR_INVALID_ARG),
    (dict(E=0), _lib.GNF4_ERR_INVALID_ARG),
    (dict(R=-1), _lib.GNF4_ERR_INVALID_ARG),
    (dict(flags=0x40), _lib.GNF4_ERR_INVALID_ARG),
    (dict(flags=_lib.GNF4_FORCE_DECODE | _lib.GNF4_FORCE_PREFILL), _lib.GNF4_ERR_INVALID_ARG),
    (dict(K=96), _lib.GNF4_ERR_UNSUPPORTED_SHAPE),
    (dict(N=120), _lib.GNF4_ERR_UNSUPPORTED_SHAPE),
    (dict(E=4096), _lib.GNF4_ERR_UNSUPPORTED_SHAPE),
    (dict(T_in=4), _lib.GNF4_ERR_INVALID_ARG),          # row_token NULL needs T_in >= R
    (dict(T_out=4), _lib.GNF4_ERR_INVALID_ARG),         # row_dest NULL needs T_out >= R
    (dict(x=FAKE + 8), _lib.GNF4_ERR_MISALIGNED),
    (dict(out=FAKE + 2), _lib.GNF4_ERR_MISALIGNED),
    # fp32 absmax at a non-float boundary, offsets off their 8-byte boundary, row arrays off 4:
    # all refused before any launch (no kernel ever sees an unaligned vector load)
    (dict(s=FAKE + 2), _lib.GNF4_ERR_MISALIGNED),
    (dict(off=FAKE + 4), _lib.GNF4_ERR_MISALIGNED),
    (dict(tok=FAKE + 2), _lib.GNF4_ERR_MISALIGNED),
    (dict(wt=FAKE + 1), _lib.GNF4_ERR_MISALIGNED),
    (dict(dst=FAKE + 2), _lib.GNF4_ERR_MISALIGNED),
])
def test_grouped_gemm_argument_errors(kw, status):
    assert _gemm(**kw) == status
    assert lib.gnf4_last_error()


def test_mxfp4_shape_rule_is_k_multiple_of_32():
    st = lib.gnf4_grouped_gemm_mxfp4(FAKE, FAKE, FAKE, FAKE, None, None, None, 4, 128, 48, 8, 8, 8,
                                     FAKE, 0, None)
    assert st == _lib.GNF4_ERR_UNSUPPORTED_SHAPE


def test_quantize_argument_errors():
    assert lib.gnf4_quantize_nf4(None, 4, 64, FAKE, FAKE, None) == _lib.GNF4_ERR_INVALID_ARG
    assert lib.gnf4_quantize_nf4(FAKE, 4, 96, FAKE, FAKE, None) == _lib.GNF4_ERR_UNSUPPORTED_SHAPE
    assert lib.gnf4_quantize_mxfp4(FAKE, 4, 48, FAKE, FAKE, None) == _lib.GNF4_ERR_UNSUPPORTED_SHAPE
    assert lib.gnf4_quantize_mxfp4(FAKE, -1, 64, FAKE, FAKE, None) == _lib.GNF4_ERR_INVALID_ARG
    assert lib.gnf4_quantize_nf4(FAKE + 4, 4, 64, FAKE, FAKE, None) == _lib.GNF4_ERR_MISALIGNED


def test_glue_argument_errors():
    sw = lib.gnf4_swiglu
    assert sw(None, 4, 64, FAKE, None) == _lib.GNF4_ERR_INVALID_ARG
    assert sw(FAKE, -1, 64, FAKE, None) == _lib.GNF4_ERR_INVALID_ARG
    assert sw(FAKE, 4, 0, FAKE, None) == _lib.GNF4_ERR_INVALID_ARG
    assert sw(FAKE, 4, 60, FAKE, None) == _lib.GNF4_ERR_UNSUPPORTED_SHAPE
    assert sw(FAKE + 2, 4, 64, FAKE, None) == _lib.GNF4_ERR_MISALIGNED
    assert sw(FAKE, 4, 64, FAKE + 8, None) == _lib.GNF4_ERR_MISALIGNED
    cb = lib.gnf4_combine_topk
    assert cb(None, 8, 64, None, None, 2, 4, FAKE, None) == _lib.GNF4_ERR_INVALID_ARG
    assert cb(None, 8, 64, None, None, 0, 4, None, None) == _lib.GNF4_OK        # no work
    assert sw(None, 0, 64, None, None) == _lib.GNF4_OK
    assert cb(FAKE, 8, 64, None, None, 2, 0, FAKE, None) == _lib.GNF4_ERR_INVALID_ARG
    assert cb(FAKE, 8, 64, None, None, -1, 4, FAKE, None) == _lib.GNF4_ERR_INVALID_ARG
    assert cb(FAKE, 8, 60, None, None, 2, 4, FAKE, None) == _lib.GNF4_ERR_UNSUPPORTED_SHAPE
    assert cb(FAKE, 8, 64, None, None, 2, 1 << 31, FAKE, None) == _lib.GNF4_ERR_UNSUPPORTED_SHAPE
    assert cb(FAKE + 4, 8, 64, None, None, 2, 4, FAKE, None) == _lib.GNF4_ERR_MISALIGNED
    # host memory is refused (checked before any launch)
    buf = (ctypes.c_uint16 * 1024)()
    addr = (ctypes.addressof(buf) + 15) & ~15
    assert sw(addr, 1, 8, addr + 64, None) == _lib.GNF4_ERR_INVALID_ARG
    assert b"device memory" in lib.gnf4_last_error()


def test_dgrad_argument_errors():
    dg = lib.gnf4_dgrad_nf4

    def call(**kw):
        a = dict(g=FAKE, W=FAKE, s=FAKE, off=FAKE, src=None, wt=None, E=4, N=128, K=256, R=8, T_in=8,
                 out=FAKE, flags=0)
        a.update(kw)
        return dg(a["g"], a["W"], a["s"], a["off"], a["src"], a["wt"], a["E"], a["N"], a["K"], a["R"],
                  a["T_in"], a["out"], a["flags"], None)

    assert call(g=None) == _lib.GNF4_ERR_INVALID_ARG
    assert call(E=0) == _lib.GNF4_ERR_INVALID_ARG
    assert call(flags=_lib.GNF4_FORCE_DECODE) == _lib.GNF4_ERR_INVALID_ARG
    assert call(K=96) == _lib.GNF4_ERR_UNSUPPORTED_SHAPE          # K % 64, both formats
    assert lib.gnf4_dgrad_mxfp4(FAKE, FAKE, FAKE, FAKE, None, None, 4, 128, 96, 8, 8, FAKE, 0,
                                None) == _lib.GNF4_ERR_UNSUPPORTED_SHAPE
    assert call(N=120) == _lib.GNF4_ERR_UNSUPPORTED_SHAPE
    assert call(E=4096) == _lib.GNF4_ERR_UNSUPPORTED_SHAPE
    assert call(T_in=4) == _lib.GNF4_ERR_INVALID_ARG               # row_src NULL needs T_in >= R
    assert call(g=FAKE + 4) == _lib.GNF4_ERR_MISALIGNED
    assert call(R=0, g=None, W=None, s=None, off=None, out=None) == _lib.GNF4_OK   # no work


def test_routing_argument_errors():
    rm = lib.gnf4_routing_metadata
    assert rm(FAKE, FAKE, 8, 0, 16, FAKE, FAKE, FAKE, FAKE, None) == _lib.GNF4_ERR_INVALID_ARG     # k = 0
    assert rm(FAKE, FAKE, 8, 2, 0, FAKE, FAKE, FAKE, FAKE, None) == _lib.GNF4_ERR_INVALID_ARG     # E = 0
    assert rm(FAKE, FAKE, 8, 2, 4096, FAKE, FAKE, FAKE, FAKE, None) == _lib.GNF4_ERR_UNSUPPORTED_SHAPE
    assert rm(FAKE, FAKE, 1 << 30, 4, 16, FAKE, FAKE, FAKE, FAKE, None) == _lib.GNF4_ERR_UNSUPPORTED_SHAPE
    assert rm(None, FAKE, 8, 2, 16, FAKE, FAKE, FAKE, FAKE, None) == _lib.GNF4_ERR_INVALID_ARG
    assert rm(FAKE, FAKE, 8, 2, 16, FAKE, FAKE, None, FAKE, None) == _lib.GNF4_ERR_INVALID_ARG    # weights without row_weight
    assert rm(FAKE + 2, None, 8, 2, 16, FAKE, FAKE, None, FAKE, None) == _lib.GNF4_ERR_MISALIGNED
