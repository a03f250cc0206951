"""Thin torch-facing wrappers over the C ABI (argument marshalling only).

Every step of the computation runs in the CUDA kernels of libgnf4.so; these
functions only pass device pointers, sizes and the current stream.
"""
from __future__ import annotations

from typing import Optional

import torch

from . import _lib
from ._lib import lib, check


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _stream(stream) -> int:
    """A torch.cuda.Stream, a raw cudaStream_t handle as an int (0 = the legacy default
    stream), or None for torch's current stream."""
    if stream is None:
        stream = torch.cuda.current_stream()
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _need(t: torch.Tensor, dtype: torch.dtype, name: str) -> None:
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def quantize_nf4(w: torch.Tensor, packed: Optional[torch.Tensor] = None,
                 absmax: Optional[torch.Tensor] = None, stream=None):
    """fp32 ``[..., K]`` device tensor -> (packed uint8 ``[..., K//2]``, absmax fp32 ``[..., K//64]``)."""
    _need(w, torch.float32, "w")
    K = w.shape[-1]
    rows = w.numel() // K if K else 0
    lead = tuple(w.shape[:-1])
    if packed is None:
        packed = torch.empty(lead + (K // 2,), dtype=torch.uint8, device=w.device)
    if absmax is None:
        absmax = torch.empty(lead + (K // 64,), dtype=torch.float32, device=w.device)
    check(lib.gnf4_quantize_nf4(_ptr(w), rows, K, _ptr(packed), _ptr(absmax), _stream(stream)),
          "gnf4_quantize_nf4")
    return packed, absmax


def quantize_mxfp4(w: torch.Tensor, blocks: Optional[torch.Tensor] = None,
                   scales: Optional[torch.Tensor] = None, stream=None):
    """fp32 ``[..., K]`` device tensor -> (blocks uint8 ``[..., K//2]``, scales uint8 ``[..., K//32]``)."""
    _need(w, torch.float32, "w")
    K = w.shape[-1]
    rows = w.numel() // K if K else 0
    lead = tuple(w.shape[:-1])
    if blocks is None:
        blocks = torch.empty(lead + (K // 2,), dtype=torch.uint8, device=w.device)
    if scales is None:
        scales = torch.empty(lead + (K // 32,), dtype=torch.uint8, device=w.device)
    check(lib.gnf4_quantize_mxfp4(_ptr(w), rows, K, _ptr(blocks), _ptr(scales), _stream(stream)),
          "gnf4_quantize_mxfp4")
    return blocks, scales


def grouped_gemm(fmt: str, x: torch.Tensor, W: torch.Tensor, scales: torch.Tensor,
                 expert_offsets: torch.Tensor, row_token: Optional[torch.Tensor] = None,
                 row_weight: Optional[torch.Tensor] = None, row_dest: Optional[torch.Tensor] = None,
                 out: Optional[torch.Tensor] = None, T_out: Optional[int] = None, flags: int = 0,
                 R: Optional[int] = None, stream=None) -> torch.Tensor:
    """One grouped GEMM call (see include/gnf4.h). ``R`` (the routed row count) is
    taken from ``row_token``/``row_weight``/``row_dest`` when one is given, else it
    must be passed (it is never read back from the device). ``x`` is bf16 or fp16 (the
    output has its type); NF4 ``scales`` (absmax) are fp32 or bf16 (the bf16-absmax
    storage, see ``absmax_to_bf16``)."""
    if fmt not in ("nf4", "mxfp4"):
        raise ValueError("fmt must be 'nf4' or 'mxfp4'")
    if x.dtype not in (torch.bfloat16, torch.float16):
        raise TypeError(f"x must be torch.bfloat16 or torch.float16, got {x.dtype}")
    _need(x, x.dtype, "x")
    _need(W, torch.uint8, "W")
    if fmt == "nf4":
        if scales.dtype not in (torch.float32, torch.bfloat16):
            raise TypeError(f"NF4 absmax must be torch.float32 or torch.bfloat16, got {scales.dtype}")
        _need(scales, scales.dtype, "scales")
    else:
        _need(scales, torch.uint8, "scales")
    _need(expert_offsets, torch.int64, "expert_offsets")
    for name, t, dt in (("row_token", row_token, torch.int32), ("row_weight", row_weight, torch.float32),
                        ("row_dest", row_dest, torch.int32)):
        if t is not None:
            _need(t, dt, name)
    E, N, K2 = W.shape
    K = x.shape[1]
    if K2 * 2 != K:
        raise ValueError(f"W is [E, N, K/2] = {tuple(W.shape)} but x has K = {K}")
    if R is None:
        for t in (row_token, row_weight, row_dest):
            if t is not None:
                R = t.numel()
                break
    if R is None:
        raise ValueError("pass R (routed rows) when row_token, row_weight and row_dest are all None")
    if out is None:
        T_out = R if T_out is None else T_out
        out = torch.empty((T_out, N), dtype=x.dtype, device=x.device)
    else:
        _need(out, x.dtype, "out")
        T_out = out.shape[0]
    xdt = _lib.GNF4_DTYPE_F16 if x.dtype == torch.float16 else _lib.GNF4_DTYPE_BF16
    if fmt == "nf4":
        sdt = _lib.GNF4_DTYPE_BF16 if scales.dtype == torch.bfloat16 else _lib.GNF4_DTYPE_F32
        st = lib.gnf4_grouped_gemm_nf4_ex(_ptr(x), xdt, _ptr(W), _ptr(scales), sdt, _ptr(expert_offsets),
                                          _ptr(row_token), _ptr(row_weight), _ptr(row_dest), E, N, K, R,
                                          x.shape[0], T_out, _ptr(out), flags, _stream(stream))
    else:
        st = lib.gnf4_grouped_gemm_mxfp4_ex(_ptr(x), xdt, _ptr(W), _ptr(scales), _ptr(expert_offsets),
                                            _ptr(row_token), _ptr(row_weight), _ptr(row_dest), E, N, K, R,
                                            x.shape[0], T_out, _ptr(out), flags, _stream(stream))
    check(st, f"gnf4_grouped_gemm_{fmt}_ex")
    return out


def grouped_gemm_swiglu(fmt: str, x: torch.Tensor, W: torch.Tensor, scales: torch.Tensor,
                        expert_offsets: torch.Tensor, row_token: Optional[torch.Tensor] = None,
                        row_weight: Optional[torch.Tensor] = None, row_dest: Optional[torch.Tensor] = None,
                        out: Optional[torch.Tensor] = None, T_out: Optional[int] = None, flags: int = 0,
                        R: Optional[int] = None, stream=None) -> torch.Tensor:
    """gate_up grouped GEMM with the SwiGLU fused into its epilogue (include/gnf4.h,
    gnf4_grouped_gemm_swiglu_*): ``W`` is the fused gate_up stack ``[E, 2I, K/2]``, the
    result ``[T_out, I]`` holds silu(gate) * up in the activations' type."""
    if fmt not in ("nf4", "mxfp4"):
        raise ValueError("fmt must be 'nf4' or 'mxfp4'")
    if x.dtype not in (torch.bfloat16, torch.float16):
        raise TypeError(f"x must be torch.bfloat16 or torch.float16, got {x.dtype}")
    _need(x, x.dtype, "x")
    _need(W, torch.uint8, "W")
    if fmt == "nf4":
        if scales.dtype not in (torch.float32, torch.bfloat16):
            raise TypeError(f"NF4 absmax must be torch.float32 or torch.bfloat16, got {scales.dtype}")
        _need(scales, scales.dtype, "scales")
    else:
        _need(scales, torch.uint8, "scales")
    _need(expert_offsets, torch.int64, "expert_offsets")
    for name, t, dt in (("row_token", row_token, torch.int32), ("row_weight", row_weight, torch.float32),
                        ("row_dest", row_dest, torch.int32)):
        if t is not None:
            _need(t, dt, name)
    E, N, K2 = W.shape
    K = x.shape[1]
    if K2 * 2 != K:
        raise ValueError(f"W is [E, N, K/2] = {tuple(W.shape)} but x has K = {K}")
    if R is None:
        for t in (row_token, row_weight, row_dest):
            if t is not None:
                R = t.numel()
                break
    if R is None:
        raise ValueError("pass R (routed rows) when row_token, row_weight and row_dest are all None")
    if out is None:
        T_out = R if T_out is None else T_out
        out = torch.empty((T_out, N // 2), dtype=x.dtype, device=x.device)
    else:
        _need(out, x.dtype, "out")
        T_out = out.shape[0]
    xdt = _lib.GNF4_DTYPE_F16 if x.dtype == torch.float16 else _lib.GNF4_DTYPE_BF16
    if fmt == "nf4":
        sdt = _lib.GNF4_DTYPE_BF16 if scales.dtype == torch.bfloat16 else _lib.GNF4_DTYPE_F32
        st = lib.gnf4_grouped_gemm_swiglu_nf4(_ptr(x), xdt, _ptr(W), _ptr(scales), sdt, _ptr(expert_offsets),
                                              _ptr(row_token), _ptr(row_weight), _ptr(row_dest), E, N, K, R,
                                              x.shape[0], T_out, _ptr(out), flags, _stream(stream))
    else:
        st = lib.gnf4_grouped_gemm_swiglu_mxfp4(_ptr(x), xdt, _ptr(W), _ptr(scales), _ptr(expert_offsets),
                                                _ptr(row_token), _ptr(row_weight), _ptr(row_dest), E, N, K, R,
                                                x.shape[0], T_out, _ptr(out), flags, _stream(stream))
    check(st, f"gnf4_grouped_gemm_swiglu_{fmt}")
    return out


def absmax_to_bf16(absmax: torch.Tensor, out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """The lossless fp32 -> bf16 NF4 absmax cast (include/gnf4.h, gnf4_absmax_to_bf16):
    raises Gnf4Error if any value has no bf16 equal (an fp32 source)."""
    _need(absmax, torch.float32, "absmax")
    if out is None:
        out = torch.empty(absmax.shape, dtype=torch.bfloat16, device=absmax.device)
    else:
        _need(out, torch.bfloat16, "out")
    check(lib.gnf4_absmax_to_bf16(_ptr(absmax), absmax.numel(), _ptr(out), _stream(stream)),
          "gnf4_absmax_to_bf16")
    return out


def grouped_gemm_nf4(x, W, absmax, expert_offsets, **kw):
    return grouped_gemm("nf4", x, W, absmax, expert_offsets, **kw)


def grouped_gemm_mxfp4(x, W, scales, expert_offsets, **kw):
    return grouped_gemm("mxfp4", x, W, scales, expert_offsets, **kw)


def dgrad(fmt: str, grad_out: torch.Tensor, W: torch.Tensor, scales: torch.Tensor,
          expert_offsets: torch.Tensor, row_src: Optional[torch.Tensor] = None,
          row_weight: Optional[torch.Tensor] = None, R: Optional[int] = None,
          out: Optional[torch.Tensor] = None, flags: int = 0, stream=None) -> torch.Tensor:
    """Input gradient of a grouped GEMM call (include/gnf4.h): bf16 ``[R, K]`` with
    ``out[r] = w(r) * grad_out[src(r)] @ dequant(W[e(r)])``. ``R`` is taken from
    ``row_src`` / ``row_weight`` when given, else from ``grad_out`` (rows in routed order)."""
    if fmt not in ("nf4", "mxfp4"):
        raise ValueError("fmt must be 'nf4' or 'mxfp4'")
    _need(grad_out, torch.bfloat16, "grad_out")
    _need(W, torch.uint8, "W")
    _need(scales, torch.float32 if fmt == "nf4" else torch.uint8, "scales")
    _need(expert_offsets, torch.int64, "expert_offsets")
    for name, t, dt in (("row_src", row_src, torch.int32), ("row_weight", row_weight, torch.float32)):
        if t is not None:
            _need(t, dt, name)
    E, N, K2 = W.shape
    if grad_out.dim() != 2 or grad_out.shape[1] != N:
        raise ValueError(f"grad_out must be [T_in, N = {N}], got {tuple(grad_out.shape)}")
    if R is None:
        for t in (row_src, row_weight):
            if t is not None:
                R = t.numel()
                break
    if R is None:
        R = grad_out.shape[0]
    K = 2 * K2
    if out is None:
        out = torch.empty((R, K), dtype=torch.bfloat16, device=grad_out.device)
    else:
        _need(out, torch.bfloat16, "out")
        if tuple(out.shape) != (R, K):
            raise ValueError(f"out must be [{R}, {K}], got {tuple(out.shape)}")
    fn = lib.gnf4_dgrad_nf4 if fmt == "nf4" else lib.gnf4_dgrad_mxfp4
    check(fn(_ptr(grad_out), _ptr(W), _ptr(scales), _ptr(expert_offsets), _ptr(row_src), _ptr(row_weight),
             E, N, K, R, grad_out.shape[0], _ptr(out), flags, _stream(stream)), f"gnf4_dgrad_{fmt}")
    return out


def routing_metadata(topk_ids: torch.Tensor, topk_weights: Optional[torch.Tensor], E: int,
                     stream=None):
    """Router top-k ``[T, k]`` (int32 ids, fp32 weights or None) -> (expert_offsets int64 [E+1],
    row_token int32 [T*k], row_weight fp32 [T*k] or None, row_dest int32 [T*k]) on the device,
    rows sorted by (expert, token, slot) (include/gnf4.h)."""
    _need(topk_ids, torch.int32, "topk_ids")
    if topk_ids.dim() != 2:
        raise ValueError("topk_ids must be [T, k]")
    T, k = topk_ids.shape
    if topk_weights is not None:
        _need(topk_weights, torch.float32, "topk_weights")
        if tuple(topk_weights.shape) != (T, k):
            raise ValueError("topk_weights must match topk_ids")
    dev = topk_ids.device
    offsets = torch.empty(E + 1, dtype=torch.int64, device=dev)
    row_token = torch.empty(T * k, dtype=torch.int32, device=dev)
    row_weight = None if topk_weights is None else torch.empty(T * k, dtype=torch.float32, device=dev)
    row_dest = torch.empty(T * k, dtype=torch.int32, device=dev)
    check(lib.gnf4_routing_metadata(_ptr(topk_ids), _ptr(topk_weights), T, k, E, _ptr(offsets), _ptr(row_token),
                                    _ptr(row_weight), _ptr(row_dest), _stream(stream)), "gnf4_routing_metadata")
    return offsets, row_token, row_weight, row_dest


def swiglu(gate_up: torch.Tensor, out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """bf16 ``[R, 2I]`` gate_up rows -> bf16 ``[R, I]``: ``silu(gate) * up`` (include/gnf4.h)."""
    _need(gate_up, torch.bfloat16, "gate_up")
    if gate_up.dim() != 2 or gate_up.shape[1] % 2:
        raise ValueError(f"gate_up must be [R, 2I], got {tuple(gate_up.shape)}")
    R, I = gate_up.shape[0], gate_up.shape[1] // 2
    if out is None:
        out = torch.empty((R, I), dtype=torch.bfloat16, device=gate_up.device)
    else:
        _need(out, torch.bfloat16, "out")
        if tuple(out.shape) != (R, I):
            raise ValueError(f"out must be [{R}, {I}], got {tuple(out.shape)}")
    check(lib.gnf4_swiglu(_ptr(gate_up), R, I, _ptr(out), _stream(stream)), "gnf4_swiglu")
    return out


def combine_topk(y: torch.Tensor, T: int, k: int, row_of_slot: Optional[torch.Tensor] = None,
                 slot_weight: Optional[torch.Tensor] = None, out: Optional[torch.Tensor] = None,
                 stream=None) -> torch.Tensor:
    """bf16 ``[R, N]`` down rows -> bf16 ``[T, N]``: the fp32 slot-order sum over each
    token's k slots (include/gnf4.h)."""
    _need(y, torch.bfloat16, "y")
    if y.dim() != 2:
        raise ValueError("y must be [R, N]")
    for name, t, dt in (("row_of_slot", row_of_slot, torch.int32), ("slot_weight", slot_weight, torch.float32)):
        if t is not None:
            _need(t, dt, name)
            if t.numel() != T * k:
                raise ValueError(f"{name} must hold T*k = {T * k} entries, got {t.numel()}")
    R, N = y.shape
    if out is None:
        out = torch.empty((T, N), dtype=torch.bfloat16, device=y.device)
    else:
        _need(out, torch.bfloat16, "out")
        if tuple(out.shape) != (T, N):
            raise ValueError(f"out must be [{T}, {N}], got {tuple(out.shape)}")
    check(lib.gnf4_combine_topk(_ptr(y), R, N, _ptr(row_of_slot), _ptr(slot_weight), T, k, _ptr(out),
                                _stream(stream)), "gnf4_combine_topk")
    return out


def device_status(stream=None) -> None:
    """Synchronise the stream; raise if a kernel gave up waiting on a barrier."""
    check(lib.gnf4_device_status(_stream(stream)), "gnf4_device_status")


def launches_per_call(R: int, flags: int = 0) -> int:
    return lib.gnf4_grouped_gemm_launches(R, flags)


version = lib.gnf4_version
