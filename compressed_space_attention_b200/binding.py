"""ctypes binding of libisoq (``include/isoq.h``): argument marshalling only.

Every function here has the name of the C entry point it calls.  Tensors
provide device memory and strides; the current torch CUDA stream of the
tensors' device is passed as the stream.  All computation happens in the
library's CUDA kernels: there is no CPU or Python fallback, and a missing
library raises at import of this module's functions.
"""

from __future__ import annotations

import ctypes
import math
import os
from typing import Optional, Tuple

import numpy as np

ISOQ_OK = 0
ISOQ_ERR_INVALID_ARG = -1
ISOQ_ERR_UNSUPPORTED = -2
ISOQ_ERR_CUDA = -3
ISOQ_ERR_TIMEOUT = -4
ISOQ_FULL = 0
ISOQ_FAST = 1
ISOQ_PLANAR = 2
ISOQ_BLOCK_SO4 = 3
ISOQ_SO3 = 4
ISOQ_F16 = 0
ISOQ_F32 = 1

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libisoq.so")

# (name, restype, argtypes) of every exported entry point of include/isoq.h.
_P = ctypes.c_void_p
_I = ctypes.c_int
_I64 = ctypes.c_int64
_SZ = ctypes.c_size_t
_F = ctypes.c_float
SIGNATURES = [
    ("isoq_status_string", ctypes.c_char_p, [_I]),
    ("isoq_last_error", ctypes.c_char_p, []),
    ("isoq_abi_version", _I, []),
    ("isoq_params_size", _I, [_I]),
    ("isoq_packed_bytes", _SZ, [_I, _I]),
    ("isoq_make_params", _I, [_I, _I, ctypes.c_uint64, _I, _P]),
    ("isoq_make_codebook", _I, [_I, _I, _P, _P]),
    ("isoq_quantize", _I, [_P, _I, _I, _I64, _I, _I, _I, _I64, _I64, _P, _P, _P, _I64, _P]),
    ("isoq_dequantize", _I, [_P, _P, _I, _I64, _I, _I, _I, _I64, _P, _P, _I, _I64, _I64, _P]),
    ("isoq_decode_num_splits", _I, [_I, _I, _I64, _I]),
    ("isoq_decode_workspace_size", _SZ, [_I, _I, _I, _I64, _I]),
    ("isoq_decode_attention", _I, [_P, _I, _P, _P, _P, _P, _P, _I, _I, _I, _I64, _I, _I, _I,
                                   _P, _P, _F, _P, _P, _SZ, _P]),
    ("isoq_decode_split", _I, [_P, _I, _P, _P, _P, _P, _P, _I, _I, _I, _I64, _I, _I, _I, _P,
                               _F, _P, _SZ, _P]),
    ("isoq_decode_combine", _I, [_I, _P, _I, _I, _I, _I64, _I, _I, _P, _P, _P, _SZ, _P]),
    ("isoq_decode_append", _I, [_P, _P, _I, _P, _P, _P, _P, _P, _I, _I, _I64, _I, _I, _I, _P, _P, _P]),
    ("isoq_decode_step", _I, [_P, _P, _P, _I, _P, _P, _P, _P, _P, _I, _I, _I, _I64, _I, _I, _I, _P, _P,
                              _F, _P, _P, _SZ, _P]),
    ("isoq_check_device_error", _I, [_P]),
    ("isoq_selftest_wait_timeout", _I, [ctypes.c_uint64, _P]),
    ("isoq_prefill_attention", _I, [_P, _I, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I64, _I, _I, _I,
                                    _P, _P, _F, _P, _P]),
    ("isoq_rotor_groups", _I, [_I]),
    ("isoq_rotor_packed_bytes", _SZ, [_I, _I]),
    ("isoq_rotor_make_params", _I, [_I, ctypes.c_uint64, _I, _P]),
    ("isoq_rotor_quantize", _I, [_P, _I, _I, _I64, _I, _I, _I64, _I64, _P, _P, _P, _I64, _P]),
    ("isoq_rotor_dequantize", _I, [_P, _P, _I, _I64, _I, _I, _I64, _P, _P, _I, _I64, _I64, _P]),
    ("isoq_decode_static_workspace_bytes", _SZ, []),
    ("isoq_decode_attention_static", _I, [_P, _I, _P, _P, _P, _P, _P, _I, _I, _I, _I64, _I, _I,
                                          _I, _P, _P, _F, _P, _P]),
]

_lib = None


class IsoqError(RuntimeError):
    """A non-zero status from libisoq."""

    def __init__(self, status: int, where: str, detail: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)} ({status}): {detail}")


def lib() -> ctypes.CDLL:
    """The loaded library (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing; build it with "
                              "`python -m compressed_space_attention_b200.build`")
        handle = ctypes.CDLL(LIB_PATH)
        for name, res, args in SIGNATURES:
            fn = getattr(handle, name)
            fn.restype = res
            fn.argtypes = args
        _lib = handle
    return _lib


def status_string(status: int) -> str:
    return lib().isoq_status_string(status).decode()


def last_error() -> str:
    return lib().isoq_last_error().decode()


def _check(status: int, where: str) -> None:
    if status != ISOQ_OK:
        raise IsoqError(status, where, last_error())


# ---------------------------------------------------------------------------
# Host-only entry points
# ---------------------------------------------------------------------------

def isoq_abi_version() -> int:
    return lib().isoq_abi_version()


def isoq_params_size(d: int) -> int:
    return lib().isoq_params_size(d)


def isoq_packed_bytes(d: int, bits: int) -> int:
    return lib().isoq_packed_bytes(d, bits)


def isoq_make_params(d: int, variant: int, seed: int, n_heads: int = 1) -> np.ndarray:
    """float32 [n_heads][d/4][8] rotation parameters (host array)."""
    out = np.empty((n_heads, d // 4, 8), dtype=np.float32)
    _check(lib().isoq_make_params(d, variant, ctypes.c_uint64(seed & (2 ** 64 - 1)), n_heads,
                                  out.ctypes.data_as(_P)), "isoq_make_params")
    return out


def isoq_make_codebook(d: int, bits: int) -> Tuple[np.ndarray, np.ndarray]:
    """(centroids[2^bits], thresholds[2^bits - 1]) as float64 host arrays."""
    c = np.empty(1 << bits, dtype=np.float64)
    t = np.empty((1 << bits) - 1, dtype=np.float64)
    _check(lib().isoq_make_codebook(d, bits, c.ctypes.data_as(_P), t.ctypes.data_as(_P)),
           "isoq_make_codebook")
    return c, t


def isoq_decode_num_splits(B: int, Hkv: int, Tmax: int, d: int) -> int:
    n = lib().isoq_decode_num_splits(B, Hkv, Tmax, d)
    if n < 0:
        raise IsoqError(n, "isoq_decode_num_splits", "")
    return n


def isoq_decode_workspace_size(B: int, Hq: int, Hkv: int, Tmax: int, d: int) -> int:
    return lib().isoq_decode_workspace_size(B, Hq, Hkv, Tmax, d)


# ---------------------------------------------------------------------------
# Device entry points (torch tensors)
# ---------------------------------------------------------------------------

def _torch():
    import torch
    return torch


def _dtype_code(t) -> int:
    torch = _torch()
    if t.dtype == torch.float16:
        return ISOQ_F16
    if t.dtype == torch.float32:
        return ISOQ_F32
    raise TypeError(f"unsupported dtype {t.dtype}; float16 or float32 expected")


def _torch_dtype(code: int):
    torch = _torch()
    return torch.float16 if code == ISOQ_F16 else torch.float32


def _require_cuda(*tensors):
    dev = None
    for t in tensors:
        if t is None:
            continue
        if not t.is_cuda:
            raise ValueError("libisoq entry points take CUDA tensors (there is no CPU path)")
        if dev is None:
            dev = t.device
        elif t.device != dev:
            raise ValueError("all tensors must be on the same device")
    return dev


def _stream(dev, stream=None) -> int:
    torch = _torch()
    if stream is not None:
        return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)
    return torch.cuda.current_stream(dev).cuda_stream


def _ptr(t) -> Optional[int]:
    return None if t is None else t.data_ptr()


def isoq_quantize(x, params, bits: int, variant: int, codes=None, norms=None,
                  out_head_stride: Optional[int] = None, stream=None):
    """Compresses x [n_heads][n_vec][d] (or [n_vec][d]); returns (codes, norms).

    codes: uint8 [n_heads][n_vec][d*bits/8]; norms: float16 [n_heads][n_vec].
    Preallocated outputs may be views into a larger cache: pass
    ``out_head_stride`` (vectors between heads) for that.
    """
    torch = _torch()
    if x.dim() == 2:
        x = x.unsqueeze(0)
    n_heads, n_vec, d = x.shape
    if x.stride(2) != 1:
        raise ValueError("the last dimension of x must be contiguous")
    dev = _require_cuda(x, params, codes, norms)
    pb = isoq_packed_bytes(d, bits)
    if codes is None:
        codes = torch.empty((n_heads, n_vec, pb), dtype=torch.uint8, device=dev)
    if norms is None:
        norms = torch.empty((n_heads, n_vec), dtype=torch.float16, device=dev)
    if out_head_stride is None:
        out_head_stride = n_vec
    with torch.cuda.device(dev):
        st = lib().isoq_quantize(_ptr(x), _dtype_code(x), n_heads, n_vec, d, bits, variant,
                                 x.stride(0), x.stride(1), _ptr(params), _ptr(codes), _ptr(norms),
                                 out_head_stride, _stream(dev, stream))
    _check(st, "isoq_quantize")
    return codes, norms


def isoq_dequantize(codes, norms, params, d: int, bits: int, variant: int, out_dtype=None,
                    out=None, in_head_stride: Optional[int] = None, stream=None):
    """Reconstructs [n_heads][n_vec][d] vectors from codes and float16 norms."""
    torch = _torch()
    if codes.dim() == 2:
        codes = codes.unsqueeze(0)
        norms = norms.unsqueeze(0)
    n_heads, n_vec, _ = codes.shape
    dev = _require_cuda(codes, norms, params, out)
    if out is None:
        out = torch.empty((n_heads, n_vec, d), dtype=out_dtype or torch.float32, device=dev)
    if in_head_stride is None:
        in_head_stride = n_vec
    with torch.cuda.device(dev):
        st = lib().isoq_dequantize(_ptr(codes), _ptr(norms), n_heads, n_vec, d, bits, variant,
                                   in_head_stride, _ptr(params), _ptr(out), _dtype_code(out),
                                   out.stride(0), out.stride(1), _stream(dev, stream))
    _check(st, "isoq_dequantize")
    return out


def isoq_prefill_attention(q, packed_k, packed_v, norms_k, norms_v, seq_lens, params_k, params_v,
                           bits: int, variant: int, scale: Optional[float] = None, out=None, stream=None):
    """Causal attention of q [B][Tq][Hq][d] over the packed cache that holds
    the chunk (seq_lens counts it); returns out [B][Tq][Hq][d] (dtype of q)."""
    torch = _torch()
    B, Tq, Hq, d = q.shape
    _, Hkv, Tmax, pb = packed_k.shape
    if pb != isoq_packed_bytes(d, bits):
        raise ValueError("packed row size does not match d and bits")
    if not q.is_contiguous():
        raise ValueError("q must be contiguous")
    dev = _require_cuda(q, packed_k, packed_v, norms_k, norms_v, seq_lens, params_k, params_v, out)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty((B, Tq, Hq, d), dtype=q.dtype, device=dev)
    with torch.cuda.device(dev):
        st = lib().isoq_prefill_attention(
            _ptr(q), _dtype_code(q), _ptr(packed_k), _ptr(packed_v), _ptr(norms_k), _ptr(norms_v),
            _ptr(seq_lens), B, Tq, Hq, Hkv, Tmax, d, bits, variant, _ptr(params_k), _ptr(params_v),
            float(scale), _ptr(out), _stream(dev, stream))
    _check(st, "isoq_prefill_attention")
    return out


def isoq_rotor_groups(d: int) -> int:
    return lib().isoq_rotor_groups(d)


def isoq_rotor_packed_bytes(d: int, bits: int) -> int:
    return lib().isoq_rotor_packed_bytes(d, bits)


def isoq_rotor_make_params(d: int, seed: int, n_heads: int = 1) -> np.ndarray:
    """float32 [n_heads][G][4] unit rotors (s, p12, p13, p23) (host array)."""
    out = np.empty((n_heads, max(isoq_rotor_groups(d), 0), 4), dtype=np.float32)
    _check(lib().isoq_rotor_make_params(d, ctypes.c_uint64(seed & (2 ** 64 - 1)), n_heads,
                                        out.ctypes.data_as(_P)), "isoq_rotor_make_params")
    return out


def isoq_rotor_quantize(x, rotors, bits: int, codes=None, norms=None, stream=None):
    """RotorQuant comparator: compresses x [n_heads][n_vec][d]; returns (codes, norms)."""
    torch = _torch()
    if x.dim() == 2:
        x = x.unsqueeze(0)
    n_heads, n_vec, d = x.shape
    if x.stride(2) != 1:
        raise ValueError("the last dimension of x must be contiguous")
    dev = _require_cuda(x, rotors, codes, norms)
    if codes is None:
        codes = torch.empty((n_heads, n_vec, isoq_rotor_packed_bytes(d, bits)), dtype=torch.uint8, device=dev)
    if norms is None:
        norms = torch.empty((n_heads, n_vec), dtype=torch.float16, device=dev)
    with torch.cuda.device(dev):
        st = lib().isoq_rotor_quantize(_ptr(x), _dtype_code(x), n_heads, n_vec, d, bits, x.stride(0),
                                       x.stride(1), _ptr(rotors), _ptr(codes), _ptr(norms), n_vec,
                                       _stream(dev, stream))
    _check(st, "isoq_rotor_quantize")
    return codes, norms


def isoq_rotor_dequantize(codes, norms, rotors, d: int, bits: int, out_dtype=None, out=None, stream=None):
    """RotorQuant comparator: reconstructs [n_heads][n_vec][d] from codes and norms."""
    torch = _torch()
    if codes.dim() == 2:
        codes = codes.unsqueeze(0)
        norms = norms.unsqueeze(0)
    n_heads, n_vec, _ = codes.shape
    dev = _require_cuda(codes, norms, rotors, out)
    if out is None:
        out = torch.empty((n_heads, n_vec, d), dtype=out_dtype or torch.float32, device=dev)
    with torch.cuda.device(dev):
        st = lib().isoq_rotor_dequantize(_ptr(codes), _ptr(norms), n_heads, n_vec, d, bits, n_vec,
                                         _ptr(rotors), _ptr(out), _dtype_code(out), out.stride(0),
                                         out.stride(1), _stream(dev, stream))
    _check(st, "isoq_rotor_dequantize")
    return out


def _decode_shapes(q, packed_k, bits):
    B, Hq, d = q.shape
    _, Hkv, Tmax, pb = packed_k.shape
    if pb != isoq_packed_bytes(d, bits):
        raise ValueError("packed row size does not match d and bits")
    return B, Hq, Hkv, Tmax, d


def isoq_decode_attention(q, packed_k, packed_v, norms_k, norms_v, seq_lens, params_k,
                          params_v, bits: int, variant: int, scale: Optional[float] = None,
                          out=None, workspace=None, stream=None):
    """Decode attention over packed K/V; returns out [B][Hq][d] (dtype of q)."""
    torch = _torch()
    B, Hq, Hkv, Tmax, d = _decode_shapes(q, packed_k, bits)
    dev = _require_cuda(q, packed_k, packed_v, norms_k, norms_v, seq_lens, params_k, params_v,
                        out, workspace)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty((B, Hq, d), dtype=q.dtype, device=dev)
    ws_bytes = isoq_decode_workspace_size(B, Hq, Hkv, Tmax, d)
    if workspace is None:
        workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    with torch.cuda.device(dev):
        st = lib().isoq_decode_attention(
            _ptr(q), _dtype_code(q), _ptr(packed_k), _ptr(packed_v), _ptr(norms_k), _ptr(norms_v),
            _ptr(seq_lens), B, Hq, Hkv, Tmax, d, bits, variant, _ptr(params_k), _ptr(params_v),
            float(scale), _ptr(out), _ptr(workspace), workspace.numel() * workspace.element_size(),
            _stream(dev, stream))
    _check(st, "isoq_decode_attention")
    return out


def isoq_decode_append(k_new, v_new, packed_k, packed_v, norms_k, norms_v, seq_lens, params_k,
                       params_v, bits: int, variant: int, stream=None):
    """Compresses k_new/v_new [B][Hkv][d] into the packed cache at seq_lens[b]
    and advances seq_lens, in place on the device."""
    B, Hkv, d = k_new.shape
    _, _, Tmax, pb = packed_k.shape
    if pb != isoq_packed_bytes(d, bits):
        raise ValueError("packed row size does not match d and bits")
    dev = _require_cuda(k_new, v_new, packed_k, packed_v, norms_k, norms_v, seq_lens, params_k,
                        params_v)
    torch = _torch()
    with torch.cuda.device(dev):
        st = lib().isoq_decode_append(
            _ptr(k_new), _ptr(v_new), _dtype_code(k_new), _ptr(packed_k), _ptr(packed_v),
            _ptr(norms_k), _ptr(norms_v), _ptr(seq_lens), B, Hkv, Tmax, d, bits, variant,
            _ptr(params_k), _ptr(params_v), _stream(dev, stream))
    _check(st, "isoq_decode_append")


def isoq_decode_step(q, k_new, v_new, packed_k, packed_v, norms_k, norms_v, seq_lens, params_k,
                     params_v, bits: int, variant: int, scale: Optional[float] = None, out=None,
                     workspace=None, stream=None):
    """Append (k_new, v_new) to the packed cache, then decode attention of q
    over it; returns out [B][Hq][d] (dtype of q)."""
    torch = _torch()
    B, Hq, Hkv, Tmax, d = _decode_shapes(q, packed_k, bits)
    dev = _require_cuda(q, k_new, v_new, packed_k, packed_v, norms_k, norms_v, seq_lens, params_k,
                        params_v, out, workspace)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty((B, Hq, d), dtype=q.dtype, device=dev)
    ws_bytes = isoq_decode_workspace_size(B, Hq, Hkv, Tmax, d)
    if workspace is None:
        workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    with torch.cuda.device(dev):
        st = lib().isoq_decode_step(
            _ptr(q), _ptr(k_new), _ptr(v_new), _dtype_code(q), _ptr(packed_k), _ptr(packed_v),
            _ptr(norms_k), _ptr(norms_v), _ptr(seq_lens), B, Hq, Hkv, Tmax, d, bits, variant,
            _ptr(params_k), _ptr(params_v), float(scale), _ptr(out), _ptr(workspace),
            workspace.numel() * workspace.element_size(), _stream(dev, stream))
    _check(st, "isoq_decode_step")
    return out


def isoq_decode_split(q, packed_k, packed_v, norms_k, norms_v, seq_lens, params_k, bits: int,
                      variant: int, workspace, scale: Optional[float] = None, stream=None):
    """First launch of the decode: partial states into ``workspace``."""
    B, Hq, Hkv, Tmax, d = _decode_shapes(q, packed_k, bits)
    dev = _require_cuda(q, packed_k, packed_v, norms_k, norms_v, seq_lens, params_k, workspace)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    torch = _torch()
    with torch.cuda.device(dev):
        st = lib().isoq_decode_split(
            _ptr(q), _dtype_code(q), _ptr(packed_k), _ptr(packed_v), _ptr(norms_k), _ptr(norms_v),
            _ptr(seq_lens), B, Hq, Hkv, Tmax, d, bits, variant, _ptr(params_k), float(scale),
            _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(dev, stream))
    _check(st, "isoq_decode_split")


def isoq_decode_combine(out, seq_lens, B: int, Hq: int, Hkv: int, Tmax: int, d: int,
                        variant: int, params_v, workspace, stream=None):
    """Second launch of the decode: merge + inverse rotation into ``out``."""
    dev = _require_cuda(out, seq_lens, params_v, workspace)
    torch = _torch()
    with torch.cuda.device(dev):
        st = lib().isoq_decode_combine(
            _dtype_code(out), _ptr(seq_lens), B, Hq, Hkv, Tmax, d, variant, _ptr(params_v),
            _ptr(out), _ptr(workspace), workspace.numel() * workspace.element_size(),
            _stream(dev, stream))
    _check(st, "isoq_decode_combine")
    return out


def isoq_selftest_wait_timeout(limit_ns: int = 50_000_000, stream=None, device=None) -> None:
    """Launches the failure-path self-test (a device wait on a barrier that
    nothing arrives at, given up after limit_ns); the next
    isoq_check_device_error then returns ISOQ_ERR_TIMEOUT."""
    torch = _torch()
    dev = device if device is not None else torch.device("cuda", torch.cuda.current_device())
    with torch.cuda.device(dev):
        _check(lib().isoq_selftest_wait_timeout(int(limit_ns), _stream(dev, stream)),
               "isoq_selftest_wait_timeout")


def isoq_check_device_error(stream=None, device=None) -> int:
    """Synchronises the stream and returns (and clears) the device error status."""
    torch = _torch()
    dev = device if device is not None else torch.device("cuda", torch.cuda.current_device())
    with torch.cuda.device(dev):
        return lib().isoq_check_device_error(_stream(dev, stream))


def _torch_dtype_of(code: int):
    return _torch_dtype(code)


def isoq_decode_attention_static(q, packed_k, packed_v, norms_k, norms_v, seq_lens, params_k,
                                 params_v, bits: int, variant: int, scale: Optional[float] = None,
                                 out=None, stream=None):
    """isoq_decode_attention with the library's built-in device workspace.

    For callers that cannot allocate device scratch; the output buffer may be
    passed in (``out``) so that the call itself allocates nothing.
    """
    torch = _torch()
    B, Hq, Hkv, Tmax, d = _decode_shapes(q, packed_k, bits)
    dev = _require_cuda(q, packed_k, packed_v, norms_k, norms_v, seq_lens, params_k, params_v, out)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty((B, Hq, d), dtype=q.dtype, device=dev)
    with torch.cuda.device(dev):
        st = lib().isoq_decode_attention_static(
            _ptr(q), _dtype_code(q), _ptr(packed_k), _ptr(packed_v), _ptr(norms_k), _ptr(norms_v),
            _ptr(seq_lens), B, Hq, Hkv, Tmax, d, bits, variant, _ptr(params_k), _ptr(params_v),
            float(scale), _ptr(out), _stream(dev, stream))
    _check(st, "isoq_decode_attention_static")
    return out


def isoq_decode_static_workspace_bytes() -> int:
    return lib().isoq_decode_static_workspace_bytes()
