"""Thin ctypes binding of libbsq (include/bsq.h), one Python function per entry point.

Argument marshalling only: each function takes torch tensors that already
live on the GPU, allocates any output the caller did not pass (torch is the
allocator), and calls the C entry point of the same name on torch's current
stream.  Every step of the computation runs in the CUDA kernels of libbsq;
there is no CPU or library fallback -- importing this module raises if
libbsq.so has not been built, and a call raises BsqError if the library
rejects it.  bf16 tensors may be passed as torch.bfloat16 (or as int16/uint16
bit patterns).
"""
from __future__ import annotations

import ctypes
import enum
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
# BSQ_LIBRARY may name another build of the same library, e.g. the
# bounds-checking libbsq_debug.so
lib_path = os.environ.get("BSQ_LIBRARY") or os.path.join(_HERE, "libbsq.so")

if not os.path.exists(lib_path):
    raise ImportError(f"libbsq is not built at {lib_path}; run "
                      "`python -m fp8_microscaling_quantization_b200.build` (nvcc, sm_100a)")

_L = ctypes.CDLL(lib_path)


class DType(enum.IntEnum):
    BF16 = 0
    FP32 = 1


class Format(enum.IntEnum):
    FP8 = 0
    MXFP4 = 1
    NVFP4 = 2
    MXFP8 = 3


class Direction(enum.IntEnum):
    FWD = 0
    BWD = 1


DEVERR_BAD_OFFS = 1
DEVERR_TIMEOUT = 2


class BsqError(RuntimeError):
    def __init__(self, fn, status, msg):
        super().__init__(f"{fn}: {_status_string(status)} ({status}): {msg}")
        self.status = status


_P, _I64, _I32, _SZ = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_size_t
_SIGS = {
    "bsq_status_string": (ctypes.c_char_p, [_I32]),
    "bsq_last_error": (ctypes.c_char_p, []),
    "bsq_version": (_I32, []),
    "bsq_debug_counters": (_I32, [_P, _P]),
    "bsq_quantize_nvfp4": (_I32, [_P, _I32, _I64, _I64, _P, _P, _P, _P, _P]),
    "bsq_nvfp4_tensor_scratch_bytes": (_SZ, [_I64, _I64]),
    "bsq_quantize_nvfp4_tensor": (_I32, [_P, _I32, _I64, _I64, _P, _P, _P, _P, _SZ, _P]),
    "bsq_quantize_nvfp4_tensor_noalloc": (_I32, [_P, _I32, _I64, _I64, _P, _P, _P, _P]),
    "bsq_dequantize_nvfp4": (_I32, [_P, _P, _P, _I64, _I64, _P, _I32, _P]),
    "bsq_quantize_mxfp4": (_I32, [_P, _I32, _I64, _I64, _P, _P, _P]),
    "bsq_dequantize_mxfp4": (_I32, [_P, _P, _I64, _I64, _P, _I32, _P]),
    "bsq_fake_quantize_nvfp4_static": (_I32, [_P, _I32, _I64, _I64, _P, _P, _P, _P]),
    "bsq_dequantize_kv_cache_nvfp4": (_I32, [_P, _P, _P, _I64, _I64, _I64, _P, _I32, _P]),
    "bsq_quantize_mxfp8": (_I32, [_P, _I32, _I64, _I64, _P, _P, _P]),
    "bsq_dequantize_mxfp8": (_I32, [_P, _P, _I64, _I64, _P, _I32, _P]),
    "bsq_quantize_fp8": (_I32, [_P, _I32, _I64, _I64, _I32, _P, _P, _P]),
    "bsq_dequantize_fp8": (_I32, [_P, _P, _I64, _I64, _I32, _P, _I32, _P]),
    "bsq_quantize_cache": (_I32, [_I32, _I32, _P, _P, _I32, _I64, _I64, _P]),
    "bsq_quantize_cache_backward": (_I32, [_P, _P, _I32, _I64, _P]),
    "bsq_grouped_mm_fp4": (_I32, [_I32, _I32, _P, _P, _P, _P, _P, _I32, _I64, _I64, _I64, _P, _P, _P]),
}
for _name, (_res, _args) in _SIGS.items():
    _fn = getattr(_L, _name)
    _fn.restype = _res
    _fn.argtypes = _args

EXPORTED = tuple(_SIGS)


def _status_string(s):
    return _L.bsq_status_string(int(s)).decode()


def bsq_status_string(s) -> str:
    return _status_string(s)


def bsq_last_error() -> str:
    return _L.bsq_last_error().decode()


def bsq_version() -> int:
    return _L.bsq_version()


def bsq_debug_counters():
    """(failed index checks, code of the first) since the last call, in a
    BSQ_DEBUG build; raises BsqError (unsupported) in a normal build."""
    c, f = ctypes.c_uint32(0), ctypes.c_uint32(0)
    _call("bsq_debug_counters", ctypes.byref(c), ctypes.byref(f))
    return int(c.value), int(f.value)


def _call(name, *args):
    rc = getattr(_L, name)(*args)
    if rc != 0:
        raise BsqError(name, rc, bsq_last_error())


def _ptr(t):
    if t is None:
        return None
    if not isinstance(t, torch.Tensor):
        return int(t)  # raw device address
    if t.numel() and not t.is_cuda:
        raise ValueError("libbsq takes device tensors")
    if not t.is_contiguous():
        raise ValueError("libbsq takes contiguous tensors")
    return t.data_ptr() if t.numel() else None


def _stream(stream):
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _dtype_of(t) -> DType:
    if t.dtype in (torch.bfloat16, torch.int16, torch.uint16):
        return DType.BF16
    if t.dtype == torch.float32:
        return DType.FP32
    raise TypeError(f"libbsq tensors are bf16 or fp32, got {t.dtype}")


def _torch_dtype(dt: DType):
    return torch.bfloat16 if dt == DType.BF16 else torch.float32


def _rows_k(x):
    K = x.shape[-1] if x.dim() else 1
    rows = x.numel() // K if K else 0
    return rows, K


def _empty(shape, dtype, like):
    return torch.empty(shape, dtype=dtype, device=like.device)


# ------------------------------------------------------------------ NVFP4 ---

def bsq_quantize_nvfp4(x, row_scale_in=None, packed=None, scales=None, row_scale_out=None, stream=None):
    """-> (packed uint8 [..., K/2], scales e4m3 as uint8 [..., K/16], row scale fp32 [...])."""
    rows, K = _rows_k(x)
    lead = tuple(x.shape[:-1])
    packed = _empty(lead + (K // 2,), torch.uint8, x) if packed is None else packed
    scales = _empty(lead + (K // 16,), torch.uint8, x) if scales is None else scales
    row_scale_out = _empty(lead, torch.float32, x) if row_scale_out is None else row_scale_out
    _call("bsq_quantize_nvfp4", _ptr(x), _dtype_of(x), rows, K, _ptr(row_scale_in), _ptr(packed), _ptr(scales),
          _ptr(row_scale_out), _stream(stream))
    return packed, scales, row_scale_out


def bsq_nvfp4_tensor_scratch_bytes(rows, K) -> int:
    return _L.bsq_nvfp4_tensor_scratch_bytes(rows, K)


def bsq_quantize_nvfp4_tensor(x, packed=None, scales=None, tensor_scale=None, scratch=None, stream=None):
    """ModelOpt layout -> (packed [out, in/2], scales [out, in/16], tensor scale fp32 [1])."""
    rows, K = _rows_k(x)
    lead = tuple(x.shape[:-1])
    packed = _empty(lead + (K // 2,), torch.uint8, x) if packed is None else packed
    scales = _empty(lead + (K // 16,), torch.uint8, x) if scales is None else scales
    tensor_scale = _empty((1,), torch.float32, x) if tensor_scale is None else tensor_scale
    nbytes = bsq_nvfp4_tensor_scratch_bytes(rows, K)
    if scratch is None:
        scratch = _empty((nbytes,), torch.uint8, x)
    _call("bsq_quantize_nvfp4_tensor", _ptr(x), _dtype_of(x), rows, K, _ptr(packed), _ptr(scales),
          _ptr(tensor_scale), _ptr(scratch), scratch.numel() * scratch.element_size(), _stream(stream))
    return packed, scales, tensor_scale


def bsq_quantize_nvfp4_tensor_noalloc(x, packed=None, scales=None, tensor_scale=None, stream=None):
    """bsq_quantize_nvfp4_tensor without a scratch buffer (the library's own
    device array holds the partial maxima; see include/bsq.h for the limits)."""
    rows, K = _rows_k(x)
    lead = tuple(x.shape[:-1])
    packed = _empty(lead + (K // 2,), torch.uint8, x) if packed is None else packed
    scales = _empty(lead + (K // 16,), torch.uint8, x) if scales is None else scales
    tensor_scale = _empty((1,), torch.float32, x) if tensor_scale is None else tensor_scale
    _call("bsq_quantize_nvfp4_tensor_noalloc", _ptr(x), _dtype_of(x), rows, K, _ptr(packed), _ptr(scales),
          _ptr(tensor_scale), _stream(stream))
    return packed, scales, tensor_scale


def bsq_dequantize_nvfp4(packed, scales, row_scale, out_dtype=DType.BF16, y=None, stream=None):
    rows, Kh = _rows_k(packed)
    K = Kh * 2
    y = _empty(tuple(packed.shape[:-1]) + (K,), _torch_dtype(out_dtype), packed) if y is None else y
    _call("bsq_dequantize_nvfp4", _ptr(packed), _ptr(scales), _ptr(row_scale), rows, K, _ptr(y), _dtype_of(y),
          _stream(stream))
    return y


# ------------------------------------------------------------------ MXFP4 ---

def bsq_quantize_mxfp4(x, packed=None, scales=None, stream=None):
    """-> (packed int8 bits as uint8 [..., K/2], scales e8m0 as uint8 [..., K/32])."""
    rows, K = _rows_k(x)
    lead = tuple(x.shape[:-1])
    packed = _empty(lead + (K // 2,), torch.uint8, x) if packed is None else packed
    scales = _empty(lead + (K // 32,), torch.uint8, x) if scales is None else scales
    _call("bsq_quantize_mxfp4", _ptr(x), _dtype_of(x), rows, K, _ptr(packed), _ptr(scales), _stream(stream))
    return packed, scales


def bsq_dequantize_mxfp4(packed, scales, out_dtype=DType.BF16, y=None, stream=None):
    rows, Kh = _rows_k(packed)
    K = Kh * 2
    y = _empty(tuple(packed.shape[:-1]) + (K,), _torch_dtype(out_dtype), packed) if y is None else y
    _call("bsq_dequantize_mxfp4", _ptr(packed), _ptr(scales), rows, K, _ptr(y), _dtype_of(y), _stream(stream))
    return y


# -------------------------------------------------------------------- FP8 ---

def kv_block_table(values, scales, amax, device=None):
    """Device arrays of the blocks' pointers for bsq_dequantize_kv_cache_nvfp4
    (lists of uint8 [rows, 64] codes, uint8 [rows, 8] scales and fp32 [1] amax
    tensors).  Build once per cache layout; the tensors must stay alive."""
    dev_ = device if device is not None else values[0].device
    def table(ts):
        return torch.tensor([t.data_ptr() for t in ts], dtype=torch.int64).to(dev_)
    return table(values), table(scales), table(amax)


def bsq_dequantize_kv_cache_nvfp4(table, nblocks, block_tokens, heads, out_dtype=DType.BF16, y=None, stream=None):
    """Dequantize a list-of-blocks NVFP4 KV cache into [1, nblocks * block_tokens,
    heads, 128]; `table` is the (values, scales, amax) pointer arrays of
    kv_block_table."""
    vt, st_, at = table
    if y is None:
        y = torch.empty((1, nblocks * block_tokens, heads, 128), dtype=_torch_dtype(out_dtype), device=vt.device)
    _call("bsq_dequantize_kv_cache_nvfp4", _ptr(vt), _ptr(st_), _ptr(at), int(nblocks), int(block_tokens), int(heads),
          _ptr(y), _dtype_of(y), _stream(stream))
    return y


def bsq_fake_quantize_nvfp4_static(x, block_amax, global_amax, y=None, stream=None):
    """Static two-level NVFP4 fake-quant: block_amax fp32 [..., K/16] and
    global_amax fp32 [1] on the device; returns y (x's dtype; y may be x)."""
    rows, K = _rows_k(x)
    y = torch.empty_like(x) if y is None else y
    _call("bsq_fake_quantize_nvfp4_static", _ptr(x), _dtype_of(x), rows, K, _ptr(block_amax), _ptr(global_amax),
          _ptr(y), _stream(stream))
    return y


def bsq_quantize_mxfp8(x, codes=None, scales=None, stream=None):
    rows, K = _rows_k(x)
    lead = tuple(x.shape[:-1])
    codes = _empty(tuple(x.shape), torch.uint8, x) if codes is None else codes
    scales = _empty(lead + (K // 32,), torch.uint8, x) if scales is None else scales
    _call("bsq_quantize_mxfp8", _ptr(x), _dtype_of(x), rows, K, _ptr(codes), _ptr(scales), _stream(stream))
    return codes, scales


def bsq_dequantize_mxfp8(codes, scales, out_dtype=DType.BF16, y=None, stream=None):
    rows, K = _rows_k(codes)
    y = _empty(tuple(codes.shape), _torch_dtype(out_dtype), codes) if y is None else y
    _call("bsq_dequantize_mxfp8", _ptr(codes), _ptr(scales), rows, K, _ptr(y), _dtype_of(y), _stream(stream))
    return y


def bsq_quantize_fp8(x, block=32, codes=None, scales=None, stream=None):
    rows, K = _rows_k(x)
    lead = tuple(x.shape[:-1])
    codes = _empty(tuple(x.shape), torch.uint8, x) if codes is None else codes
    scales = _empty(lead + (K // block,), torch.uint8, x) if scales is None else scales
    _call("bsq_quantize_fp8", _ptr(x), _dtype_of(x), rows, K, int(block), _ptr(codes), _ptr(scales),
          _stream(stream))
    return codes, scales


def bsq_dequantize_fp8(codes, scales, block=32, out_dtype=DType.BF16, y=None, stream=None):
    rows, K = _rows_k(codes)
    y = _empty(tuple(codes.shape), _torch_dtype(out_dtype), codes) if y is None else y
    _call("bsq_dequantize_fp8", _ptr(codes), _ptr(scales), rows, K, int(block), _ptr(y), _dtype_of(y),
          _stream(stream))
    return y


# ---------------------------------------------------------- quantize_cache ---

def bsq_quantize_cache(x, fmt, block, y=None, stream=None):
    rows, C = _rows_k(x)
    y = torch.empty_like(x) if y is None else y
    _call("bsq_quantize_cache", int(fmt), int(block), _ptr(x), _ptr(y), _dtype_of(x), rows, C, _stream(stream))
    return y


def bsq_quantize_cache_backward(grad_out, grad_in=None, stream=None):
    if grad_in is None:
        grad_in = grad_out
    _call("bsq_quantize_cache_backward", _ptr(grad_out), _ptr(grad_in), _dtype_of(grad_out), grad_out.numel(),
          _stream(stream))
    return grad_in


# ------------------------------------------------------------ grouped GEMM ---

def bsq_grouped_mm_fp4(fmt, direction, a, packed, scales, row_scale, offs, out=None, err=None, stream=None):
    """Fused-dequant grouped GEMM.  a: bf16 [T, K] (FWD) or [T, N] (BWD);
    packed uint8 [E, N, K/2]; offs int32 [E] on the device.  Returns (out, err)
    where err is the device error word (uint32 bits as int32 tensor [1])."""
    E, N, Kh = packed.shape
    K = Kh * 2
    T = a.shape[0]
    width = N if int(direction) == Direction.FWD else K
    out = _empty((T, width), torch.bfloat16, a) if out is None else out
    if err is None:
        err = torch.zeros((1,), dtype=torch.int32, device=a.device)
    _call("bsq_grouped_mm_fp4", int(fmt), int(direction), _ptr(a), _ptr(packed), _ptr(scales), _ptr(row_scale),
          _ptr(offs), E, T, N, K, _ptr(out), _ptr(err), _stream(stream))
    return out, err


__all__ = [n for n in dir() if n.startswith("bsq_")] + ["BsqError", "DType", "Format", "Direction", "lib_path",
                                                       "EXPORTED"]
