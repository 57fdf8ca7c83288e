"""CPU oracle for block-scaled microscaling quantization (test infrastructure).

TEST INFRASTRUCTURE ONLY: the test suite, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` are the only callers.  The product path (the
CUDA library and its Python binding) never imports this package, and this
package never imports the product.

The scalar rules live in ``bsq_oracle.c`` (plain C, one element at a time,
binary32 round-to-nearest-even, built with ``-O2 -ffp-contract=off``).  This
module wraps it with ctypes and adds the grouped-GEMM reference, which is the
textbook product in float64 of the activations and the oracle's binary32
dequantized weights (NeMo AutoModel ``NVFP4GroupedMM`` / ``MXFP4GroupedMM``:
expert ``e`` owns rows ``[offs[e-1], offs[e])`` and computes ``x @ W_e^T`` in
forward and ``grad_out @ W_e`` in backward).

Inputs and outputs are numpy arrays; bf16 tensors travel as ``uint16`` bit
patterns.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "bsq_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")

BF16, F32 = 0, 1
FMT_FP8, FMT_MXFP4, FMT_NVFP4 = 0, 1, 2

_lib = None


def build(force: bool = False) -> str:
    """Compile bsq_oracle.c into liboracle.so next to it (gcc, no fast-math)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared",
                               "-Wall", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB_PATH)
        P, I64, I32, F = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_float
        sig = {
            "o_bf16_to_f32": (F, [ctypes.c_uint16]),
            "o_f32_to_bf16": (ctypes.c_uint16, [F]),
            "o_e2m1_val": (F, [I32]),
            "o_e2m1_round": (I32, [F]),
            "o_e4m3_val": (F, [I32]),
            "o_e4m3_round": (I32, [F]),
            "o_e8m0_val": (F, [I32]),
            "o_floor_log2": (I32, [F]),
            "o_pow2_ceil": (F, [F]),
            "o_quantize_nvfp4": (I32, [P, I32, I64, I64, P, P, P, P]),
            "o_quantize_nvfp4_tensor": (I32, [P, I32, I64, I64, P, P, P]),
            "o_dequantize_nvfp4": (I32, [P, P, P, I64, I64, P, I32]),
            "o_quantize_mxfp4": (I32, [P, I32, I64, I64, P, P]),
            "o_dequantize_mxfp4": (I32, [P, P, I64, I64, P, I32]),
            "o_fake_quantize_nvfp4_static": (I32, [P, I32, I64, I64, P, F, P]),
            "o_dequantize_kv_cache_nvfp4": (I32, [P, P, P, I64, I64, I64, P, I32]),
            "o_nvfp4_static_scale": (None, [F, F, P, P]),
            "o_quantize_mxfp8": (I32, [P, I32, I64, I64, P, P]),
            "o_dequantize_mxfp8": (I32, [P, P, I64, I64, P, I32]),
            "o_quantize_fp8": (I32, [P, I32, I64, I64, I32, P, P]),
            "o_dequantize_fp8": (I32, [P, P, I64, I64, I32, P, I32]),
            "o_quantize_cache": (I32, [I32, I32, P, P, I32, I64, I64]),
            "o_quantize_cache_backward": (I32, [P, P, I32, I64]),
            "o_e2m1_round_array": (None, [P, P, I64]),
            "o_e4m3_round_array": (None, [P, P, I64]),
            "o_f32_to_bf16_array": (None, [P, P, I64]),
            "o_pow2_ceil_array": (None, [P, P, I64]),
            "o_floor_log2_array": (None, [P, P, I64]),
        }
        for name, (res, args) in sig.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def _p(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be contiguous"
    return a.ctypes.data_as(ctypes.c_void_p)


def _dt(x: np.ndarray) -> int:
    if x.dtype == np.uint16:
        return BF16
    if x.dtype == np.float32:
        return F32
    raise TypeError(f"oracle input must be bf16 bits (uint16) or float32, got {x.dtype}")


def _out(shape, dt: int):
    return np.empty(shape, dtype=np.uint16 if dt == BF16 else np.float32)


def _check(rc: int, what: str):
    if rc != 0:
        raise ValueError(f"oracle {what}: rejected arguments (rc={rc})")


# ---------------------------------------------------------------- scalars ---

def bf16_to_f32(bits: np.ndarray) -> np.ndarray:
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def f32_to_bf16(x: np.ndarray) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float32)
    out = np.empty(x.shape, dtype=np.uint16)
    lib().o_f32_to_bf16_array(_p(x), _p(out), x.size)
    return out


def e2m1_round(q: np.ndarray) -> np.ndarray:
    q = np.ascontiguousarray(q, dtype=np.float32)
    out = np.empty(q.shape, dtype=np.uint8)
    lib().o_e2m1_round_array(_p(q), _p(out), q.size)
    return out


def e4m3_round(x: np.ndarray) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float32)
    out = np.empty(x.shape, dtype=np.uint8)
    lib().o_e4m3_round_array(_p(x), _p(out), x.size)
    return out


def pow2_ceil(x: np.ndarray) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float32)
    out = np.empty(x.shape, dtype=np.float32)
    lib().o_pow2_ceil_array(_p(x), _p(out), x.size)
    return out


def floor_log2(x: np.ndarray) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float32)
    out = np.empty(x.shape, dtype=np.int32)
    lib().o_floor_log2_array(_p(x), _p(out), x.size)
    return out


def e2m1_val(code: int) -> float:
    return lib().o_e2m1_val(int(code))


def e4m3_val(code: int) -> float:
    return lib().o_e4m3_val(int(code))


def e8m0_val(code: int) -> float:
    return lib().o_e8m0_val(int(code))


# ---------------------------------------------------------------- tensors ---

def quantize_nvfp4(x: np.ndarray, row_scale: np.ndarray | None = None):
    """NVFP4 along the last dim; returns (packed uint8 [...,K/2], e4m3 [...,K/16], fp32 [...])."""
    x = np.ascontiguousarray(x)
    K = x.shape[-1]
    rows = x.size // K if K else 0
    lead = x.shape[:-1]
    packed = np.zeros(lead + (K // 2,), np.uint8)
    scales = np.zeros(lead + (K // 16,), np.uint8)
    g = np.zeros(lead, np.float32)
    gin = None
    if row_scale is not None:
        gin = np.ascontiguousarray(np.broadcast_to(row_scale, lead), dtype=np.float32)
    rc = lib().o_quantize_nvfp4(_p(x), _dt(x), rows, K, _p(gin) if gin is not None else None,
                                _p(packed), _p(scales), _p(g))
    _check(rc, "quantize_nvfp4")
    return packed, scales, g


def quantize_nvfp4_tensor(x: np.ndarray):
    """ModelOpt layout: one tensor scale; returns (packed, e4m3 scales, fp32 scalar)."""
    x = np.ascontiguousarray(x)
    K = x.shape[-1]
    rows = x.size // K if K else 0
    packed = np.zeros(x.shape[:-1] + (K // 2,), np.uint8)
    scales = np.zeros(x.shape[:-1] + (K // 16,), np.uint8)
    g = np.zeros(1, np.float32)
    _check(lib().o_quantize_nvfp4_tensor(_p(x), _dt(x), rows, K, _p(packed), _p(scales), _p(g)),
           "quantize_nvfp4_tensor")
    return packed, scales, g[0]


def dequantize_nvfp4(packed, scales, row_scale, out_dtype=BF16):
    packed = np.ascontiguousarray(packed, dtype=np.uint8)
    scales = np.ascontiguousarray(scales, dtype=np.uint8)
    K = packed.shape[-1] * 2
    lead = packed.shape[:-1]
    rows = int(np.prod(lead)) if lead else 1
    g = np.ascontiguousarray(np.broadcast_to(np.asarray(row_scale, np.float32), lead), dtype=np.float32)
    y = _out(lead + (K,), out_dtype)
    _check(lib().o_dequantize_nvfp4(_p(packed), _p(scales), _p(g), rows, K, _p(y), out_dtype),
           "dequantize_nvfp4")
    return y


def quantize_mxfp4(x: np.ndarray):
    x = np.ascontiguousarray(x)
    K = x.shape[-1]
    rows = x.size // K if K else 0
    packed = np.zeros(x.shape[:-1] + (K // 2,), np.uint8)
    scales = np.zeros(x.shape[:-1] + (K // 32,), np.uint8)
    _check(lib().o_quantize_mxfp4(_p(x), _dt(x), rows, K, _p(packed), _p(scales)), "quantize_mxfp4")
    return packed, scales


def dequantize_mxfp4(packed, scales, out_dtype=BF16):
    packed = np.ascontiguousarray(packed).view(np.uint8)
    scales = np.ascontiguousarray(scales, dtype=np.uint8)
    K = packed.shape[-1] * 2
    lead = packed.shape[:-1]
    rows = int(np.prod(lead)) if lead else 1
    y = _out(lead + (K,), out_dtype)
    _check(lib().o_dequantize_mxfp4(_p(packed), _p(scales), rows, K, _p(y), out_dtype), "dequantize_mxfp4")
    return y


def dequantize_kv_cache_nvfp4(values, scales, amax, block_tokens: int, heads: int, out_dtype=BF16):
    """List-of-blocks NVFP4 KV cache -> [1, nblocks * block_tokens, heads, 128].
    values[b] uint8 [block_tokens * heads, 64], scales[b] uint8 [.., 8],
    amax float32 [nblocks] (one per block)."""
    nb = len(values)
    rows = block_tokens * heads
    vals = [np.ascontiguousarray(v, dtype=np.uint8) for v in values]
    scs = [np.ascontiguousarray(s_, dtype=np.uint8) for s_ in scales]
    for v, s_ in zip(vals, scs):
        assert v.shape == (rows, 64) and s_.shape == (rows, 8)
    vp = (ctypes.c_void_p * max(nb, 1))(*[v.ctypes.data for v in vals])
    sp = (ctypes.c_void_p * max(nb, 1))(*[s_.ctypes.data for s_ in scs])
    am = np.ascontiguousarray(amax, dtype=np.float32)
    y = _out((1, nb * block_tokens, heads, 128), out_dtype)
    _check(lib().o_dequantize_kv_cache_nvfp4(vp, sp, _p(am), nb, block_tokens, heads, _p(y), out_dtype),
           "dequantize_kv_cache_nvfp4")
    return y


def fake_quantize_nvfp4_static(x: np.ndarray, block_amax: np.ndarray, global_amax: float):
    """Static two-level NVFP4 fake-quant along the last dim (K % 16 == 0) with
    calibrated per-16-block amax [..., K/16] and a global amax; same dtype as x."""
    x = np.ascontiguousarray(x)
    K = x.shape[-1]
    rows = x.size // K if K else 0
    a = np.ascontiguousarray(block_amax, dtype=np.float32)
    assert a.size == rows * (K // 16), "one amax per 16-block"
    y = np.empty_like(x)
    _check(lib().o_fake_quantize_nvfp4_static(_p(x), _dt(x), rows, K, _p(a), float(global_amax), _p(y)),
           "fake_quantize_nvfp4_static")
    return y


def nvfp4_static_scale(amax_b: float, global_amax: float):
    """(physical block scale, e4m3 code) of one block of the static rule."""
    sq = ctypes.c_float()
    code = ctypes.c_int()
    lib().o_nvfp4_static_scale(float(amax_b), float(global_amax), ctypes.byref(sq), ctypes.byref(code))
    return sq.value, code.value


def quantize_mxfp8(x: np.ndarray):
    """MXFP8 along the last dim: e4m3 codes [..., K] and e8m0 scales [..., K/32]."""
    x = np.ascontiguousarray(x)
    K = x.shape[-1]
    rows = x.size // K if K else 0
    codes = np.zeros(x.shape, np.uint8)
    scales = np.zeros(x.shape[:-1] + (K // 32,), np.uint8)
    _check(lib().o_quantize_mxfp8(_p(x), _dt(x), rows, K, _p(codes), _p(scales)), "quantize_mxfp8")
    return codes, scales


def dequantize_mxfp8(codes, scales, out_dtype=BF16):
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    scales = np.ascontiguousarray(scales, dtype=np.uint8)
    K = codes.shape[-1]
    rows = codes.size // K if K else 0
    y = _out(codes.shape, out_dtype)
    _check(lib().o_dequantize_mxfp8(_p(codes), _p(scales), rows, K, _p(y), out_dtype), "dequantize_mxfp8")
    return y


def quantize_fp8(x: np.ndarray, block: int = 32):
    x = np.ascontiguousarray(x)
    K = x.shape[-1]
    rows = x.size // K if K else 0
    codes = np.zeros(x.shape, np.uint8)
    scales = np.zeros(x.shape[:-1] + (K // block,), np.uint8)
    _check(lib().o_quantize_fp8(_p(x), _dt(x), rows, K, block, _p(codes), _p(scales)), "quantize_fp8")
    return codes, scales


def dequantize_fp8(codes, scales, block: int = 32, out_dtype=BF16):
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    scales = np.ascontiguousarray(scales, dtype=np.uint8)
    K = codes.shape[-1]
    rows = codes.size // K if K else 0
    y = _out(codes.shape, out_dtype)
    _check(lib().o_dequantize_fp8(_p(codes), _p(scales), rows, K, block, _p(y), out_dtype), "dequantize_fp8")
    return y


def quantize_cache(x: np.ndarray, fmt: int, block: int):
    """Fake-quant (quantize then dequantize) along the last dim; same dtype as x."""
    x = np.ascontiguousarray(x)
    C = x.shape[-1]
    rows = x.size // C if C else 0
    y = np.empty_like(x)
    _check(lib().o_quantize_cache(fmt, block, _p(x), _p(y), _dt(x), rows, C), "quantize_cache")
    return y


def quantize_cache_backward(grad_out: np.ndarray) -> np.ndarray:
    g = np.ascontiguousarray(grad_out)
    out = np.empty_like(g)
    lib().o_quantize_cache_backward(_p(g), _p(out), _dt(g), g.size)
    return out


# ------------------------------------------------------- grouped GEMM ref ---

def dequant_expert_f32(fmt: int, packed_e, scales_e, row_scale_e=None) -> np.ndarray:
    """Oracle binary32 dequantization of one expert's [N, K] weight."""
    if fmt == FMT_MXFP4:
        return dequantize_mxfp4(packed_e, scales_e, out_dtype=F32)
    if fmt == FMT_NVFP4:
        return dequantize_nvfp4(packed_e, scales_e, row_scale_e, out_dtype=F32)
    raise ValueError("grouped GEMM formats: MXFP4 or NVFP4")


def grouped_mm_rows(fmt: int, backward: bool, a_bits: np.ndarray, packed, scales, row_scale,
                    offs: np.ndarray, rows: np.ndarray) -> np.ndarray:
    """float64 reference rows of the grouped GEMM.

    forward:  out[t, :]    = x[t, :]        @ W_e^T   (a = x, [T, K])
    backward: grad_x[t, :] = grad_out[t, :] @ W_e     (a = grad_out, [T, N])
    for the expert e whose segment [offs[e-1], offs[e]) holds t; rows at or past
    offs[-1] are zero.  W_e is the oracle's binary32 dequantization (exact
    weights), the product is a library float64 matmul.
    """
    offs = np.asarray(offs, dtype=np.int64)
    rows = np.asarray(rows, dtype=np.int64)
    E, N, Kh = packed.shape
    K = Kh * 2
    width = K if backward else N
    out = np.zeros((rows.size, width), dtype=np.float64)
    starts = np.concatenate([[0], offs[:-1]])
    for e in range(E):
        sel = np.nonzero((rows >= starts[e]) & (rows < offs[e]))[0]
        if sel.size == 0:
            continue
        W = dequant_expert_f32(fmt, packed[e], scales[e], None if row_scale is None else row_scale[e])
        W = W.astype(np.float64)
        A = bf16_to_f32(a_bits[rows[sel]]).astype(np.float64)
        out[sel] = A @ W if backward else A @ W.T
    return out
