"""C-ABI boundary tests that need no GPU: the library loads, exports every
entry point include/bsq.h declares, and rejects bad arguments on the host
before launching anything."""
import ctypes
import os
import re

import pytest

from conftest import ROOT

HEADER = os.path.join(ROOT, "include", "bsq.h")


@pytest.fixture(scope="module")
def lib():
    from fp8_microscaling_quantization_b200 import build
    path = build.build()
    return ctypes.CDLL(path)


def declared_entry_points():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(bsq_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_hot_path():
    names = declared_entry_points()
    for n in ["bsq_quantize_nvfp4", "bsq_quantize_nvfp4_tensor", "bsq_dequantize_nvfp4", "bsq_quantize_mxfp4",
              "bsq_dequantize_mxfp4", "bsq_quantize_fp8", "bsq_dequantize_fp8", "bsq_quantize_cache",
              "bsq_quantize_cache_backward", "bsq_grouped_mm_fp4"]:
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    missing = [n for n in declared_entry_points() if not hasattr(lib, n)]
    assert not missing, missing


def test_binding_covers_every_entry_point():
    from fp8_microscaling_quantization_b200 import bsq
    assert set(declared_entry_points()) <= set(bsq.EXPORTED)
    for n in declared_entry_points():
        assert callable(getattr(bsq, n))


def test_status_strings(lib):
    lib.bsq_status_string.restype = ctypes.c_char_p
    assert lib.bsq_status_string(0) == b"ok"
    assert lib.bsq_status_string(1) == b"invalid argument"
    assert lib.bsq_version() >= 1


# --- host-side validation (nothing is launched for a rejected call) --------

FAKE = ctypes.c_void_p(0x10000)  # never dereferenced: every call below is rejected first
I64 = ctypes.c_int64
INVALID, UNSUPPORTED = 1, 2


def _err(lib):
    lib.bsq_last_error.restype = ctypes.c_char_p
    return lib.bsq_last_error().decode()


def test_nvfp4_rejects_ragged_k(lib):
    rc = lib.bsq_quantize_nvfp4(FAKE, 0, I64(4), I64(24), None, FAKE, FAKE, FAKE, None)
    assert rc == INVALID and "16-column blocks" in _err(lib)


def test_mxfp4_rejects_ragged_k(lib):
    assert lib.bsq_quantize_mxfp4(FAKE, 0, I64(4), I64(48), FAKE, FAKE, None) == INVALID
    assert lib.bsq_dequantize_mxfp4(FAKE, FAKE, I64(4), I64(48), FAKE, 0, None) == INVALID


def test_rejects_null_and_negative(lib):
    assert lib.bsq_quantize_nvfp4(None, 0, I64(4), I64(32), None, FAKE, FAKE, FAKE, None) == INVALID
    assert lib.bsq_quantize_nvfp4(FAKE, 0, I64(4), I64(32), None, None, FAKE, FAKE, None) == INVALID
    assert lib.bsq_quantize_mxfp4(FAKE, 0, I64(-1), I64(32), FAKE, FAKE, None) == INVALID
    assert lib.bsq_dequantize_nvfp4(FAKE, None, FAKE, I64(4), I64(32), FAKE, 0, None) == INVALID


def test_rejects_bad_dtype_format_block(lib):
    assert lib.bsq_quantize_mxfp4(FAKE, 7, I64(4), I64(32), FAKE, FAKE, None) == UNSUPPORTED
    assert lib.bsq_quantize_fp8(FAKE, 0, I64(4), I64(64), 8, FAKE, FAKE, None) == INVALID
    assert lib.bsq_quantize_cache(9, 16, FAKE, ctypes.c_void_p(0x90000), 0, I64(4), I64(64), None) == UNSUPPORTED
    assert lib.bsq_quantize_cache(0, 24, FAKE, ctypes.c_void_p(0x90000), 0, I64(4), I64(64), None) == INVALID


def test_cache_rejects_overlap(lib):
    rc = lib.bsq_quantize_cache(0, 32, FAKE, ctypes.c_void_p(0x10000 + 64), 0, I64(4), I64(64), None)
    assert rc == INVALID and "overlap" in _err(lib)


def test_misaligned_pointers_rejected(lib):
    rc = lib.bsq_quantize_mxfp4(ctypes.c_void_p(0x10002), 0, I64(4), I64(32), FAKE, FAKE, None)
    assert rc == INVALID and "misaligned" in _err(lib)


def test_empty_tensors_are_no_ops(lib):
    # zero rows: nothing to do, nothing launched, OK even with null pointers
    assert lib.bsq_quantize_mxfp4(None, 0, I64(0), I64(32), None, None, None) == 0
    assert lib.bsq_dequantize_fp8(None, None, I64(0), I64(64), 32, None, 0, None) == 0
    assert lib.bsq_quantize_cache(1, 32, None, None, 0, I64(0), I64(520), None) == 0
    assert lib.bsq_quantize_cache_backward(FAKE, FAKE, 0, I64(100), None) == 0  # aliased: identity, no copy


def test_tensor_scratch_size(lib):
    lib.bsq_nvfp4_tensor_scratch_bytes.restype = ctypes.c_size_t
    n = lib.bsq_nvfp4_tensor_scratch_bytes(I64(7168), I64(18432))
    assert n >= 4 and n % 16 == 0
    rc = lib.bsq_quantize_nvfp4_tensor(FAKE, 0, I64(7168), I64(18432), FAKE, FAKE, FAKE, FAKE,
                                       ctypes.c_size_t(0), None)
    assert rc == INVALID and "scratch" in _err(lib)


def test_kv_cache_host_checks(lib):
    P = ctypes.c_void_p
    # no blocks (or an empty block shape): nothing to do, even with null pointers
    assert lib.bsq_dequantize_kv_cache_nvfp4(None, None, None, I64(0), I64(64), I64(8), None, 0, None) == 0
    assert lib.bsq_dequantize_kv_cache_nvfp4(None, None, None, I64(4), I64(0), I64(8), None, 0, None) == 0
    assert lib.bsq_dequantize_kv_cache_nvfp4(FAKE, FAKE, FAKE, I64(-1), I64(64), I64(8), FAKE, 0, None) == INVALID
    assert lib.bsq_dequantize_kv_cache_nvfp4(FAKE, None, FAKE, I64(4), I64(64), I64(8), FAKE, 0, None) == INVALID
    # the pointer arrays hold 8-byte pointers; the output takes 16-byte stores
    assert lib.bsq_dequantize_kv_cache_nvfp4(P(0x10004), FAKE, FAKE, I64(4), I64(64), I64(8), FAKE, 0,
                                             None) == INVALID
    rc = lib.bsq_dequantize_kv_cache_nvfp4(FAKE, FAKE, FAKE, I64(4), I64(64), I64(8), P(0x10008), 0, None)
    assert rc == INVALID and "misaligned" in _err(lib)
    # 2**33 outputs in one block: beyond the kernel's 32-bit in-block index
    rc = lib.bsq_dequantize_kv_cache_nvfp4(FAKE, FAKE, FAKE, I64(1), I64(1 << 25), I64(2), FAKE, 0, None)
    assert rc == UNSUPPORTED and "2**32" in _err(lib)
    assert lib.bsq_dequantize_kv_cache_nvfp4(FAKE, FAKE, FAKE, I64(4), I64(64), I64(8), FAKE, 5, None) == UNSUPPORTED


def test_static_fake_quant_host_checks(lib):
    P = ctypes.c_void_p
    f = lib.bsq_fake_quantize_nvfp4_static
    assert f(FAKE, 0, I64(4), I64(24), FAKE, FAKE, P(0x90000), None) == INVALID  # K not a multiple of 16
    assert f(None, 0, I64(0), I64(32), None, None, None, None) == 0  # empty
    assert f(FAKE, 0, I64(4), I64(32), None, FAKE, P(0x90000), None) == INVALID  # no block amax
    assert f(FAKE, 0, I64(4), I64(32), FAKE, FAKE, P(0x90008), None) == INVALID  # misaligned output
    rc = f(FAKE, 0, I64(4), I64(32), FAKE, FAKE, P(0x10000 + 32), None)  # partial overlap (in place is fine)
    assert rc == INVALID and "overlap" in _err(lib)


def test_mxfp8_host_checks(lib):
    assert lib.bsq_quantize_mxfp8(FAKE, 0, I64(4), I64(48), FAKE, FAKE, None) == INVALID  # K % 32
    assert lib.bsq_dequantize_mxfp8(FAKE, FAKE, I64(4), I64(48), FAKE, 0, None) == INVALID
    assert lib.bsq_quantize_mxfp8(None, 0, I64(0), I64(64), None, None, None) == 0


def test_grouped_mm_host_checks(lib):
    g = lib.bsq_grouped_mm_fp4
    MX, NV, FWD, BWD = 1, 2, 0, 1
    args = lambda fmt, d, E, T, N, K, err=FAKE, rs=FAKE: (fmt, d, FAKE, FAKE, FAKE, rs, FAKE, E, I64(T), I64(N),
                                                          I64(K), FAKE, err, None)
    assert g(*args(0, FWD, 4, 256, 256, 256)) == UNSUPPORTED  # FP8 weights are not a GEMM format here
    assert g(*args(MX, 7, 4, 256, 256, 256)) == INVALID  # direction
    assert g(*args(MX, FWD, 0, 256, 256, 256)) == INVALID  # no experts
    assert g(*args(MX, FWD, 4, 256, 256, 200)) == UNSUPPORTED  # K not a multiple of 64
    assert g(*args(MX, FWD, 4, 256, 256, 256, err=None)) == INVALID  # the error word is required
    assert g(*args(NV, FWD, 4, 256, 256, 256, rs=None)) == INVALID  # NVFP4 needs its row scales
    assert g(*args(MX, FWD, 4, 0, 256, 256)) == 0  # no tokens: nothing to do


def test_debug_counters_in_the_normal_build(lib):
    """The index-check counters exist only in the bounds-checking build; the
    normal library answers that it is not one (no CUDA call is made)."""
    c, f = ctypes.c_uint32(7), ctypes.c_uint32(7)
    lib.bsq_debug_counters.restype = ctypes.c_int
    assert lib.bsq_debug_counters(ctypes.byref(c), ctypes.byref(f)) == UNSUPPORTED
    assert c.value == 0 and f.value == 0


def test_debug_build_exports_the_same_symbols():
    from fp8_microscaling_quantization_b200 import build
    dbg = ctypes.CDLL(build.build(debug=True))
    missing = [n for n in declared_entry_points() if not hasattr(dbg, n)]
    assert not missing, missing


def test_tensors_past_the_size_limit_are_rejected(lib):
    """Up to 2**35 elements per call (every chunk and block index then fits
    in 32 bits); larger shapes, including ones whose rows * K overflows
    int64, are rejected before anything is launched."""
    big = [(I64(1 << 20), I64(1 << 15)),            # exactly 2**35
           (I64(1 << 40), I64(1 << 40)),            # rows * K overflows int64
           (I64((1 << 62) // 32), I64(64))]
    for rows, K in big:
        assert lib.bsq_quantize_mxfp4(FAKE, 0, rows, K, FAKE, FAKE, None) == UNSUPPORTED
        assert lib.bsq_quantize_nvfp4(FAKE, 0, rows, K, None, FAKE, FAKE, FAKE, None) == UNSUPPORTED
        assert lib.bsq_dequantize_nvfp4(FAKE, FAKE, FAKE, rows, K, FAKE, 0, None) == UNSUPPORTED
        assert "too large" in _err(lib)
