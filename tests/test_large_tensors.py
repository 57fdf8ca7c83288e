"""Tensors of more than 2**31 elements, so that every 64-bit element and
byte offset in the kernels is exercised: MXFP4 and NVFP4 quantize and
dequantize, and the FP8 cache fake-quant, compared with the oracle on the
rows around the 2**31-element mark and at both ends."""
import numpy as np
import pytest
import torch

from gpu_util import assert_bits_equal, host_bits

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def B():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from fp8_microscaling_quantization_b200 import bsq
    return bsq

N31 = 1 << 31


def sample_rows(rows, K):
    r = N31 // K
    return sorted({0, 1, r - 1, r, r + 1, rows // 2, rows - 2, rows - 1})


def bits_of(t):
    return host_bits(t.contiguous())


def test_mxfp4_past_2_31_elements(B, oracle):
    rows, K = 262144, 8448          # 2.21e9 elements
    g = torch.Generator(device="cuda").manual_seed(31)
    x = (torch.randn((rows, K), generator=g, device="cuda") * 0.02).to(torch.bfloat16)
    p, s = B.bsq_quantize_mxfp4(x)
    y = B.bsq_dequantize_mxfp4(p, s)
    torch.cuda.synchronize()
    idx = sample_rows(rows, K)
    xr = bits_of(x[idx])
    op, os_ = oracle.quantize_mxfp4(xr)
    assert_bits_equal(host_bits(p[idx].contiguous()), op, "packed")
    assert_bits_equal(host_bits(s[idx].contiguous()), os_, "scales")
    assert_bits_equal(bits_of(y[idx]), oracle.dequantize_mxfp4(op, os_), "dequant bf16")


def test_nvfp4_per_row_past_2_31_elements(B, oracle):
    rows, K = 131072, 16416         # 2.15e9 elements, staged rows
    g = torch.Generator(device="cuda").manual_seed(32)
    x = (torch.randn((rows, K), generator=g, device="cuda") * 0.01).to(torch.bfloat16)
    p, s, rs = B.bsq_quantize_nvfp4(x)
    y = B.bsq_dequantize_nvfp4(p, s, rs)
    torch.cuda.synchronize()
    idx = sample_rows(rows, K)
    xr = bits_of(x[idx])
    op, os_, og = oracle.quantize_nvfp4(xr)
    assert_bits_equal(host_bits(rs[idx].contiguous()), og, "row scale")
    assert_bits_equal(host_bits(s[idx].contiguous()), os_, "e4m3 scales")
    assert_bits_equal(host_bits(p[idx].contiguous()), op, "packed")
    assert_bits_equal(bits_of(y[idx]), oracle.dequantize_nvfp4(op, os_, og), "dequant bf16")


def test_cache_fp8_past_2_31_elements(B, oracle):
    rows, C = 4194816, 512          # 2.15e9 elements
    g = torch.Generator(device="cuda").manual_seed(33)
    x = torch.randn((rows, C), generator=g, device="cuda").to(torch.bfloat16)
    y = B.bsq_quantize_cache(x, B.Format.FP8, 32)
    torch.cuda.synchronize()
    idx = sample_rows(rows, C)
    want = oracle.quantize_cache(bits_of(x[idx]), oracle.FMT_FP8, 32)
    assert_bits_equal(bits_of(y[idx]), want, "fake-quant")
