"""GPU parity of the static two-level NVFP4 fake-quant against the CPU oracle:
bit-exact outputs, through the C ABI."""
import numpy as np
import pytest
import torch

from gpu_util import assert_bits_equal, dev, dev_bf16, host_bits

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def B():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from fp8_microscaling_quantization_b200 import bsq
    return bsq


@pytest.fixture(scope="module")
def S():
    from fp8_microscaling_quantization_b200 import synth
    return synth


def f32_of(bits):
    return (bits.astype(np.uint32) << 16).view(np.float32)


def calibrated_amax(xf, rng, spread=True):
    """Per-16-block amax as a calibration would leave it: the data's own, or
    scaled by 0.5 / 1 / 2 per block (saturating or under-using the range)."""
    a = np.abs(xf.reshape(-1, 16)).max(axis=1).astype(np.float32)
    if spread:
        a = (a * rng.choice(np.array([0.5, 1.0, 2.0], np.float32), size=a.size)).astype(np.float32)
    return a


def run(B, x_host, amax, A, fp32=False, inplace=False):
    x = dev(x_host) if fp32 else dev_bf16(x_host)
    a = dev(np.ascontiguousarray(amax, np.float32))
    g = dev(np.array([A], np.float32))
    y = B.bsq_fake_quantize_nvfp4_static(x, a, g, y=x if inplace else None)
    torch.cuda.synchronize()
    return host_bits(y)


def test_static_full_size_linear_weight(B, S, oracle):
    """[7168, 18432] linear weight with calibrated block amax (0.5x / 1x / 2x of
    the data's) and the tensor amax as the global amax: every output."""
    x = S.linear_weight()
    xf = f32_of(x)
    rng = np.random.default_rng(61)
    amax = calibrated_amax(xf, rng)
    A = np.float32(np.abs(xf).max())
    got = run(B, x, amax, A)
    assert_bits_equal(got, oracle.fake_quantize_nvfp4_static(x, amax, A), "static fake-quant bf16")


@pytest.mark.parametrize("rows,K", [(1, 16), (37, 272), (300, 4096), (5, 40000)])
def test_static_ragged_bf16_and_fp32(B, S, oracle, rows, K):
    x = S.nvfp4_matrix(rows=rows, cols=K, seed=rows * 13 + K)
    xf = f32_of(x)
    rng = np.random.default_rng(rows + K)
    amax = calibrated_amax(xf, rng)
    A = np.float32(np.abs(xf).max() * 0.75)
    assert_bits_equal(run(B, x, amax, A), oracle.fake_quantize_nvfp4_static(x, amax, A), "bf16")
    xs = (xf * np.exp(rng.uniform(-30, 30, (rows, 1))).astype(np.float32)).astype(np.float32)
    amax_s = calibrated_amax(xs, rng)
    As = np.float32(np.abs(xs).max())
    assert_bits_equal(run(B, xs, amax_s, As, fp32=True), oracle.fake_quantize_nvfp4_static(xs, amax_s, As), "fp32")


def test_static_edge_cases(B, oracle):
    """Zero and tiny block amax (the min_value floor), a zero global amax (the
    1e-8 floor), signed zeros and values far past the calibrated range."""
    rng = np.random.default_rng(62)
    x = (rng.standard_normal((64, 256)) * 3).astype(np.float32)
    x[0, :16] = 0.0
    x[1, :16] = -0.0
    x[2, :16] *= 1e6  # saturates against its calibrated amax
    amax = np.abs(x.reshape(-1, 16)).max(axis=1).astype(np.float32)
    amax[2 * 16] = 1.0
    amax[5:40] = 0.0
    amax[40:60] = 1e-30
    for A in (np.float32(0.0), np.float32(1e-9), np.float32(12.0), np.float32(3e7)):
        assert_bits_equal(run(B, x, amax, A, fp32=True), oracle.fake_quantize_nvfp4_static(x, amax, A),
                          f"fp32 A={A}")
        xb = oracle.f32_to_bf16(x)
        assert_bits_equal(run(B, xb, amax, A), oracle.fake_quantize_nvfp4_static(xb, amax, A), f"bf16 A={A}")


def test_static_in_place(B, S, oracle):
    x = S.nvfp4_matrix(rows=129, cols=1024, seed=63)
    xf = f32_of(x)
    amax = calibrated_amax(xf, np.random.default_rng(64))
    A = np.float32(np.abs(xf).max())
    assert_bits_equal(run(B, x, amax, A, inplace=True), oracle.fake_quantize_nvfp4_static(x, amax, A), "in place")


def test_static_rejects_bad_arguments(B):
    x = torch.zeros((4, 32), dtype=torch.bfloat16, device="cuda")
    a = torch.zeros((8,), dtype=torch.float32, device="cuda")
    g = torch.zeros((1,), dtype=torch.float32, device="cuda")
    with pytest.raises(B.BsqError):  # K not a multiple of 16
        B.bsq_fake_quantize_nvfp4_static(torch.zeros((4, 24), dtype=torch.bfloat16, device="cuda"), a, g)
    big = torch.zeros((8, 32), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(B.BsqError):  # partial overlap of x and y
        B.bsq_fake_quantize_nvfp4_static(big[:4], a, g, y=big[2:6])
    B.bsq_fake_quantize_nvfp4_static(x, a, g)  # a valid call still works
    torch.cuda.synchronize()
