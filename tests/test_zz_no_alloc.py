"""The no-allocation variant of the per-tensor NVFP4 quantizer.

Callers that cannot allocate device memory -- a serving engine that reserves
its whole memory budget at start-up and allows no allocation afterwards, or a
plain C caller without a device allocator -- cannot pass the scratch buffer
bsq_quantize_nvfp4_tensor needs.  bsq_quantize_nvfp4_tensor_noalloc keeps that
scratch in a fixed array inside the library instead.  This test checks,
through the C ABI, that it produces exactly the bytes of the scratch-buffer
entry point, on two calls in a row (the shared array keeps the previous
call's contents, which must not leak into the next result).

The file name makes pytest collect it last, so a run that stops at the first
failure has already run every other test; it also passes alone in a fresh
process.
"""
import numpy as np
import pytest
import torch

from gpu_util import assert_bits_equal, dev_bf16, host_bits

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def B():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from fp8_microscaling_quantization_b200 import bsq
    return bsq


def _both(B, x):
    p0, s0, t0 = B.bsq_quantize_nvfp4_tensor(x)
    p1, s1, t1 = B.bsq_quantize_nvfp4_tensor_noalloc(x)
    torch.cuda.synchronize()
    return (host_bits(p0), host_bits(s0), host_bits(t0)), (host_bits(p1), host_bits(s1), host_bits(t1))


def test_noalloc_matches_scratch_entry_point_twice(B):
    from fp8_microscaling_quantization_b200 import synth
    # a large matrix first (many partial maxima), then a small one: the second
    # call must ignore what the first left in the shared array
    big = dev_bf16(synth.linear_weight(out=1024, inp=4096, seed=901))
    small = dev_bf16(synth.linear_weight(out=8, inp=64, seed=902))
    for x in (big, small, big):
        want, got = _both(B, x)
        assert_bits_equal(got[2], want[2], "tensor scale")
        assert_bits_equal(got[1], want[1], "e4m3 scales")
        assert_bits_equal(got[0], want[0], "packed")


def test_noalloc_same_shape_lower_amax(B):
    """Two calls of one shape back to back, the second on a tensor whose
    maximum is far lower: every partial maximum the second call reads must be
    its own, or the first call's larger amax would leak into its tensor scale."""
    from fp8_microscaling_quantization_b200 import synth
    big = dev_bf16(synth.linear_weight(out=1024, inp=4096, seed=904))
    low = (big.float() * 0.01).to(torch.bfloat16)
    for x in (big, low):
        want, got = _both(B, x)
        assert_bits_equal(got[2], want[2], "tensor scale")
        assert_bits_equal(got[1], want[1], "e4m3 scales")
        assert_bits_equal(got[0], want[0], "packed")
    amax_low = low.float().abs().max().item()
    assert got[2].view(np.float32)[0] == np.float32(amax_low) / np.float32(2688.0)


def test_noalloc_fp32_input_and_empty(B):
    rng = np.random.default_rng(903)
    x = torch.from_numpy(rng.standard_normal((300, 512)).astype(np.float32)).cuda()
    for _ in range(2):
        want, got = _both(B, x)
        for g, w, what in zip(got, want, ("packed", "scales", "tensor scale")):
            assert_bits_equal(g, w, what)
    t = torch.full((1,), 7.0, device="cuda")
    e = torch.empty((0, 64), dtype=torch.bfloat16, device="cuda")
    B.bsq_quantize_nvfp4_tensor_noalloc(e, tensor_scale=t)
    torch.cuda.synchronize()
    assert t.item() == 0.0
