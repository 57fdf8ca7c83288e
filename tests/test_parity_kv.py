"""GPU parity of the list-of-blocks NVFP4 KV-cache dequantization against the
CPU oracle: bit-exact, through the C ABI."""
import numpy as np
import pytest
import torch

from gpu_util import assert_bits_equal, dev, host_bits

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def B():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from fp8_microscaling_quantization_b200 import bsq
    return bsq


def make_cache(oracle, nblocks, block_tokens, heads, seed):
    """KV blocks as a quantizer would leave them: bf16 activations per block,
    quantized with the block's own global scale amax / 2688 (host arrays)."""
    from fp8_microscaling_quantization_b200 import synth
    rng = np.random.default_rng(seed)
    rows = block_tokens * heads
    vals, scs, amax = [], [], []
    for b in range(nblocks):
        x = synth.to_bf16_bits((rng.standard_normal((rows, 128)) * np.exp(rng.uniform(-3, 3))).astype(np.float32))
        a = np.float32(np.abs(synth.bf16_bits_to_f32(x)).max())
        p, s, _ = oracle.quantize_nvfp4(x, row_scale=np.float32(a) / np.float32(2688.0))
        vals.append(p)
        scs.append(s)
        amax.append(a)
    amax = np.array(amax, np.float32)
    if nblocks > 2:
        amax[1] = 0.0  # an all-zero block
    return vals, scs, amax


def to_device(B, vals, scs, amax, offset=0):
    """Per-block device tensors (optionally starting `offset` bytes into a
    larger allocation) and the pointer table."""
    dv, ds, da = [], [], []
    for v, s, a in zip(vals, scs, amax):
        if offset:
            big = torch.zeros(v.size + offset, dtype=torch.uint8, device="cuda")
            big[offset:] = torch.from_numpy(v.reshape(-1)).cuda()
            dv.append(big[offset:])
            bs = torch.zeros(s.size + offset, dtype=torch.uint8, device="cuda")
            bs[offset:] = torch.from_numpy(s.reshape(-1)).cuda()
            ds.append(bs[offset:])
        else:
            dv.append(dev(v))
            ds.append(dev(s))
        da.append(dev(np.array([a], np.float32)))
    return (dv, ds, da), B.kv_block_table(dv, ds, da)


@pytest.mark.parametrize("nblocks,block_tokens,heads", [(1, 16, 1), (7, 16, 8), (33, 64, 2), (1024, 64, 8)])
def test_kv_cache_dequant(B, oracle, nblocks, block_tokens, heads):
    vals, scs, amax = make_cache(oracle, nblocks, block_tokens, heads, seed=nblocks + block_tokens + heads)
    keep, table = to_device(B, vals, scs, amax)
    for dt, odt in ((B.DType.BF16, oracle.BF16), (B.DType.FP32, oracle.F32)):
        y = B.bsq_dequantize_kv_cache_nvfp4(table, nblocks, block_tokens, heads, out_dtype=dt)
        torch.cuda.synchronize()
        want = oracle.dequantize_kv_cache_nvfp4(vals, scs, amax, block_tokens, heads, out_dtype=odt)
        assert_bits_equal(host_bits(y), want, f"kv dequant {dt}")


@pytest.mark.parametrize("offset", [1, 2, 3])
def test_kv_cache_unaligned_blocks(B, oracle, offset):
    """Blocks that start at odd byte offsets take the byte-load path."""
    vals, scs, amax = make_cache(oracle, 5, 16, 4, seed=80 + offset)
    keep, table = to_device(B, vals, scs, amax, offset=offset)
    for dt, odt in ((B.DType.BF16, oracle.BF16), (B.DType.FP32, oracle.F32)):
        y = B.bsq_dequantize_kv_cache_nvfp4(table, 5, 16, 4, out_dtype=dt)
        torch.cuda.synchronize()
        assert_bits_equal(host_bits(y), oracle.dequantize_kv_cache_nvfp4(vals, scs, amax, 16, 4, out_dtype=odt),
                          f"offset {offset} {dt}")


def test_kv_cache_empty_and_rejects(B):
    t = torch.zeros((1,), dtype=torch.int64, device="cuda")
    y = torch.empty((1, 0, 8, 128), dtype=torch.bfloat16, device="cuda")
    B.bsq_dequantize_kv_cache_nvfp4((t, t, t), 0, 64, 8, y=y)  # no blocks: nothing to do
    with pytest.raises(B.BsqError):
        B.bsq_dequantize_kv_cache_nvfp4((t, t, t), -1, 64, 8, y=y)
    torch.cuda.synchronize()


def test_kv_cache_dequant_all_scale_codes(B, oracle):
    """Arbitrary bytes in the cache: every e2m1 code next to every finite e4m3
    scale code, negative scales included (the sign of a zero product follows
    the scale), so the decode order and signed zeros are checked bit for bit."""
    rng = np.random.default_rng(21)
    codes = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], np.uint8)
    block_tokens, heads = 16, 2
    rows = block_tokens * heads
    vals, scs, amax = [], [], []
    for b in range(8):
        vals.append(rng.integers(0, 256, (rows, 64), dtype=np.uint8))
        scs.append(codes[rng.integers(0, codes.size, (rows, 8))])
        amax.append(np.float32(rng.uniform(1e-3, 1e4)))
    scs[0] = np.resize(codes, (rows, 8))  # block 0 holds every scale code
    amax = np.array(amax, np.float32)
    _, table = to_device(B, vals, scs, amax)
    for dt, odt in ((B.DType.BF16, oracle.BF16), (B.DType.FP32, oracle.F32)):
        y = B.bsq_dequantize_kv_cache_nvfp4(table, len(vals), block_tokens, heads, out_dtype=dt)
        assert_bits_equal(host_bits(y), oracle.dequantize_kv_cache_nvfp4(vals, scs, amax, block_tokens, heads,
                                                                          out_dtype=odt), f"kv all codes {dt}")


def test_kv_cache_long_blocks(B, oracle):
    """Two blocks of 16384 tokens x 8 heads: each block is 1024 work units of
    the kernel, more than the CTAs resident on the device, so a CTA's next
    unit often lies in the block it is working on (the pointers it
    prefetched are the current ones) and sometimes in the other block."""
    vals, scs, amax = make_cache(oracle, 2, 16384, 8, seed=31)
    _, table = to_device(B, vals, scs, amax)
    for dt, odt in ((B.DType.BF16, oracle.BF16), (B.DType.FP32, oracle.F32)):
        y = B.bsq_dequantize_kv_cache_nvfp4(table, 2, 16384, 8, out_dtype=dt)
        want = oracle.dequantize_kv_cache_nvfp4(vals, scs, amax, 16384, 8, out_dtype=odt)
        assert_bits_equal(host_bits(y), want, f"kv long blocks {dt}")
