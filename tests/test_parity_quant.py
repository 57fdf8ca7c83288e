"""GPU parity of the quantize / dequantize / cache kernels against the CPU
oracle: bit-exact on codes, scales and dequantized values.  Every call goes
through the C ABI (the ctypes binding)."""
import numpy as np
import pytest
import torch

from gpu_util import assert_bits_equal, dev, dev_bf16, host_bits, sample_rows

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


def edge_bf16_values():
    """All finite bf16 values (bit patterns)."""
    b = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    f = f32_of(b)
    return b[np.isfinite(f)]


# ---------------------------------------------------------------- NVFP4 -----

# Rows of up to 2048 blocks (bf16 K <= 32768) are staged whole in shared
# memory by per-thread cp.async copies (at most 4 blocks per thread: K = 8240
# gives 515 blocks on 160 threads, the last ones with fewer than 4); longer
# rows up to K = 65536 run the one-CTA-per-row
# kernel that re-reads the row from L2; K > 65536 takes the two-kernel form
# (row amax pass, then the flat quantize reading the computed row scales).
@pytest.mark.parametrize("rows,K", [(256, 2048), (37, 272), (5, 16), (129, 4096), (7, 8240), (3, 40000),
                                    (1, 32768), (1, 65536), (3, 65552), (2, 131072)])
def test_nvfp4_rowamax_bf16(B, S, oracle, rows, K):
    x = S.nvfp4_matrix(rows=rows, cols=K, seed=1000 + rows + K)
    p, s, g = B.bsq_quantize_nvfp4(dev_bf16(x))
    torch.cuda.synchronize()
    op, os_, og = oracle.quantize_nvfp4(x)
    assert_bits_equal(host_bits(g), og, "row scale")
    assert_bits_equal(host_bits(s), os_, "e4m3 scales")
    assert_bits_equal(host_bits(p), op, "packed")
    y = B.bsq_dequantize_nvfp4(p, s, g)
    y32 = B.bsq_dequantize_nvfp4(p, s, g, out_dtype=B.DType.FP32)
    assert_bits_equal(host_bits(y), oracle.dequantize_nvfp4(op, os_, og), "dequant bf16")
    assert_bits_equal(host_bits(y32), oracle.dequantize_nvfp4(op, os_, og, out_dtype=oracle.F32), "dequant fp32")


# fp32 rows are staged up to 100 KiB (K = 25600, two stages of 100 KiB);
# K = 25616 and longer rows take the other kernels
@pytest.mark.parametrize("rows,K", [(64, 1024), (5, 25600), (4, 25616), (3, 65552)])
def test_nvfp4_rowamax_fp32_input(B, S, oracle, rows, K):
    rng = np.random.default_rng(5 + K)
    x = (rng.standard_normal((rows, K)) * np.exp(rng.uniform(-20, 20, (rows, 1)))).astype(np.float32)
    x[0, 7] *= 30.0  # an outlier that sets the row maximum
    p, s, g = B.bsq_quantize_nvfp4(dev(x))
    op, os_, og = oracle.quantize_nvfp4(x)
    assert_bits_equal(host_bits(g), og, "row scale")
    assert_bits_equal(host_bits(s), os_, "scales")
    assert_bits_equal(host_bits(p), op, "packed")


@pytest.mark.parametrize("fp32", [False, True])
def test_nvfp4_boundary_hits(B, oracle, fp32):
    """Rows whose blocks each hold 1.0 and 1/8 of it: with g = amax / 2688 the
    block scale is 448 and the quotient of 1/8 lands on the e2m1 midpoint 0.75
    up to the roundings of g and d, so the division-free brackets disagree in
    every block (1024 per row, more than the kernel's redo queue holds) and the
    plain rule decides.  Per-row, per-tensor and given (data-derived) scales."""
    rng = np.random.default_rng(31)
    rows, K = 6, 16384
    x = np.zeros((rows, K), np.uint16)
    x[:, 0::16] = 0x3F80                                   # 1.0
    x[:, 1::16] = 0x3E00                                   # 0.125
    x[:, 2::16] = rng.choice([0x3EC0, 0x3F40, 0x3D00], (rows, K // 16))  # 0.375, 0.75, 1/32
    x[:, 3::16] = rng.integers(0, 0x3F80, (rows, K // 16)).astype(np.uint16)
    x[1] = x[0] ^ 0x8000                                   # negative copy
    x[3, 0] = 0x4000                                       # row max 2.0: quotients of 1/16 ...
    xin = dev(f32_of(x)) if fp32 else dev_bf16(x)
    xo = f32_of(x) if fp32 else x
    p, s, g = B.bsq_quantize_nvfp4(xin)
    op, os_, og = oracle.quantize_nvfp4(xo)
    assert_bits_equal(host_bits(g), og, "row scale (hits)")
    assert_bits_equal(host_bits(s), os_, "scales (hits)")
    assert_bits_equal(host_bits(p), op, "packed (hits)")
    p, s, t = B.bsq_quantize_nvfp4_tensor(xin)
    op, os_, ot = oracle.quantize_nvfp4_tensor(xo)
    assert_bits_equal(host_bits(t)[:1], np.array([ot], np.float32), "tensor scale (hits)")
    assert_bits_equal(host_bits(s), os_, "tensor scales (hits)")
    assert_bits_equal(host_bits(p), op, "tensor packed (hits)")
    p, s, g = B.bsq_quantize_nvfp4(xin, row_scale_in=dev(og))
    op, os_, _ = oracle.quantize_nvfp4(xo, row_scale=og)
    assert_bits_equal(host_bits(s), os_, "given scales (hits)")
    assert_bits_equal(host_bits(p), op, "given packed (hits)")


def test_nvfp4_edge_values(B, oracle):
    """Zero rows, zero blocks, signed zeros, subnormals, the largest bf16 values
    and exact e2m1 ties (row scale 1 with a block maximum of 6 makes the block
    scale exactly 1, so the codes see the bf16 values themselves)."""
    vals = edge_bf16_values()
    f = f32_of(vals)
    small = vals[np.abs(f) <= 6.0]
    K = 1024
    n_full = -(-small.size // 15)
    blocks = np.zeros((n_full, 16), np.uint16)
    flat = np.zeros(n_full * 15, np.uint16)
    flat[:small.size] = small
    blocks[:, 0] = 0x40C0  # 6.0
    blocks[:, 1:] = flat.reshape(n_full, 15)
    x = blocks.reshape(-1)
    pad = (-x.size) % K
    x = np.concatenate([x, np.zeros(pad, np.uint16)]).reshape(-1, K)
    ones = np.ones(x.shape[0], np.float32)
    p, s, g = B.bsq_quantize_nvfp4(dev_bf16(x), row_scale_in=dev(ones))
    op, os_, og = oracle.quantize_nvfp4(x, row_scale=ones)
    assert_bits_equal(host_bits(s), os_, "scales (given g)")
    assert_bits_equal(host_bits(p), op, "packed (given g)")
    # per-row rule on rows with zero rows, -0.0, subnormals and huge values
    rng = np.random.default_rng(6)
    picks = rng.choice(vals, size=(64, 256))
    picks[3] = 0
    picks[4] = 0x8000
    picks[5, :16] = 0
    picks[6] = rng.integers(1, 0x7F, 256)           # positive subnormals
    picks[7] = 0x7F7F                               # max bf16
    picks[8, ::2] = 0x8001
    p, s, g = B.bsq_quantize_nvfp4(dev_bf16(picks))
    op, os_, og = oracle.quantize_nvfp4(picks)
    assert_bits_equal(host_bits(g), og, "row scale (edges)")
    assert_bits_equal(host_bits(s), os_, "scales (edges)")
    assert_bits_equal(host_bits(p), op, "packed (edges)")
    y = B.bsq_dequantize_nvfp4(p, s, g, out_dtype=B.DType.FP32)
    assert_bits_equal(host_bits(y), oracle.dequantize_nvfp4(op, os_, og, out_dtype=oracle.F32), "dequant (edges)")


@pytest.mark.parametrize("rows,K", [(96, 2048), (9, 8240), (3, 40000)])
def test_nvfp4_given_row_scales(B, S, oracle, rows, K):
    x = S.linear_weight(out=rows, inp=K, seed=77 + K)
    rng = np.random.default_rng(8)
    g_in = rng.uniform(1e-6, 1e-4, rows).astype(np.float32)
    g_in[min(5, rows - 1)] = 0.0
    g_in[0] = 1e-9  # block scales saturate at 448: codes of quotients far above 6
    # d = s * g below 2**-64 and above 2**100: outside the range of the
    # division-free codes, these blocks take the plain division
    g_in[1] = 1e-25
    if rows > 6:
        g_in[6] = 1e33
    p, s, g = B.bsq_quantize_nvfp4(dev_bf16(x), row_scale_in=dev(g_in))
    op, os_, og = oracle.quantize_nvfp4(x, row_scale=g_in)
    assert_bits_equal(host_bits(g), og, "row scale copy")
    assert_bits_equal(host_bits(s), os_, "scales")
    assert_bits_equal(host_bits(p), op, "packed")
    # fp32 input with the same scales
    xf = f32_of(x)
    p, s, g = B.bsq_quantize_nvfp4(dev(xf), row_scale_in=dev(g_in))
    op, os_, og = oracle.quantize_nvfp4(xf, row_scale=g_in)
    assert_bits_equal(host_bits(s), os_, "scales fp32")
    assert_bits_equal(host_bits(p), op, "packed fp32")


def test_nvfp4_dequant_all_scale_codes(B, oracle):
    rng = np.random.default_rng(9)
    rows, K = 254 * 4, 64
    packed = rng.integers(0, 256, (rows, K // 2), dtype=np.uint8)
    codes = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], np.uint8)
    scales = np.repeat(codes, 4 * (K // 16)).reshape(rows, K // 16)
    g = rng.uniform(1e-8, 1e3, rows).astype(np.float32)
    for dt, odt in ((B.DType.BF16, oracle.BF16), (B.DType.FP32, oracle.F32)):
        y = B.bsq_dequantize_nvfp4(dev(packed), dev(scales), dev(g), out_dtype=dt)
        assert_bits_equal(host_bits(y), oracle.dequantize_nvfp4(packed, scales, g, out_dtype=odt), f"dequant {dt}")


@pytest.mark.parametrize("rows,K", [(300, 4096), (5, 40000)])
def test_nvfp4_modelopt_tensor_scale(B, S, oracle, rows, K):
    x = S.linear_weight(out=rows, inp=K, seed=78 + K)
    p, s, t = B.bsq_quantize_nvfp4_tensor(dev_bf16(x))
    op, os_, ot = oracle.quantize_nvfp4_tensor(x)
    assert_bits_equal(host_bits(t)[:1], np.array([ot], np.float32), "tensor scale")
    assert_bits_equal(host_bits(s), os_, "scales")
    assert_bits_equal(host_bits(p), op, "packed")


def test_nvfp4_full_size_linear_weight(B, S, oracle):
    """[7168, 18432]: ModelOpt per-tensor, per-row and gate/up, sampled rows."""
    x = S.linear_weight()
    xd = dev_bf16(x)
    p, s, t = B.bsq_quantize_nvfp4_tensor(xd)
    pr, sr, gr = B.bsq_quantize_nvfp4(xd)
    torch.cuda.synchronize()
    amax = np.abs(f32_of(x)).max()
    t_ref = np.float32(amax) / np.float32(2688.0)
    assert host_bits(t)[0] == t_ref
    rows = sample_rows(x.shape[0], 48, 1)
    sub = np.ascontiguousarray(x[rows])
    op, os_, _ = oracle.quantize_nvfp4(sub, row_scale=np.full(rows.size, t_ref, np.float32))
    assert_bits_equal(host_bits(p)[rows], op, "tensor packed (sampled rows)")
    assert_bits_equal(host_bits(s)[rows], os_, "tensor scales (sampled rows)")
    op, os_, og = oracle.quantize_nvfp4(sub)
    assert_bits_equal(host_bits(gr)[rows], og, "row scales (sampled rows)")
    assert_bits_equal(host_bits(pr)[rows], op, "row packed (sampled rows)")
    assert_bits_equal(host_bits(sr)[rows], os_, "row scales e4m3 (sampled rows)")
    # storage: 0.5625 bytes per parameter plus 4 bytes per row
    assert pr.numel() + sr.numel() + 4 * gr.numel() == 0.5625 * x.size + 4 * x.shape[0]
    # gate/up: the concatenation carrying both halves' tensor scales
    up = S.linear_weight(seed=20260005)
    ud = dev_bf16(up)
    pu, su, tu = B.bsq_quantize_nvfp4_tensor(ud)
    cat = torch.cat([xd, ud], dim=0)
    rs = torch.cat([t.expand(x.shape[0]), tu.expand(up.shape[0])]).contiguous()
    pc, sc, gc = B.bsq_quantize_nvfp4(cat, row_scale_in=rs)
    torch.cuda.synchronize()
    tu_ref = np.float32(np.abs(f32_of(up)).max()) / np.float32(2688.0)
    assert host_bits(tu)[0] == tu_ref
    # both halves of the concatenation against the oracle, each row with its
    # half's tensor scale
    urows = sample_rows(up.shape[0], 48, 2)
    cat_rows = np.concatenate([rows, x.shape[0] + urows])
    csub = np.ascontiguousarray(np.concatenate([x[rows], up[urows]]))
    g_rows = np.concatenate([np.full(rows.size, t_ref, np.float32), np.full(urows.size, tu_ref, np.float32)])
    op, os_, og = oracle.quantize_nvfp4(csub, row_scale=g_rows)
    assert_bits_equal(host_bits(gc)[cat_rows], og, "gate/up row scales (sampled rows)")
    assert_bits_equal(host_bits(pc)[cat_rows], op, "gate/up packed (sampled rows)")
    assert_bits_equal(host_bits(sc)[cat_rows], os_, "gate/up e4m3 scales (sampled rows)")
    # and the up half's own per-tensor quantization on its sampled rows
    assert_bits_equal(host_bits(pu)[urows], op[rows.size:], "up tensor packed (sampled rows)")
    assert_bits_equal(host_bits(su)[urows], os_[rows.size:], "up tensor scales (sampled rows)")
    assert torch.equal(pc, torch.cat([p, pu])) and torch.equal(sc, torch.cat([s, su]))


# ---------------------------------------------------------------- MXFP4 -----

def test_mxfp4_full_size_expert_weights(B, S, oracle):
    """[8, 2048, 7168] routed-expert weights: quantize, dequantize to bf16 and fp32,
    compared in full."""
    x = S.expert_weights()
    p, s = B.bsq_quantize_mxfp4(dev_bf16(x))
    yb = B.bsq_dequantize_mxfp4(p, s)
    yf = B.bsq_dequantize_mxfp4(p, s, out_dtype=B.DType.FP32)
    op, os_ = oracle.quantize_mxfp4(x)
    assert_bits_equal(host_bits(s), os_, "e8m0 scales")
    assert_bits_equal(host_bits(p), op, "packed")
    del x
    assert_bits_equal(host_bits(yb), oracle.dequantize_mxfp4(op, os_), "dequant bf16")
    assert_bits_equal(host_bits(yf), oracle.dequantize_mxfp4(op, os_, out_dtype=oracle.F32), "dequant fp32")
    assert (host_bits(s) == 0).sum() == 8 * 16  # the exact-zero blocks


@pytest.mark.parametrize("rows,K", [(3, 32), (77, 96), (1000, 1024)])
def test_mxfp4_small_and_ragged(B, S, oracle, rows, K):
    x = S.nvfp4_matrix(rows=rows, cols=K, seed=rows * 7 + K)
    p, s = B.bsq_quantize_mxfp4(dev_bf16(x))
    op, os_ = oracle.quantize_mxfp4(x)
    assert_bits_equal(host_bits(s), os_, "scales")
    assert_bits_equal(host_bits(p), op, "packed")
    xf = f32_of(x) * np.float32(1e-30)
    p, s = B.bsq_quantize_mxfp4(dev(xf))
    op, os_ = oracle.quantize_mxfp4(xf)
    assert_bits_equal(host_bits(s), os_, "scales fp32 tiny")
    assert_bits_equal(host_bits(p), op, "packed fp32 tiny")


def test_mxfp4_every_bf16_value_as_quotient(B, oracle):
    """Blocks led by 7.5 have exponent 0, so the e2m1 rounding sees every bf16
    value of magnitude <= 7.5 unchanged: ties, saturation and signed zeros."""
    vals = edge_bf16_values()
    v = vals[np.abs(f32_of(vals)) <= 7.5]
    n = -(-v.size // 31)
    flat = np.zeros(n * 31, np.uint16)
    flat[:v.size] = v
    blocks = np.zeros((n, 32), np.uint16)
    blocks[:, 0] = 0x40F0  # 7.5
    blocks[:, 1:] = flat.reshape(n, 31)
    p, s = B.bsq_quantize_mxfp4(dev_bf16(blocks))
    op, os_ = oracle.quantize_mxfp4(blocks)
    assert np.all(os_ == 127)
    assert_bits_equal(host_bits(s), os_, "scales")
    assert_bits_equal(host_bits(p), op, "packed")


def test_mxfp4_dequant_all_scale_codes(B, oracle):
    rng = np.random.default_rng(10)
    packed = rng.integers(0, 256, (256, 16), dtype=np.uint8)
    scales = np.arange(256, dtype=np.uint8).reshape(256, 1)  # 255 = NaN
    for dt, odt in ((B.DType.BF16, oracle.BF16), (B.DType.FP32, oracle.F32)):
        y = B.bsq_dequantize_mxfp4(dev(packed), dev(scales), out_dtype=dt)
        want = oracle.dequantize_mxfp4(packed, scales, out_dtype=odt)
        got = host_bits(y)
        if odt == oracle.BF16:
            nan = np.isnan(f32_of(want))
            assert np.array_equal(np.isnan(f32_of(got)), nan)
            got, want = got[~nan], want[~nan]
        assert_bits_equal(got, want, f"dequant {dt}")


# ---------------------------------------------------------------- MXFP8 -----

def test_mxfp8_full_size_expert_weights(B, S, oracle):
    """[8, 2048, 7168] routed-expert weights as MXFP8: scales, codes and both
    dequantized outputs compared in full."""
    x = S.expert_weights()
    c, s = B.bsq_quantize_mxfp8(dev_bf16(x))
    yb = B.bsq_dequantize_mxfp8(c, s)
    yf = B.bsq_dequantize_mxfp8(c, s, out_dtype=B.DType.FP32)
    oc, os_ = oracle.quantize_mxfp8(x)
    del x
    assert_bits_equal(host_bits(s), os_, "e8m0 scales")
    assert_bits_equal(host_bits(c), oc, "e4m3 codes")
    assert_bits_equal(host_bits(yb), oracle.dequantize_mxfp8(oc, os_), "dequant bf16")
    assert_bits_equal(host_bits(yf), oracle.dequantize_mxfp8(oc, os_, out_dtype=oracle.F32), "dequant fp32")
    assert (host_bits(s) == 0).sum() == 8 * 16  # the exact-zero blocks


@pytest.mark.parametrize("rows,K", [(3, 32), (77, 96), (1000, 1024)])
def test_mxfp8_small_and_ragged(B, S, oracle, rows, K):
    x = S.nvfp4_matrix(rows=rows, cols=K, seed=rows * 11 + K)
    c, s = B.bsq_quantize_mxfp8(dev_bf16(x))
    oc, os_ = oracle.quantize_mxfp8(x)
    assert_bits_equal(host_bits(s), os_, "scales")
    assert_bits_equal(host_bits(c), oc, "codes")
    # fp32 input far below 2**-118: the block exponent sits on the e8m0 floor
    xf = f32_of(x) * np.float32(1e-36)
    c, s = B.bsq_quantize_mxfp8(dev(xf))
    oc, os_ = oracle.quantize_mxfp8(xf)
    assert (os_ == 0).any()
    assert_bits_equal(host_bits(s), os_, "scales fp32 tiny")
    assert_bits_equal(host_bits(c), oc, "codes fp32 tiny")


def test_mxfp8_every_bf16_value_as_quotient(B, oracle):
    """Blocks led by 256 have exponent 0, so the e4m3 rounding sees every bf16
    value of magnitude below 512 unchanged: ties, subnormals, signed zeros and
    the saturation of (448, 512)."""
    vals = edge_bf16_values()
    v = vals[np.abs(f32_of(vals)) < 512]
    n = -(-v.size // 31)
    flat = np.zeros(n * 31, np.uint16)
    flat[:v.size] = v
    blocks = np.zeros((n, 32), np.uint16)
    blocks[:, 0] = 0x4380  # 256
    blocks[:, 1:] = flat.reshape(n, 31)
    c, s = B.bsq_quantize_mxfp8(dev_bf16(blocks))
    oc, os_ = oracle.quantize_mxfp8(blocks)
    assert np.all(os_ == 127)
    assert_bits_equal(host_bits(s), os_, "scales")
    assert_bits_equal(host_bits(c), oc, "codes")


def test_mxfp8_dequant_all_scale_codes(B, oracle):
    rng = np.random.default_rng(14)
    codes = rng.integers(0, 256, (256, 32), dtype=np.uint8)  # includes the NaN codes
    scales = np.arange(256, dtype=np.uint8).reshape(256, 1)  # 255 = NaN
    for dt, odt in ((B.DType.BF16, oracle.BF16), (B.DType.FP32, oracle.F32)):
        y = B.bsq_dequantize_mxfp8(dev(codes), dev(scales), out_dtype=dt)
        want = oracle.dequantize_mxfp8(codes, scales, out_dtype=odt)
        got = host_bits(y)
        nan = np.isnan(f32_of(want) if odt == oracle.BF16 else want)
        assert np.array_equal(np.isnan(f32_of(got) if odt == oracle.BF16 else got.view(np.float32)), nan)
        assert_bits_equal(got[~nan], want[~nan], f"dequant {dt}")


# ------------------------------------------------------------------ FP8 -----

@pytest.mark.parametrize("block", [16, 32])
def test_fp8_quant_dequant(B, S, oracle, block):
    x, _ = S.cache_acts(B=2, T=300, C=512, seed=40 + block)
    c, s = B.bsq_quantize_fp8(dev_bf16(x), block=block)
    oc, os_ = oracle.quantize_fp8(x, block)
    assert_bits_equal(host_bits(s), os_, "e8m0 scales")
    assert_bits_equal(host_bits(c), oc, "e4m3 codes")
    for dt, odt in ((B.DType.BF16, oracle.BF16), (B.DType.FP32, oracle.F32)):
        y = B.bsq_dequantize_fp8(c, s, block=block, out_dtype=dt)
        assert_bits_equal(host_bits(y), oracle.dequantize_fp8(oc, os_, block, out_dtype=odt), f"dequant {dt}")


def test_fp8_every_bf16_value(B, oracle):
    """Blocks led by 448 have scale 1, so the e4m3 rounding sees every bf16
    value of magnitude <= 448 unchanged."""
    vals = edge_bf16_values()
    v = vals[np.abs(f32_of(vals)) <= 448]
    n = -(-v.size // 31)
    flat = np.zeros(n * 31, np.uint16)
    flat[:v.size] = v
    blocks = np.zeros((n, 32), np.uint16)
    blocks[:, 0] = 0x43E0  # 448
    blocks[:, 1:] = flat.reshape(n, 31)
    c, s = B.bsq_quantize_fp8(dev_bf16(blocks), block=32)
    oc, os_ = oracle.quantize_fp8(blocks, 32)
    assert np.all(os_ == 127)
    assert_bits_equal(host_bits(c), oc, "codes")
    rng = np.random.default_rng(12)
    xf = (rng.standard_normal((64, 64)) * np.exp(rng.uniform(-80, 80, (64, 1)))).astype(np.float32)
    c, s = B.bsq_quantize_fp8(dev(xf), block=16)
    oc, os_ = oracle.quantize_fp8(xf, 16)
    assert_bits_equal(host_bits(s), os_, "scales fp32")
    assert_bits_equal(host_bits(c), oc, "codes fp32")


# -------------------------------------------------------- quantize_cache -----

CACHE_FULL = [(0, 32, (4, 8192, 512)), (1, 32, (4, 8192, 128)), (2, 16, (4, 2048, 512)),
              (0, 32, (4, 2048, 520)), (1, 32, (4, 2048, 520)), (2, 16, (4, 2048, 520))]


@pytest.mark.parametrize("fmt,block,shape", CACHE_FULL)
def test_cache_full_size(B, S, oracle, fmt, block, shape):
    x, g = S.cache_acts(*shape)
    y = B.bsq_quantize_cache(dev_bf16(x), fmt, block)
    rows = sample_rows(shape[0] * shape[1], 512, fmt * 100 + block)
    flat = x.reshape(-1, shape[2])
    want = oracle.quantize_cache(np.ascontiguousarray(flat[rows]), fmt, block)
    assert_bits_equal(host_bits(y).reshape(-1, shape[2])[rows], want, "cache fake-quant (sampled rows)")
    # straight-through backward: identity, aliased and copied
    gd = dev_bf16(g)
    assert B.bsq_quantize_cache_backward(gd) is gd
    gi = torch.empty_like(gd)
    B.bsq_quantize_cache_backward(gd, gi)
    assert_bits_equal(host_bits(gi), g, "STE gradient")


@pytest.mark.parametrize("fmt", [0, 1, 2])
@pytest.mark.parametrize("block", [16, 32])
@pytest.mark.parametrize("C", [1, 8, 13, 40, 128, 264, 300, 520, 640, 4104])
def test_cache_shapes(B, S, oracle, fmt, block, C):
    x, _ = S.cache_acts(B=2, T=37, C=C, seed=C * 3 + block + fmt)
    xd = dev_bf16(x)
    y = B.bsq_quantize_cache(xd, fmt, block)
    assert_bits_equal(host_bits(y), oracle.quantize_cache(x, fmt, block), f"cache bf16 C={C}")
    assert_bits_equal(host_bits(xd), x, "input unchanged")
    xf = f32_of(x) * np.float32(3.0e-3)
    y = B.bsq_quantize_cache(dev(xf), fmt, block)
    assert_bits_equal(host_bits(y), oracle.quantize_cache(xf, fmt, block), f"cache fp32 C={C}")


def test_cache_edge_values(B, oracle):
    rng = np.random.default_rng(14)
    vals = edge_bf16_values()
    x = rng.choice(vals, size=(64, 96))
    x[0] = 0
    x[1] = 0x8000
    x[2, :40] = 0
    x[3] = rng.integers(1, 0x7F, 96)
    x[4] = 0x7F7F
    for fmt in (0, 1, 2):
        for block in (16, 32):
            y = B.bsq_quantize_cache(dev_bf16(x), fmt, block)
            assert_bits_equal(host_bits(y), oracle.quantize_cache(x, fmt, block), f"edges fmt={fmt} b={block}")
