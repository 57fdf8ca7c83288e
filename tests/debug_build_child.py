"""Child process of test_debug_build.py: loads the bounds-checking library
(BSQ_LIBRARY names libbsq_debug.so), runs every entry point on tiny and
ragged shapes, checks the results against the CPU oracle and prints the
index-check counters as one JSON line."""
import json
import os
import sys

import numpy as np
import torch

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(HERE))
sys.path.insert(0, HERE)

import oracle  # noqa: E402
from fp8_microscaling_quantization_b200 import bsq, synth  # noqa: E402
from gpu_util import dev, dev_bf16, host_bits  # noqa: E402


def same(a, b, what):
    assert np.array_equal(np.asarray(a), np.asarray(b)), what


def main():
    assert bsq.lib_path.endswith("libbsq_debug.so"), bsq.lib_path
    torch.cuda.set_device(0)
    bsq.bsq_debug_counters()  # start from zero
    # NVFP4: per-row (staged rows, L2 re-read and two-kernel forms), given and tensor scales
    for rows, K in ((3, 16), (5, 48), (7, 8240), (2, 40000), (2, 65552)):
        x = synth.nvfp4_matrix(rows=rows, cols=K, seed=rows + K)
        p, s, g = bsq.bsq_quantize_nvfp4(dev_bf16(x))
        op, os_, og = oracle.quantize_nvfp4(x)
        same(host_bits(p), op, f"nvfp4 packed {rows}x{K}")
        same(host_bits(s), os_, f"nvfp4 scales {rows}x{K}")
        p2, s2, _ = bsq.bsq_quantize_nvfp4(dev_bf16(x), row_scale_in=dev(og))
        same(host_bits(p2), op, f"nvfp4 given {rows}x{K}")
        p3, s3, t3 = bsq.bsq_quantize_nvfp4_tensor(dev_bf16(x))
        p4, s4, t4 = bsq.bsq_quantize_nvfp4_tensor_noalloc(dev_bf16(x))
        same(host_bits(p3), host_bits(p4), f"nvfp4 tensor / no-alloc {rows}x{K}")
        y = bsq.bsq_dequantize_nvfp4(p, s, g, out_dtype=bsq.DType.FP32)
        same(host_bits(y), oracle.dequantize_nvfp4(op, os_, og, out_dtype=oracle.F32), f"nvfp4 dequant {rows}x{K}")
    # MXFP4, MXFP8, FP8
    for rows, K in ((1, 32), (9, 96), (33, 160)):
        x = synth.nvfp4_matrix(rows=rows, cols=K, seed=7 * rows + K)
        p, s = bsq.bsq_quantize_mxfp4(dev_bf16(x))
        op, os_ = oracle.quantize_mxfp4(x)
        same(host_bits(p), op, "mxfp4")
        same(host_bits(bsq.bsq_dequantize_mxfp4(p, s)), oracle.dequantize_mxfp4(op, os_), "mxfp4 dequant")
        c, s = bsq.bsq_quantize_mxfp8(dev_bf16(x))
        same(host_bits(c), oracle.quantize_mxfp8(x)[0], "mxfp8")
        bsq.bsq_dequantize_mxfp8(c, s)
        for block in (16, 32):
            c, s = bsq.bsq_quantize_fp8(dev_bf16(x), block=block)
            same(host_bits(c), oracle.quantize_fp8(x, block)[0], "fp8")
            bsq.bsq_dequantize_fp8(c, s, block=block)
    # cache fake-quant, ragged and partial groups
    for fmt in (0, 1, 2):
        for block in (16, 32):
            for C in (1, 13, 40, 520):
                x, _ = synth.cache_acts(B=1, T=9, C=C, seed=C + block + fmt)
                y = bsq.bsq_quantize_cache(dev_bf16(x), fmt, block)
                same(host_bits(y), oracle.quantize_cache(x, fmt, block), f"cache {fmt} {block} {C}")
    # static two-level fake-quant
    x = synth.linear_weight(out=5, inp=64, seed=3)
    xf = synth.bf16_bits_to_f32(x)
    bam = np.abs(xf).reshape(5, -1, 16).max(axis=2).astype(np.float32)
    gam = np.float32(np.abs(xf).max())
    y = bsq.bsq_fake_quantize_nvfp4_static(dev_bf16(x), dev(bam), dev(np.array([gam], np.float32)))
    same(host_bits(y), oracle.fake_quantize_nvfp4_static(x, bam, gam), "static")
    # KV cache, three blocks
    rng = np.random.default_rng(5)
    bt, hd = 4, 2
    vals = [rng.integers(0, 256, (bt * hd, 64), dtype=np.uint8) for _ in range(3)]
    scs = [rng.integers(0, 0x7E, (bt * hd, 8), dtype=np.uint8) for _ in range(3)]
    am = rng.random(3).astype(np.float32) * 10
    dv, ds, da = [dev(v) for v in vals], [dev(v) for v in scs], [dev(am[i:i + 1]) for i in range(3)]
    table = bsq.kv_block_table(dv, ds, da)
    yk = bsq.bsq_dequantize_kv_cache_nvfp4(table, 3, bt, hd)
    same(host_bits(yk), oracle.dequantize_kv_cache_nvfp4(vals, scs, am, bt, hd), "kv")
    # grouped GEMM, both formats and directions, ragged experts (checked for the error word only)
    T, K, N, E = 300, 256, 256, 4
    offs = np.array([0, 1, 130, 290], np.int32)
    xa = synth.to_bf16_bits(rng.standard_normal((T, K), dtype=np.float32))
    go = synth.to_bf16_bits(rng.standard_normal((T, N), dtype=np.float32))
    w = synth.to_bf16_bits(rng.standard_normal((E, N, K), dtype=np.float32) * np.float32(0.02))
    mp, ms = oracle.quantize_mxfp4(w)
    npk, nsc, ng = oracle.quantize_nvfp4(w)
    for f, p_, s_, g_ in ((bsq.Format.MXFP4, mp, ms, None), (bsq.Format.NVFP4, npk, nsc, ng)):
        for d, a in ((bsq.Direction.FWD, xa), (bsq.Direction.BWD, go)):
            _, err = bsq.bsq_grouped_mm_fp4(f, d, dev_bf16(a), dev(p_), dev(s_), None if g_ is None else dev(g_),
                                            dev(offs))
            torch.cuda.synchronize()
            assert int(err.item()) == 0
    count, first = bsq.bsq_debug_counters()
    print(json.dumps({"failed_checks": count, "first_code": first}), flush=True)


if __name__ == "__main__":
    main()
