"""The hot path captured into a CUDA graph and replayed.

Every entry point enqueues its work on the caller's stream only and, once its
host-side caches are warm (SM count, occupancy, shared-memory opt-in, the
tensor-map encoder), calls nothing that a stream capture forbids.  So one
eager pass, then a capture of the same calls on a side stream, replays them:
the replay, on new values written into the captured input buffers, must give
bit for bit what eager calls give on those values (the eager path itself is
checked against the oracle by the parity tests)."""
import pytest
import torch

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def B():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from fp8_microscaling_quantization_b200 import bsq
    return bsq


def test_hot_path_replays_from_a_cuda_graph(B):
    d = "cuda"
    u8, bf, f32 = torch.uint8, torch.bfloat16, torch.float32
    # inputs, rewritten in place before each run
    xm = torch.empty(4, 256, 2048, dtype=bf, device=d)      # MXFP4 round trip
    xn = torch.empty(256, 2048, dtype=bf, device=d)         # NVFP4 per row and per tensor
    kv = torch.empty(2, 64, 520, dtype=bf, device=d)        # cache fake-quant, partial group
    E, N, K, T = 4, 256, 512, 300
    xg = torch.empty(T, K, dtype=bf, device=d)              # grouped GEMM tokens
    gen = torch.Generator(device=d).manual_seed(20260011)
    w = (torch.randn(E, N, K, generator=gen, device=d) * 0.02).to(bf)
    wp, ws = B.bsq_quantize_mxfp4(w)
    offs = torch.tensor([37, 37, 200, 300], dtype=torch.int32, device=d)  # one empty expert

    def fill(seed):
        g = torch.Generator(device=d).manual_seed(seed)
        for t in (xm, xn, kv, xg):
            t.copy_(torch.randn(t.shape, generator=g, device=d).to(t.dtype))

    # outputs, allocated once (a capture must not allocate)
    pm, sm = torch.empty(4, 256, 1024, dtype=u8, device=d), torch.empty(4, 256, 64, dtype=u8, device=d)
    ym, ym32 = torch.empty_like(xm), torch.empty(4, 256, 2048, dtype=f32, device=d)
    pn, sn = torch.empty(256, 1024, dtype=u8, device=d), torch.empty(256, 128, dtype=u8, device=d)
    gn, yn = torch.empty(256, dtype=f32, device=d), torch.empty_like(xn)
    pt, st = torch.empty_like(pn), torch.empty_like(sn)
    ts = torch.empty(1, dtype=f32, device=d)
    scratch = torch.empty(B.bsq_nvfp4_tensor_scratch_bytes(256, 2048), dtype=u8, device=d)
    kvy = torch.empty_like(kv)
    yg = torch.empty(T, N, dtype=bf, device=d)
    err = torch.zeros(1, dtype=torch.int32, device=d)
    outs = {"mxfp4 packed": pm, "mxfp4 scales": sm, "mxfp4 dequant bf16": ym, "mxfp4 dequant fp32": ym32,
            "nvfp4 packed": pn, "nvfp4 scales": sn, "nvfp4 row scales": gn, "nvfp4 dequant": yn,
            "nvfp4 tensor packed": pt, "nvfp4 tensor scales": st, "nvfp4 tensor scale": ts,
            "cache nvfp4": kvy, "grouped gemm": yg, "gemm error word": err}

    def run():
        B.bsq_quantize_mxfp4(xm, packed=pm, scales=sm)
        B.bsq_dequantize_mxfp4(pm, sm, y=ym)
        B.bsq_dequantize_mxfp4(pm, sm, out_dtype=B.DType.FP32, y=ym32)
        B.bsq_quantize_nvfp4(xn, packed=pn, scales=sn, row_scale_out=gn)
        B.bsq_dequantize_nvfp4(pn, sn, gn, y=yn)
        B.bsq_quantize_nvfp4_tensor(xn, packed=pt, scales=st, tensor_scale=ts, scratch=scratch)
        B.bsq_quantize_cache(kv, B.Format.NVFP4, 16, y=kvy)
        B.bsq_grouped_mm_fp4(B.Format.MXFP4, B.Direction.FWD, xg, wp, ws, None, offs, out=yg, err=err)

    fill(1)
    run()  # warms the library's host-side caches
    torch.cuda.synchronize()
    first = {k: v.clone() for k, v in outs.items()}

    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):  # a side stream; the binding enqueues on torch's current stream
        run()
    fill(2)
    graph.replay()
    torch.cuda.synchronize()
    replayed = {k: v.clone() for k, v in outs.items()}

    for v in outs.values():
        v.zero_()
    run()  # eager, on the same inputs
    torch.cuda.synchronize()

    assert int(err.item()) == 0 and int(replayed["gemm error word"].item()) == 0
    for k, v in outs.items():
        a, b = replayed[k].view(-1).view(u8), v.view(-1).view(u8)
        assert torch.equal(a, b), f"{k}: the graph replay differs from the eager call"
    for k in ("mxfp4 dequant bf16", "nvfp4 dequant", "cache nvfp4", "grouped gemm"):
        assert not torch.equal(first[k], replayed[k]), f"{k}: the replay did not recompute"
