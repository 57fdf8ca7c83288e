"""GPU parity of the fused-dequant grouped GEMM against the float64 oracle.

Tolerances (per output, fp32 accumulation on bf16 operands, bf16 output):
relative Frobenius error <= 5e-3 and max-abs error <=
1e-2 * sqrt(K_contraction) * max|a| * max|W|.  Rows at or past offs[-1] must
be exactly zero.  Every call goes through the C ABI (ctypes binding)."""
import numpy as np
import pytest
import torch

from gpu_util import dev, dev_bf16, host_bits, sample_rows

pytestmark = pytest.mark.gpu

REL_FRO = 5e-3
MAXABS_C = 1e-2


@pytest.fixture(scope="module")
def B():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from fp8_microscaling_quantization_b200 import bsq
    return bsq


def f32(bits):
    return (np.asarray(bits, np.uint16).astype(np.uint32) << 16).view(np.float32)


def quantize_weights(oracle, fmt, w_bits):
    if fmt == oracle.FMT_MXFP4:
        p, s = oracle.quantize_mxfp4(w_bits)
        return p, s, None
    p, s, g = oracle.quantize_nvfp4(w_bits)
    return p, s, g


def run_gemm(B, oracle, fmt, backward, a_bits, packed, scales, g, offs):
    f = B.Format.MXFP4 if fmt == oracle.FMT_MXFP4 else B.Format.NVFP4
    d = B.Direction.BWD if backward else B.Direction.FWD
    out, err = B.bsq_grouped_mm_fp4(f, d, dev_bf16(a_bits), dev(packed), dev(scales),
                                    None if g is None else dev(g), dev(offs))
    torch.cuda.synchronize()
    return f32(host_bits(out)).astype(np.float64), int(err.item())


def check_rows(got, ref, a_bits, W_absmax, kc, what):
    rel = np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-30)
    bound = MAXABS_C * np.sqrt(kc) * np.abs(f32(a_bits)).max() * W_absmax
    mx = np.abs(got - ref).max()
    assert rel <= REL_FRO, f"{what}: relative Frobenius {rel:.3e} > {REL_FRO}"
    assert mx <= bound, f"{what}: max-abs {mx:.3e} > {bound:.3e}"
    return rel


def make_problem(T, K, N, E, seed, offs=None):
    from fp8_microscaling_quantization_b200 import synth
    rng = np.random.default_rng(seed)
    if offs is None:
        offs = synth.zipf_offs(rng, T, E)
    x = synth.to_bf16_bits(rng.standard_normal((T, K), dtype=np.float32))
    w = synth.to_bf16_bits(rng.standard_normal((E, N, K), dtype=np.float32) * np.float32(0.02))
    go = synth.to_bf16_bits(rng.standard_normal((T, N), dtype=np.float32))
    return x, w, go, np.asarray(offs, np.int32)


def full_check(B, oracle, fmt, T, K, N, E, seed, offs=None):
    x, w, go, offs = make_problem(T, K, N, E, seed, offs)
    packed, scales, g = quantize_weights(oracle, fmt, w)
    rows = np.arange(T)
    Wmax = max(np.abs(oracle.dequant_expert_f32(fmt, packed[e], scales[e], None if g is None else g[e])).max()
               for e in range(E))
    for backward, a in ((False, x), (True, go)):
        got, err = run_gemm(B, oracle, fmt, backward, a, packed, scales, g, offs)
        assert err == 0
        ref = oracle.grouped_mm_rows(fmt, backward, a, packed, scales, g, offs, rows)
        end = int(offs[-1])
        assert np.all(got[end:] == 0), "rows past offs[-1] must be zero"
        if end:
            check_rows(got[:end], ref[:end], a, Wmax, N if backward else K,
                       f"fmt={fmt} {'bwd' if backward else 'fwd'} T={T} K={K} N={N} E={E}")


@pytest.mark.parametrize("fmt", [1, 2])
def test_gemm_small_ragged(B, oracle, fmt):
    full_check(B, oracle, fmt, T=300, K=256, N=256, E=4, seed=11)


@pytest.mark.parametrize("fmt", [1, 2])
def test_gemm_mid(B, oracle, fmt):
    full_check(B, oracle, fmt, T=2048, K=1024, N=512, E=8, seed=12)


@pytest.mark.parametrize("fmt", [1, 2])
def test_gemm_edge_offsets(B, oracle, fmt):
    # one expert; empty experts in front, middle and back; a tail of unrouted rows;
    # segments of 1 and 129 rows
    full_check(B, oracle, fmt, T=200, K=256, N=256, E=1, seed=13, offs=[200])
    full_check(B, oracle, fmt, T=400, K=256, N=256, E=6, seed=14, offs=[0, 1, 130, 130, 390, 390])
    full_check(B, oracle, fmt, T=64, K=256, N=256, E=3, seed=15, offs=[0, 0, 0])


@pytest.mark.parametrize("fmt", [1, 2])
def test_gemm_single_ctas(B, oracle, fmt, monkeypatch):
    # BSQ_GMM_CTA_PAIR=0 runs 128-feature x 256-token tiles on single CTAs
    # instead of the default CTA pairs (256 features x 512 tokens,
    # cta_group::2); the same shapes as the default-mode tests
    monkeypatch.setenv("BSQ_GMM_CTA_PAIR", "0")
    full_check(B, oracle, fmt, T=300, K=256, N=256, E=4, seed=11)
    full_check(B, oracle, fmt, T=2048, K=1024, N=512, E=8, seed=12)
    full_check(B, oracle, fmt, T=400, K=256, N=256, E=6, seed=14, offs=[0, 1, 130, 130, 390, 390])
    full_check(B, oracle, fmt, T=300, K=384, N=384, E=3, seed=17)


@pytest.mark.parametrize("fmt", [1, 2])
def test_gemm_output_width_not_256(B, oracle, fmt):
    # output width a multiple of 128 but not of 256 (single CTAs even in the
    # default mode), K not a multiple of 128
    full_check(B, oracle, fmt, T=300, K=384, N=384, E=3, seed=17)


def test_gemm_bad_offs_reported(B, oracle):
    x, w, go, _ = make_problem(256, 256, 256, 4, 16, offs=[0, 0, 0, 0])
    packed, scales, g = quantize_weights(oracle, oracle.FMT_MXFP4, w)
    for offs in ([10, 5, 200, 256], [10, 20, 30, 300], [-1, 5, 6, 7]):
        got, err = run_gemm(B, oracle, oracle.FMT_MXFP4, False, x, packed, scales, g, np.array(offs, np.int32))
        assert err & 1, f"offs {offs} not reported"


def test_gemm_rejects_bad_shapes(B):
    x = torch.zeros((64, 100), dtype=torch.bfloat16, device="cuda")
    p = torch.zeros((2, 256, 50), dtype=torch.uint8, device="cuda")
    s = torch.zeros((2, 256, 3), dtype=torch.uint8, device="cuda")
    offs = torch.tensor([32, 64], dtype=torch.int32, device="cuda")
    with pytest.raises(B.BsqError):
        B.bsq_grouped_mm_fp4(B.Format.MXFP4, B.Direction.FWD, x, p, s, None, offs)
    with pytest.raises(B.BsqError):
        B.bsq_grouped_mm_fp4(B.Format.FP8, B.Direction.FWD, x, p, s, None, offs)


@pytest.mark.parametrize("pair", ["0", "1"])
@pytest.mark.parametrize("fmt", [1, 2])
def test_gemm_full_size_sampled(B, oracle, fmt, pair, monkeypatch):
    """T=16384, K=7168, N=2048, E=32 with Zipf(1.1) routing (one empty expert):
    all rows of the two smallest non-empty experts, the first and last row of
    every expert and 12 seeded rows per expert, forward and backward; single
    CTAs (256-token tiles) and CTA pairs (512-token tiles)."""
    from fp8_microscaling_quantization_b200 import synth
    monkeypatch.setenv("BSQ_GMM_CTA_PAIR", pair)
    prob = synth.moe_problem()
    x, w, go, offs = prob["x"], prob["w"], prob["grad_out"], prob["offs"]
    packed, scales, g = quantize_weights(oracle, fmt, w)
    del w, prob
    starts = np.concatenate([[0], offs[:-1]]).astype(np.int64)
    counts = offs - starts
    rng = np.random.default_rng(99)
    pick = []
    nonempty = np.nonzero(counts > 0)[0]
    for e in nonempty[np.argsort(counts[nonempty])[:2]]:
        pick.append(np.arange(starts[e], offs[e]))
    for e in nonempty:
        pick.append([starts[e], offs[e] - 1])
        pick.append(rng.integers(starts[e], offs[e], 12))
    rows = np.unique(np.concatenate(pick)).astype(np.int64)
    Wmax = 0.0
    for e in range(32):
        Wmax = max(Wmax, np.abs(oracle.dequant_expert_f32(fmt, packed[e], scales[e],
                                                          None if g is None else g[e])).max())
    for backward, a in ((False, x), (True, go)):
        got, err = run_gemm(B, oracle, fmt, backward, a, packed, scales, g, offs)
        assert err == 0
        ref = oracle.grouped_mm_rows(fmt, backward, a, packed, scales, g, offs, rows)
        check_rows(got[rows], ref, a, Wmax, 2048 if backward else 7168,
                   f"full-size fmt={fmt} pair={pair} {'bwd' if backward else 'fwd'}")


@pytest.mark.parametrize("backward", [False, True])
def test_gemm_fused_gate_up_halves(B, oracle, backward):
    """A fused gate/up expert weight [E, 2H, K] quantized as one NVFP4 tensor
    whose rows carry their half's tensor scale (nvfp4 page: per-row scales let
    fused gate/up projections carry the two tensor scales of their halves
    exactly).  Forward applies the per-row scales in the epilogue, backward
    folds them into the dequantized weight (they lie on its contraction)."""
    T, K, H, E = 1200, 512, 256, 5
    x, w, go, offs = make_problem(T, K, 2 * H, E, 21)
    wf = f32(w)
    wf[:, H:] *= np.float32(7.0)  # the up half 7x larger: distinct tensor scales
    from fp8_microscaling_quantization_b200 import synth
    w = synth.to_bf16_bits(wf)
    packed = np.empty((E, 2 * H, K // 2), np.uint8)
    scales = np.empty((E, 2 * H, K // 16), np.uint8)
    g = np.empty((E, 2 * H), np.float32)
    for e in range(E):
        t_gate = np.float32(np.abs(f32(w[e, :H])).max()) / np.float32(2688.0)
        t_up = np.float32(np.abs(f32(w[e, H:])).max()) / np.float32(2688.0)
        assert t_up > 2 * t_gate
        rs = np.concatenate([np.full(H, t_gate, np.float32), np.full(H, t_up, np.float32)])
        packed[e], scales[e], g[e] = oracle.quantize_nvfp4(w[e], row_scale=rs)
        # each half equals its own ModelOpt (per-tensor) quantization
        pg, sg, tg = oracle.quantize_nvfp4_tensor(w[e, :H])
        assert tg == t_gate and np.array_equal(pg, packed[e, :H]) and np.array_equal(sg, scales[e, :H])
    fmt = oracle.FMT_NVFP4
    a = go if backward else x
    got, err = run_gemm(B, oracle, fmt, backward, a, packed, scales, g, offs)
    assert err == 0
    rows = np.arange(T)
    ref = oracle.grouped_mm_rows(fmt, backward, a, packed, scales, g, offs, rows)
    Wmax = max(np.abs(oracle.dequant_expert_f32(fmt, packed[e], scales[e], g[e])).max() for e in range(E))
    end = int(offs[-1])
    assert np.all(got[end:] == 0)
    check_rows(got[:end], ref[:end], a, Wmax, 2 * H if backward else K, f"gate/up {'bwd' if backward else 'fwd'}")
    if not backward:
        # the up half's outputs are ~7x the gate half's: the scales were applied per half
        ratio = np.abs(got[:end, H:]).mean() / np.abs(got[:end, :H]).mean()
        assert 5.0 < ratio < 9.0


@pytest.mark.parametrize("pair", ["0", "1"])
def test_gemm_wait_limit_runs_out_then_recovers(B, oracle, pair, monkeypatch):
    """Every pipeline wait of the GEMM is bounded.  With the limit cut to 1 ns
    (BSQ_GMM_WAIT_NS) the waits run out: the kernel must record
    BSQ_DEVERR_TIMEOUT in the error word and return, and the next call on the
    same stream, with the normal limit, must be correct."""
    import time
    monkeypatch.setenv("BSQ_GMM_CTA_PAIR", pair)
    T, K, N, E = 1024, 512, 256, 4
    x, w, go, offs = make_problem(T, K, N, E, 23)
    fmt = oracle.FMT_MXFP4
    packed, scales, g = quantize_weights(oracle, fmt, w)
    monkeypatch.setenv("BSQ_GMM_WAIT_NS", "1")
    t0 = time.monotonic()
    _, err = run_gemm(B, oracle, fmt, False, x, packed, scales, g, offs)
    assert time.monotonic() - t0 < 60.0
    assert err & 2, f"no timeout reported (err={err})"
    monkeypatch.delenv("BSQ_GMM_WAIT_NS")
    for backward, a in ((False, x), (True, go)):
        got, err = run_gemm(B, oracle, fmt, backward, a, packed, scales, g, offs)
        assert err == 0
        ref = oracle.grouped_mm_rows(fmt, backward, a, packed, scales, g, offs, np.arange(T))
        Wmax = max(np.abs(oracle.dequant_expert_f32(fmt, packed[e], scales[e])).max() for e in range(E))
        end = int(offs[-1])
        check_rows(got[:end], ref[:end], a, Wmax, N if backward else K, "after a timed-out call")
