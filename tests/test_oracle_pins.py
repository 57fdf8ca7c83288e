"""Pins of the CPU oracle against facts the pages and the mathematics fix.

Each test checks the oracle against something other than itself: values the
pages print (tests/golden), library routines (torch's float8 / bf16 casts),
closed forms, invariants and brute force on small inputs.  CPU only.
"""
import os

import numpy as np
import pytest
import torch

from conftest import read_golden

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


# ----------------------------------------------------------------- helpers ---

def all_bf16_finite():
    bits = np.arange(1 << 16, dtype=np.uint32)
    f = (bits << 16).view(np.float32)
    return f[np.isfinite(f)]


def e2m1_table_golden(golden_dir):
    rows = read_golden(os.path.join(golden_dir, "e2m1_table.txt"))
    return np.array([float(v) for _, v in rows], dtype=np.float64)


def brute_e2m1(q, table):
    """Nearest of the 8 magnitudes by exhaustive search (float64), ties to the
    even index, sign from the sign bit -- independent of the oracle's midpoint
    counting."""
    # clipping far above 6 keeps the float64 differences exact and cannot
    # change the nearest magnitude
    a = np.minimum(np.abs(q.astype(np.float64)), 1e6)
    mags = table[:8]
    d = np.abs(a[:, None] - mags[None, :])
    best = d.min(axis=1, keepdims=True)
    cand = d == best
    # among tied candidates take the even index
    even = cand & (np.arange(8)[None, :] % 2 == 0)
    idx = np.where(even.any(axis=1), even.argmax(axis=1), cand.argmax(axis=1))
    return (idx | (np.signbit(q) * 8)).astype(np.uint8)


def torch_e4m3(x):
    return torch.from_numpy(np.ascontiguousarray(x, np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def torch_e4m3_decode(codes):
    return torch.from_numpy(np.asarray(codes, np.uint8)).view(torch.float8_e4m3fn).float().numpy()


# ------------------------------------------------------- printed constants ---

def test_page_constants_match_enumeration(oracle, golden_dir):
    c = {r[0]: float(r[1]) for r in read_golden(os.path.join(golden_dir, "page_constants.txt"))}
    vals = np.array([oracle.e4m3_val(k) for k in range(128)])
    finite = vals[np.isfinite(vals)]
    assert finite.max() == c["E4M3_MAX"] == c["MAXBOUND_E4M3"]
    assert np.isnan(vals[0x7F])
    pos = finite[finite > 0]
    assert pos.min() == c["E4M3_MIN_SUBNORMAL"]
    # smallest subnormal = smallest normal / 8 (ModelOpt _FP8_E4M3_MIN_POSITIVE)
    smallest_normal = min(oracle.e4m3_val(k) for k in range(8, 127))
    assert pos.min() == smallest_normal / 8
    e2m1 = np.array([oracle.e2m1_val(k) for k in range(16)])
    assert e2m1.max() == c["E2M1_MAX"] == c["MAXBOUND_E2M1_WITH_E4M3_SCALE"]
    assert c["NVFP4_BLOCK_SIZE"] == 16 and c["MXFP4_BLOCK_SIZE"] == 32


def test_e2m1_table_and_midpoints_printed(oracle, golden_dir):
    table = e2m1_table_golden(golden_dir)
    got = np.array([oracle.e2m1_val(k) for k in range(16)])
    assert np.array_equal(got, table)
    assert not np.signbit(got[8]), "the printed table holds 0.0 at code 8"
    mids = np.array([float(r[0]) for r in read_golden(os.path.join(golden_dir, "e2m1_midpoints.txt"))])
    # each printed midpoint is the mean of two adjacent magnitudes
    assert np.array_equal(mids, (table[:7] + table[1:8]) / 2)


def test_byte_table_and_nibble_order(oracle, golden_dir):
    """All 256 packed bytes decode to (TABLE[b & 15], TABLE[b >> 4]) with the
    even column in the low nibble (mxfp4 page _FP4_BYTE_TABLE; nvfp4 page
    module text)."""
    table = e2m1_table_golden(golden_dir)
    packed = np.arange(256, dtype=np.uint8).reshape(8, 32)      # rows of K=64
    scales = np.full((8, 2), 127, np.uint8)                     # 2**0
    y = oracle.dequantize_mxfp4(packed, scales, out_dtype=oracle.F32).reshape(-1)
    b = np.arange(256)
    assert np.array_equal(y[0::2], table[b & 15].astype(np.float32))
    assert np.array_equal(y[1::2], table[b >> 4].astype(np.float32))


# ------------------------------------------------------------- rounding -------

def test_e2m1_round_matches_bruteforce_all_bf16(oracle, golden_dir):
    table = e2m1_table_golden(golden_dir)
    q = all_bf16_finite()
    assert np.array_equal(oracle.e2m1_round(q), brute_e2m1(q, table))


def test_e2m1_round_ties_and_neighbours(oracle, golden_dir):
    table = e2m1_table_golden(golden_dir)
    pts = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 0.5, 1, 1.5, 2, 3, 4, 6, 0, 7, 1e30], np.float32)
    q = [pts]
    for k in range(1, 4):
        q.append(np.nextafter(pts, np.float32(np.inf)))
        q.append(np.nextafter(pts, np.float32(-np.inf)))
        pts = q[-2]
    q = np.concatenate(q)
    q = np.concatenate([q, -q])
    rng = np.random.default_rng(7)
    r = rng.uniform(-8, 8, 2_000_000).astype(np.float32)
    tiny = (rng.integers(1, 1 << 23, 10000).astype(np.uint32)).view(np.float32)  # subnormals
    q = np.concatenate([q, r, tiny, -tiny, np.array([0.0, -0.0], np.float32)])
    got = oracle.e2m1_round(q)
    assert np.array_equal(got, brute_e2m1(q, table))
    # explicit ties: half to even
    ties = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0], np.float32)
    assert list(oracle.e2m1_round(ties)) == [0, 2, 2, 4, 4, 6, 6]
    assert list(oracle.e2m1_round(np.array([-0.0, -0.1, 100.0, -100.0], np.float32))) == [8, 8, 7, 15]


def test_e4m3_decode_matches_torch_all_codes(oracle):
    codes = np.arange(256, dtype=np.uint8)
    ours = np.array([oracle.e4m3_val(int(c)) for c in codes], np.float32)
    ref = torch_e4m3_decode(codes)
    both_nan = np.isnan(ours) & np.isnan(ref)
    assert np.array_equal(np.where(both_nan, 0, ours), np.where(both_nan, 0, ref))
    assert both_nan.sum() == 2  # 0x7F and 0xFF


def test_e4m3_round_matches_torch_cast(oracle):
    """torch's CPU float8_e4m3fn cast is round-to-nearest-even and agrees with
    saturation below 464 (above it torch returns NaN; the oracle saturates)."""
    f = all_bf16_finite()
    rng = np.random.default_rng(11)
    r = np.concatenate([rng.uniform(-464, 464, 2_000_000), rng.uniform(-1e-2, 1e-2, 500_000),
                        rng.uniform(-2 ** -6, 2 ** -6, 500_000)]).astype(np.float32)
    x = np.concatenate([f, r])
    inside = np.abs(x) < 464
    got = oracle.e4m3_round(x[inside])
    ref = torch_e4m3(x[inside])
    assert np.array_equal(got, ref)
    big = x[~inside]
    got_big = oracle.e4m3_round(big)
    assert np.all((got_big & 0x7F) == 0x7E)
    assert np.array_equal(got_big >> 7, np.signbit(big).astype(np.uint8))


def test_e4m3_round_ties_all_codes(oracle):
    """Every midpoint between adjacent positive e4m3 values goes to the even code."""
    vals = np.array([oracle.e4m3_val(k) for k in range(0x7F)], np.float64)
    mids = ((vals[:-1] + vals[1:]) / 2).astype(np.float32)
    assert np.array_equal(mids.astype(np.float64), (vals[:-1] + vals[1:]) / 2)  # exact in fp32
    got = oracle.e4m3_round(mids)
    lower = np.arange(0x7E)
    expect = np.where(lower % 2 == 0, lower, lower + 1)
    assert np.array_equal(got, expect.astype(np.uint8))


def test_bf16_rounding_matches_torch(oracle):
    rng = np.random.default_rng(3)
    bits = rng.integers(0, 1 << 32, 4_000_000, dtype=np.uint64).astype(np.uint32)
    # half-way cases and their neighbours
    tie = (rng.integers(0, 1 << 16, 200_000, dtype=np.uint32) << 16) | 0x8000
    bits = np.concatenate([bits, tie, tie + 1, tie - 1, np.array([0x7F7FFFFF, 0x7F7F8000, 0x00008000, 0x80018000], np.uint32)])
    x = bits.view(np.float32)
    x = x[~np.isnan(x)]
    ours = oracle.f32_to_bf16(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)


def test_e8m0_all_codes(oracle):
    codes = np.arange(256)
    ours = np.array([oracle.e8m0_val(int(c)) for c in codes], np.float32)
    assert np.isnan(ours[255])
    assert np.array_equal(ours[:255], np.ldexp(np.float32(1), codes[:255] - 127).astype(np.float32))
    if hasattr(torch, "float8_e8m0fnu"):
        ref = torch.from_numpy(codes.astype(np.uint8)).view(torch.float8_e8m0fnu).float().numpy()
        assert np.array_equal(ours[:255], ref[:255])


def test_floor_log2_exact(oracle):
    f = all_bf16_finite()
    rng = np.random.default_rng(5)
    bits = rng.integers(1, 0x7F800000, 4_000_000, dtype=np.uint32)
    a = np.concatenate([f[f > 0], bits.view(np.float32)])
    pw = np.ldexp(np.float32(1), np.arange(-149, 128)).astype(np.float32)
    a = np.concatenate([a, pw, np.nextafter(pw, np.float32(0)), np.nextafter(pw, np.float32(np.inf))])
    a = a[(a > 0) & np.isfinite(a)]
    e = oracle.floor_log2(a).astype(np.int64)
    a64 = a.astype(np.float64)
    assert np.all(np.ldexp(1.0, e) <= a64)
    assert np.all(a64 < np.ldexp(1.0, e + 1))


def test_pow2_ceil_positive_normals(oracle):
    """Positive normal binary32 values map to a power of two p with a <= p < 2a:
    every pattern of the lowest, the highest and the unit binades, and every
    61st pattern of the whole positive normal range."""
    full = [np.arange(0x00800000, 0x01000000, dtype=np.uint32),       # [2**-126, 2**-125)
            np.arange(0x3F000000, 0x3F800000, dtype=np.uint32),       # [0.5, 1)
            np.arange(0x3F800000, 0x40000000, dtype=np.uint32),       # [1, 2)
            np.arange(0x7F000000, 0x7F800000, dtype=np.uint32)]       # [2**127, 2**128)
    strided = np.arange(0x00800000, 0x7F800000, 61, dtype=np.uint32)
    for bits in full + [strided]:
        a = bits.view(np.float32)
        p = oracle.pow2_ceil(a)
        finite = np.isfinite(p)
        # only values above 2**127 round up past the binary32 range
        assert np.all(finite | (a > np.float32(2.0 ** 127)))
        pf, af = p[finite], a[finite]
        assert np.all((pf.view(np.uint32) & 0x007FFFFF) == 0)      # a power of two
        assert np.all(pf >= af)
        assert np.all(pf * np.float32(0.5) < af)                   # p/2 is exact


# ------------------------------------------------------------- NVFP4 --------

def test_nvfp4_decode_is_product_of_three(oracle):
    """decode = e2m1 * e4m3 * fp32 with binary32 intermediates and one final
    rounding: the exact float64 triple product rounded once."""
    codes = np.arange(16, dtype=np.uint8)
    sc = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], np.uint8)
    rng = np.random.default_rng(9)
    gs = np.concatenate([[1.0, 2 ** -20, 3.7e-5], rng.uniform(1e-6, 1e-2, 5)]).astype(np.float32)
    # rows: one per (scale code, g); K = 16 columns = all 16 codes, twice
    packed_row = (codes[0::2] | (codes[1::2] << 4)).astype(np.uint8)
    table = np.array([oracle.e2m1_val(k) for k in range(16)], np.float64)
    for g in gs:
        packed = np.tile(np.concatenate([packed_row, packed_row]), (sc.size, 1))
        scales = np.stack([sc, sc], axis=1)
        y32 = oracle.dequantize_nvfp4(packed, scales, np.full(sc.size, g, np.float32), out_dtype=oracle.F32)
        yb = oracle.dequantize_nvfp4(packed, scales, np.full(sc.size, g, np.float32), out_dtype=oracle.BF16)
        s64 = torch_e4m3_decode(sc).astype(np.float64)
        exact = (np.tile(table, 2)[None, :] * s64[:, None]) * np.float64(g)
        ref32 = exact.astype(np.float32)
        assert np.array_equal(y32, ref32)
        refb = torch.from_numpy(ref32).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
        assert np.array_equal(yb, refb)


def _synth():
    from fp8_microscaling_quantization_b200 import synth
    return synth


def test_nvfp4_storage_cost(oracle):
    s = _synth()
    x = s.nvfp4_matrix(rows=64, cols=2048)
    packed, scales, g = oracle.quantize_nvfp4(x)
    nbytes = packed.nbytes + scales.nbytes + g.nbytes
    assert nbytes == 0.5625 * x.size + 4 * x.shape[0]


def test_nvfp4_scale_rule_properties(oracle):
    s = _synth()
    x = s.nvfp4_matrix(rows=256, cols=2048)
    packed, scales, g = oracle.quantize_nvfp4(x)
    xf = s.bf16_bits_to_f32(x)
    amax = np.abs(xf).max(axis=1)
    assert np.array_equal(g, (amax / np.float32(2688.0)).astype(np.float32))
    assert np.all(scales <= 0x7E)
    # the block holding the row maximum takes scale 448 (0x7E)
    blk = np.abs(xf).argmax(axis=1) // 16
    assert np.all(scales[np.arange(256), blk] == 0x7E)
    # every block scale is the e4m3 value nearest (amax_b/6)/g, floored at 2**-9
    amax_b = np.abs(xf.reshape(256, -1, 16)).max(axis=2)
    t = np.maximum((amax_b / np.float32(6)) / g[:, None], np.float32(2 ** -9)).astype(np.float32)
    assert np.array_equal(scales, torch_e4m3(t))


def test_nvfp4_codes_are_nearest_given_scales(oracle, golden_dir):
    """Given the block scales, each code is the nearest e2m1 value to
    x / (scale * g) (brute force over the 16 codes)."""
    table = e2m1_table_golden(golden_dir)
    s = _synth()
    x = s.nvfp4_matrix(rows=32, cols=256, seed=123)
    packed, scales, g = oracle.quantize_nvfp4(x)
    xf = s.bf16_bits_to_f32(x).reshape(32, -1, 16)
    d = (torch_e4m3_decode(scales).astype(np.float32) * g[:, None]).astype(np.float32)
    q = (xf / d[:, :, None]).astype(np.float32).reshape(-1)
    codes = np.stack([packed & 15, packed >> 4], axis=-1).reshape(-1)
    assert np.array_equal(codes, brute_e2m1(q, table))


def test_nvfp4_gate_up_and_modelopt_equivalence(oracle):
    """Per-row storage of the tensor scale carries two halves' tensor scales
    exactly (nvfp4 page module text): quantizing the concatenation with the
    halves' tensor scales per row equals the halves' ModelOpt outputs."""
    s = _synth()
    gate = s.linear_weight(out=64, inp=512, seed=41)
    up = s.linear_weight(out=64, inp=512, seed=42)
    pg, sg, tg = oracle.quantize_nvfp4_tensor(gate)
    pu, su, tu = oracle.quantize_nvfp4_tensor(up)
    cat = np.concatenate([gate, up], axis=0)
    rs = np.concatenate([np.full(64, tg, np.float32), np.full(64, tu, np.float32)])
    pc, sc, gc = oracle.quantize_nvfp4(cat, row_scale=rs)
    assert np.array_equal(pc, np.concatenate([pg, pu]))
    assert np.array_equal(sc, np.concatenate([sg, su]))
    assert np.array_equal(gc, rs)
    # ModelOpt tensor scale = amax(tensor) / (6 * 448)
    amax = np.abs(s.bf16_bits_to_f32(gate)).max()
    assert tg == np.float32(amax / np.float32(2688.0))


def test_nvfp4_zero_row_and_zero_block(oracle):
    x = np.zeros((2, 32), np.uint16)
    x[1, :16] = 0x3F80  # 1.0 in the first block, zeros in the second
    packed, scales, g = oracle.quantize_nvfp4(x)
    assert g[0] == 0 and np.all(scales[0] == 0) and np.all(packed[0] == 0)
    assert scales[1, 1] == 0x01  # zero block: scale floored at 2**-9
    assert np.all(packed[1, 8:] == 0)
    y = oracle.dequantize_nvfp4(packed, scales, g, out_dtype=oracle.F32)
    assert np.all(y[0] == 0) and np.all(y[1, 16:] == 0)
    assert np.all(y[1, :16] == 1.0)


def test_nvfp4_rejects_ragged_k(oracle):
    with pytest.raises(ValueError):
        oracle.quantize_nvfp4(np.zeros((2, 24), np.uint16))


# ------------------------------------------------------------- MXFP4 --------

def test_mxfp4_value_exact_round_trip(oracle):
    """Values already exactly representable round-trip value-exactly (mxfp4
    page, quantize_mxfp4): random codes and every finite scale code, over
    2**20 blocks in binary32 and 2**15 in bf16."""
    rng = np.random.default_rng(13)
    R, K = 32768, 1024
    packed = rng.integers(0, 256, (R, K // 2), dtype=np.uint8)
    # scale codes 253 and 254 push 4 * 2**126 and above past the binary32
    # range (inf is not a representable value), so the claim covers codes 0..252
    scales = rng.integers(0, 253, (R, K // 32), dtype=np.uint8)
    y = oracle.dequantize_mxfp4(packed, scales, out_dtype=oracle.F32)
    assert np.all(np.isfinite(y))
    p2, s2 = oracle.quantize_mxfp4(y)
    y2 = oracle.dequantize_mxfp4(p2, s2, out_dtype=oracle.F32)
    assert np.array_equal(y, y2)
    packed, scales = packed[:2048, :256], scales[:2048, :16]
    yb = oracle.dequantize_mxfp4(packed, scales, out_dtype=oracle.BF16)
    p3, s3 = oracle.quantize_mxfp4(yb)
    assert np.array_equal(oracle.dequantize_mxfp4(p3, s3, out_dtype=oracle.BF16), yb)


def test_mxfp4_exponent_rule(oracle):
    """scale = 2**(floor(log2(amax)) - 2): the block maximum lands in [4, 8)
    before e2m1 rounding; all-zero blocks take code 0."""
    s = _synth()
    x = s.expert_weights(E=2, N=64, K=512, zero_blocks=8, seed=77)
    packed, scales = oracle.quantize_mxfp4(x)
    xf = s.bf16_bits_to_f32(x).reshape(-1, 32)
    amax = np.abs(xf).max(axis=1)
    e = scales.reshape(-1).astype(np.int64) - 127
    nz = amax > 0
    ratio = amax[nz].astype(np.float64) / np.ldexp(1.0, e[nz])
    assert np.all((ratio >= 4) & (ratio < 8))
    assert np.all(scales.reshape(-1)[~nz] == 0)
    assert (~nz).sum() == 16


# ------------------------------------------------------- paged KV cache ----

def test_kv_cache_layout_and_values(oracle, golden_dir):
    """Output [1, blocks * block_tokens, heads, 128]: element (b * bt + t, h, d)
    is code d of row t * heads + h of block b, times that row's e4m3 scale for
    column d // 16, times the block's amax / 2688 -- assembled here from the
    printed e2m1 table, torch's e4m3 decode and binary32 products."""
    rng = np.random.default_rng(71)
    nb, bt, heads = 5, 4, 3
    rows = bt * heads
    vals = [rng.integers(0, 256, (rows, 64), dtype=np.uint8) for _ in range(nb)]
    scs = []
    for _ in range(nb):
        sc = rng.integers(0, 127, (rows, 8), dtype=np.uint8)  # finite, non-negative e4m3
        scs.append(sc)
    amax = np.array([2688.0, 1.0, 0.0, 3.5e5, 7e-3], np.float32)
    table = e2m1_table_golden(golden_dir).astype(np.float32)
    for dt in (oracle.BF16, oracle.F32):
        y = oracle.dequantize_kv_cache_nvfp4(vals, scs, amax, bt, heads, out_dtype=dt)
        assert y.shape == (1, nb * bt, heads, 128)
        yf = oracle.bf16_to_f32(y) if dt == oracle.BF16 else y
        for b in range(nb):
            g = np.float32(amax[b]) / np.float32(2688.0)
            codes = np.stack([vals[b] & 15, vals[b] >> 4], axis=-1).reshape(rows, 128)
            e2 = np.where(codes >= 8, -1.0, 1.0).astype(np.float32) * table[codes & 7]
            sv = np.repeat(torch_e4m3_decode(scs[b]).astype(np.float32), 16, axis=1)
            want = (e2 * sv).astype(np.float32) * g
            if dt == oracle.BF16:
                want = oracle.bf16_to_f32(oracle.f32_to_bf16(want))
            got = yf[0, b * bt:(b + 1) * bt].reshape(rows, 128)  # row = t * heads + h
            assert np.array_equal(got, want), (b, dt)


# ------------------------------------------------- static two-level NVFP4 --

def _block_amax(xf, block=16):
    return np.abs(xf.reshape(-1, block)).max(axis=1).astype(np.float32)


def test_nvfp4_static_reduces_to_per_row_nvfp4(oracle):
    """With the block amax calibrated to the data and a global amax of
    2688 * 2**k (so A/6 and 448/(A/6) are exact), the static two-level rule
    is the NVFP4 rule with row scale g = 2**k: bit-identical to the pinned
    quantize_nvfp4(x, row_scale=2**k) -> dequantize_nvfp4 round trip."""
    s = _synth()
    x = s.nvfp4_matrix(rows=64, cols=512, seed=91)
    xf = s.bf16_bits_to_f32(x)
    for k in (-6, 0, 3):
        A = np.float32(2688.0 * 2.0 ** k)
        y = oracle.fake_quantize_nvfp4_static(x, _block_amax(xf), A)
        p, sc, g = oracle.quantize_nvfp4(x, row_scale=np.float32(2.0 ** k))
        assert np.array_equal(y, oracle.dequantize_nvfp4(p, sc, g)), k
        y32 = oracle.fake_quantize_nvfp4_static(xf, _block_amax(xf), A)
        assert np.array_equal(y32, oracle.dequantize_nvfp4(*oracle.quantize_nvfp4(xf, row_scale=np.float32(2.0 ** k)),
                                                           out_dtype=oracle.F32)), k


def test_nvfp4_static_is_nearest_multiple(oracle, golden_dir):
    """Every output is the nearest of the 16 e2m1 values times the block's
    physical scale (brute force in float64, ties to the even code, values past
    6 saturate), for calibrated amax below, at and above the data's."""
    s = _synth()
    x = s.nvfp4_matrix(rows=32, cols=256, seed=92)
    xf = s.bf16_bits_to_f32(x)
    table = e2m1_table_golden(golden_dir)
    rng = np.random.default_rng(93)
    amax = _block_amax(xf) * rng.choice([0.25, 1.0, 3.0], size=xf.size // 16).astype(np.float32)
    A = np.float32(np.abs(xf).max() * 1.5)
    y = oracle.fake_quantize_nvfp4_static(xf, amax, A)
    sq = np.array([oracle.nvfp4_static_scale(a, A)[0] for a in amax], np.float64)
    q = (xf.reshape(-1, 16).astype(np.float64) / sq[:, None]).astype(np.float32)
    codes = brute_e2m1(q.reshape(-1), table).reshape(-1, 16)
    vals = np.where(codes >= 8, -1.0, 1.0) * table[codes & 7]
    want = (vals * sq[:, None]).astype(np.float32)
    assert np.array_equal(y.reshape(-1, 16), want)
    # calibrated amax at a quarter of the data's: the block maxima saturate
    low = amax < _block_amax(xf)
    assert np.all(np.abs(y.reshape(-1, 16)[low]).max(axis=1) == (6.0 * sq[low]).astype(np.float32))


def test_nvfp4_static_scale_floor_and_range(oracle):
    """The physical scale is within e4m3 precision of amax/6, never below the
    e4m3 floor 2**-9 * A/2688, and a zero amax lands exactly on that floor."""
    rng = np.random.default_rng(94)
    A = np.float32(37.5)
    unit = np.float64(A) / 6 / 448
    for a in np.exp(rng.uniform(np.log(1e-6), np.log(37.5), 2000)).astype(np.float32):
        sq, code = oracle.nvfp4_static_scale(a, A)
        assert sq >= 2.0 ** -9 * unit * (1 - 1e-6)
        if np.float64(a) / 6 >= 2.0 ** -6 * unit:  # the e4m3 normal range: 3 mantissa bits
            assert abs(sq / (np.float64(a) / 6) - 1) <= 2.0 ** -4 * (1 + 1e-6)
    sq0, code0 = oracle.nvfp4_static_scale(0.0, A)
    assert code0 == 1 and abs(sq0 / (2.0 ** -9 * unit) - 1) < 1e-6
    # a zero global amax falls back to the 1e-8 per-tensor floor
    sqz, codez = oracle.nvfp4_static_scale(0.0, 0.0)
    assert codez == 1 and abs(sqz / (2.0 ** -9 * 1e-8 / 448) - 1) < 1e-6


# ------------------------------------------------------------- MXFP8 --------

def _mxfp8_requant_closed_form(y):
    """What requantizing e4m3 * 2**k values must give, from the rule alone:
    the block maximum m = s * 2**f moves to s * 2**(f - e) with the block
    exponent e = max(f - 8, -127) (s * 256 unless the e8m0 floor binds); e4m3
    holds every 4-bit significand up to 448 = 1.75 * 256, so every value
    returns exactly except values above 448 * 2**e (significand 1.875 at the
    block's top exponent), which saturate to +-448 * 2**e."""
    yb = y.astype(np.float64).reshape(-1, 32)
    m = np.abs(yb).max(axis=1, keepdims=True)
    f = np.floor(np.log2(np.where(m > 0, m, 1.0)))
    cap = 448.0 * np.exp2(np.maximum(f - 8, -127))
    return np.where(np.abs(yb) > cap, np.sign(yb) * cap, yb).reshape(y.shape)


def test_mxfp8_round_trip_closed_form(oracle):
    """e4m3 values times an e8m0 scale, quantized again: exact, except the
    block-top values with significand 1.875, which saturate to 1.75 * 2**f."""
    rng = np.random.default_rng(31)
    R, K = 1024, 512
    codes = rng.integers(0, 256, (R, K), dtype=np.uint8)
    codes[(codes & 0x7F) == 0x7F] = 0x01  # no NaN codes
    # scale codes up to 246 keep 448 * 2**(code - 127) finite in binary32
    scales = rng.integers(0, 247, (R, K // 32), dtype=np.uint8)
    y = oracle.dequantize_mxfp8(codes, scales, out_dtype=oracle.F32)
    assert np.all(np.isfinite(y))
    # the dequantized values are exactly e4m3 * 2**k (torch's e4m3 decode)
    ref = torch_e4m3_decode(codes).astype(np.float64) * np.ldexp(1.0, np.repeat(scales.astype(np.int64) - 127, 32, axis=1))
    assert np.array_equal(y.astype(np.float64), ref)
    c2, s2 = oracle.quantize_mxfp8(y)
    y2 = oracle.dequantize_mxfp8(c2, s2, out_dtype=oracle.F32).astype(np.float64)
    expect = _mxfp8_requant_closed_form(y)
    assert np.array_equal(y2, expect)
    assert (y2 != y).any() and (y2 == y).mean() > 0.99  # both cases occur
    # bf16 holds e4m3 * 2**k exactly above its subnormal floor
    yb_scales = np.maximum(scales, 20)
    yb = oracle.dequantize_mxfp8(codes, yb_scales, out_dtype=oracle.BF16)
    c3, s3 = oracle.quantize_mxfp8(yb)
    yb2 = oracle.f32_to_bf16(oracle.dequantize_mxfp8(c3, s3, out_dtype=oracle.F32))
    assert np.array_equal(yb2, oracle.dequantize_mxfp8(c3, s3, out_dtype=oracle.BF16))
    assert np.array_equal(oracle.bf16_to_f32(yb2).astype(np.float64),
                          _mxfp8_requant_closed_form(oracle.bf16_to_f32(yb)))


def test_mxfp8_exponent_rule_and_saturation(oracle):
    """scale = 2**(floor(log2(amax)) - 8): the block maximum lands in
    [256, 512) before rounding; values above 448 saturate to +-448; the codes
    below that are torch's e4m3 cast of x / scale; all-zero blocks take
    scale code 0."""
    s = _synth()
    x = s.expert_weights(E=2, N=64, K=512, zero_blocks=8, seed=78)
    codes, scales = oracle.quantize_mxfp8(x)
    xf = s.bf16_bits_to_f32(x).reshape(-1, 32)
    amax = np.abs(xf).max(axis=1)
    e = scales.reshape(-1).astype(np.int64) - 127
    nz = amax > 0
    ratio = amax[nz].astype(np.float64) / np.ldexp(1.0, e[nz])
    assert np.all((ratio >= 256) & (ratio < 512))
    assert np.all(scales.reshape(-1)[~nz] == 0) and (~nz).sum() == 16
    q = (xf.astype(np.float64) / np.ldexp(1.0, e)[:, None]).astype(np.float32)
    c = codes.reshape(-1, 32)
    big = np.abs(q) > 448
    assert big.any()  # the rule does saturate on this data
    assert np.all(c[big] == np.where(q[big] > 0, 0x7E, 0xFE))
    assert np.array_equal(c[~big], torch_e4m3(q[~big]))
    # a block at exactly 500 and 448: both store 448
    blk = np.zeros((1, 32), np.float32)
    blk[0, 0], blk[0, 1] = 500.0, -448.0
    cb, sb = oracle.quantize_mxfp8(blk)
    assert sb[0, 0] == 127 and cb[0, 0] == 0x7E and cb[0, 1] == 0xFE


# ------------------------------------------------------------- FP8 ----------

def test_fp8_pow2_scale_rule(oracle):
    s = _synth()
    x, _ = s.cache_acts(B=1, T=64, C=512, seed=21)
    for block in (16, 32):
        codes, scales = oracle.quantize_fp8(x, block=block)
        xf = s.bf16_bits_to_f32(x).reshape(-1, block)
        amax = np.abs(xf).max(axis=1).astype(np.float64)
        p = np.ldexp(1.0, scales.reshape(-1).astype(np.int64) - 127)
        r = amax / p
        assert np.all((r > 224) & (r <= 448))  # amax/448 <= p < 2*amax/448
        assert not np.any((codes & 0x7F) == 0x7F)
        # codes are the torch e4m3 cast of x / p (no saturation happens)
        assert np.array_equal(codes.reshape(-1, block), torch_e4m3((xf / p[:, None]).astype(np.float32)))


# ------------------------------------------------------------- cache --------

@pytest.mark.parametrize("fmt,block", [(0, 32), (1, 32), (2, 16), (0, 16), (1, 16), (2, 32)])
def test_cache_partial_group_is_zero_padding(oracle, fmt, block):
    """A final partial group is zero-padded internally: equal to padding with
    zeros outside and slicing the result back."""
    s = _synth()
    x, _ = s.cache_acts(B=2, T=16, C=520, seed=31)
    y = oracle.quantize_cache(x, fmt, block)
    P = -(-520 // block) * block
    xp = np.zeros((2, 16, P), np.uint16)
    xp[..., :520] = x
    yp = oracle.quantize_cache(xp, fmt, block)
    assert np.array_equal(y, yp[..., :520])


def test_cache_fp8_equals_stored_round_trip(oracle):
    s = _synth()
    x, _ = s.cache_acts(B=1, T=32, C=512, seed=32)
    y = oracle.quantize_cache(x, oracle.FMT_FP8, 32)
    codes, scales = oracle.quantize_fp8(x, 32)
    assert np.array_equal(y, oracle.dequantize_fp8(codes, scales, 32, out_dtype=oracle.BF16))


def test_cache_nvfp4_equals_per_row_round_trip(oracle):
    s = _synth()
    x, _ = s.cache_acts(B=1, T=32, C=512, seed=33)
    y = oracle.quantize_cache(x, oracle.FMT_NVFP4, 16)
    p, sc, g = oracle.quantize_nvfp4(x)
    assert np.array_equal(y, oracle.dequantize_nvfp4(p, sc, g, out_dtype=oracle.BF16))


def test_cache_mxfp4_pow2_ceiling_scale(oracle, golden_dir):
    """mxfp4 cache reading: scale pow2ceil(amax/6), so no value saturates and
    each output is a representable e2m1 value times that scale, the nearest
    one to the input."""
    table = e2m1_table_golden(golden_dir)
    s = _synth()
    x, _ = s.cache_acts(B=1, T=64, C=128, seed=34)
    y = s.bf16_bits_to_f32(oracle.quantize_cache(x, oracle.FMT_MXFP4, 32)).reshape(-1, 32).astype(np.float64)
    xf = s.bf16_bits_to_f32(x).reshape(-1, 32).astype(np.float64)
    amax = np.abs(xf).max(axis=1)
    p = np.exp2(np.ceil(np.log2(np.maximum(amax / 6, 2.0 ** -126))))
    q = y / p[:, None]
    assert np.all(np.isin(np.abs(q), table[:8]))
    mags = table[:8]
    err = np.abs(np.abs(xf / p[:, None])[..., None] - mags).min(axis=-1)
    assert np.allclose(np.abs(np.abs(xf / p[:, None]) - np.abs(q)), err)


def test_cache_backward_is_identity(oracle):
    s = _synth()
    _, g = s.cache_acts(B=2, T=64, C=520, seed=35)
    out = oracle.quantize_cache_backward(g)
    assert out.dtype == g.dtype and np.array_equal(out.view(np.uint16), g.view(np.uint16))


def test_cache_does_not_modify_input(oracle):
    s = _synth()
    x, _ = s.cache_acts(B=1, T=8, C=64, seed=36)
    x0 = x.copy()
    oracle.quantize_cache(x, oracle.FMT_NVFP4, 16)
    assert np.array_equal(x, x0)


# --------------------------------------------------------- grouped GEMM -----

def test_grouped_mm_reference_segments(oracle):
    """Segment handling: expert e's weight is 6 * 2**e * I, exact in both
    formats (NVFP4 with a given row scale of 1), so every row of segment e
    equals 6 * 2**e * x; the empty expert owns no row and rows past offs[-1]
    are zero.  Checked for both formats and directions."""
    E, N, K = 4, 64, 64
    offs = np.array([5, 5, 17, 20], np.int32)   # expert 1 empty; T=24 leaves 4 tail rows
    T = 24
    rng = np.random.default_rng(1)
    from fp8_microscaling_quantization_b200 import synth
    x = synth.to_bf16_bits(rng.standard_normal((T, K), dtype=np.float32))
    c = [6.0 * 2 ** e for e in range(E)]
    W = np.zeros((E, N, K), np.float32)
    for e in range(E):
        W[e] = np.eye(N, K) * c[e]
    Wb = synth.to_bf16_bits(W)
    for fmt in (oracle.FMT_MXFP4, oracle.FMT_NVFP4):
        if fmt == oracle.FMT_MXFP4:
            packed, scales = oracle.quantize_mxfp4(Wb)
            rs = None
        else:
            packed, scales, rs = oracle.quantize_nvfp4(Wb, row_scale=np.ones((E, N), np.float32))
        for e in range(E):
            assert np.array_equal(oracle.dequant_expert_f32(fmt, packed[e], scales[e],
                                                            None if rs is None else rs[e]), W[e])
        xf = synth.bf16_bits_to_f32(x).astype(np.float64)
        starts = [0, 5, 5, 17]
        for bwd in (False, True):
            ref = oracle.grouped_mm_rows(fmt, bwd, x, packed, scales, rs, offs, np.arange(T))
            for e in range(E):
                for t in range(starts[e], offs[e]):
                    assert np.array_equal(ref[t], xf[t] * c[e])
            assert np.all(ref[20:] == 0)


def test_grouped_mm_reference_bruteforce_small(oracle):
    """Tiny random problem: the reference equals a plain triple loop."""
    from fp8_microscaling_quantization_b200 import synth
    rng = np.random.default_rng(2)
    E, N, K, T = 2, 8, 32, 6
    offs = np.array([2, 6], np.int32)
    w = synth.to_bf16_bits(rng.standard_normal((E, N, K), dtype=np.float32))
    packed, scales = oracle.quantize_mxfp4(w)
    x = synth.to_bf16_bits(rng.standard_normal((T, K), dtype=np.float32))
    go = synth.to_bf16_bits(rng.standard_normal((T, N), dtype=np.float32))
    fwd = oracle.grouped_mm_rows(oracle.FMT_MXFP4, False, x, packed, scales, None, offs, np.arange(T))
    bwd = oracle.grouped_mm_rows(oracle.FMT_MXFP4, True, go, packed, scales, None, offs, np.arange(T))
    xf, gf = synth.bf16_bits_to_f32(x), synth.bf16_bits_to_f32(go)
    Wd = [oracle.dequantize_mxfp4(packed[e], scales[e], out_dtype=oracle.F32) for e in range(E)]
    for t in range(T):
        e = 0 if t < 2 else 1
        for n in range(N):
            acc = 0.0
            for k in range(K):
                acc += float(xf[t, k]) * float(Wd[e][n, k])
            assert fwd[t, n] == pytest.approx(acc, rel=1e-12, abs=1e-12)
        for k in range(K):
            acc = 0.0
            for n in range(N):
                acc += float(gf[t, n]) * float(Wd[e][n, k])
            assert bwd[t, k] == pytest.approx(acc, rel=1e-12, abs=1e-12)
