"""The seeded routing generators behind the grouped-GEMM workloads: the
offsets are valid cumulative counts and each skew has the shape it is named
for.  CPU only."""
import numpy as np
import pytest

from fp8_microscaling_quantization_b200 import synth

T, E = 16384, 32


def counts_of(offs):
    assert offs.dtype == np.int32 and offs.shape == (E,)
    c = np.diff(np.concatenate([[0], offs.astype(np.int64)]))
    assert (c >= 0).all() and offs[-1] == T
    return c


def test_zipf_routing_has_an_empty_expert_and_a_heavy_tail():
    c = counts_of(synth.zipf_offs(np.random.default_rng(20260005), T, E))
    assert (c == 0).sum() >= 1
    assert c.max() > 4 * T / E          # Zipf(1.1): the top expert is far above the mean


@pytest.mark.parametrize("kind", ["uniform", "zipf", "hot", "tiny"])
def test_skews_are_valid_and_seeded(kind):
    a = synth.skew_offs(np.random.default_rng(20260008), kind, T, E)
    b = synth.skew_offs(np.random.default_rng(20260008), kind, T, E)
    assert np.array_equal(a, b)
    counts_of(a)


def test_skew_shapes():
    rng = lambda: np.random.default_rng(20260008)
    u = counts_of(synth.skew_offs(rng(), "uniform", T, E))
    assert u.max() - u.min() <= 1 and u.max() == T // E
    h = counts_of(synth.skew_offs(rng(), "hot", T, E))
    assert h.max() == T // 2
    t = counts_of(synth.skew_offs(rng(), "tiny", T, E))
    small = t[t <= 16]
    assert small.size == E // 2 and (small >= 1).all()
    assert t[t > 16].max() - t[t > 16].min() <= 1
    with pytest.raises(ValueError):
        synth.skew_offs(rng(), "nope", T, E)
