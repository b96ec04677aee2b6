"""Pins of the oracle's scalar building blocks against things other than
itself: numpy's IEEE binary16 conversion, the published Philox known-answer
vectors, an explicit Sylvester Hadamard matrix."""
import numpy as np
import pytest
from scipy.linalg import hadamard

from conftest import golden


def test_f16_from_f32_matches_numpy(orc):
    rng = np.random.default_rng(0)
    vals = np.concatenate([
        rng.standard_normal(4000).astype(np.float32) * np.float32(10.0) ** rng.integers(-9, 6, 4000),
        np.array([0.0, -0.0, 65504.0, 65519.99, 65520.0, 65536.0, -65520.0, 6.1035156e-05,
                  5.9604645e-08, 2.9802322e-08, 2.9802326e-08, 1e-9, np.inf, -np.inf,
                  1.0 + 2 ** -11, 1.0 + 3 * 2 ** -11, 2048.0 + 1.0, 2048.0 + 3.0],
                 dtype=np.float32),
    ]).astype(np.float32)
    ours = orc.f16_from_f32(vals)
    ref = vals.astype(np.float16).view(np.uint16)
    np.testing.assert_array_equal(ours, ref)


def test_f32_from_f16_all_patterns(orc):
    pats = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ours = orc.f32_from_f16(pats)
    ref = pats.view(np.float16).astype(np.float32)
    fin = np.isfinite(ref)
    np.testing.assert_array_equal(ours[fin].view(np.uint32), ref[fin].view(np.uint32))
    assert np.all(np.isnan(ours[np.isnan(ref)]))


def test_philox_known_answers(orc):
    import os
    from conftest import ROOT
    with open(os.path.join(ROOT, "tests", "golden", "philox_kat.txt")) as f:
        rows = [l.split() for l in f if l.strip() and not l.startswith("#")]
    assert len(rows) == 3
    for r in rows:
        vals = [int(x, 16) for x in r]
        out = orc.philox(vals[0:4], vals[4:6])
        assert [int(x) for x in out] == vals[6:10]


@pytest.mark.parametrize("n", [16, 32, 64, 128])
def test_fwht_is_normalised_sylvester(orc, n):
    Hm = hadamard(n).astype(np.float64) / np.sqrt(n)
    np.testing.assert_allclose(Hm @ Hm.T, np.eye(n), atol=1e-15)
    rng = np.random.default_rng(n)
    for _ in range(20):
        x = rng.standard_normal(n).astype(np.float32)
        y = orc.fwht(x)
        ref = Hm @ x.astype(np.float64)
        # FP32 butterflies: error ~ log2(n) ulps of the row norm
        assert np.max(np.abs(y - ref)) <= 8 * np.log2(n) * 2 ** -24 * np.linalg.norm(x)
        z = orc.fwht(y)  # involution
        assert np.max(np.abs(z - x)) <= 16 * np.log2(n) * 2 ** -24 * np.linalg.norm(x)


@pytest.mark.parametrize("n", [16, 32, 64, 128])
def test_hadamard_scale_is_nearest_float(orc, n):
    s = np.float32(orc.hadamard_scale(n))
    exact = 1.0 / np.sqrt(np.float64(n))
    lo, hi = np.nextafter(s, np.float32(0)), np.nextafter(s, np.float32(1))
    assert abs(float(s) - exact) <= abs(float(lo) - exact)
    assert abs(float(s) - exact) <= abs(float(hi) - exact)
