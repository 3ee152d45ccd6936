"""Pins for the oracle's normal quantile function and NF4 codebook.

The codebook construction is described in prose only: levels from standard
normal quantiles of equal-probability pieces, normalised to [-1, 1], with the
two halves built asymmetrically so that 0 is an exact level ("QLoRA：用4比特行李箱装下整个大模型"
chapter 3; bitsandbytes article (CSDN) section 6.2).  These tests pin the
oracle's Phi^-1 against scipy and textbook values, and the codebook against
the properties the pages state plus an independent scipy construction.
"""
import math

import numpy as np
import pytest
from scipy.stats import norm


def test_ppf_textbook_values(orc):
    assert orc.normal_ppf(0.5) == pytest.approx(0.0, abs=1e-15)
    assert orc.normal_ppf(0.975) == pytest.approx(1.959963984540054, rel=1e-14)
    assert orc.normal_ppf(0.8413447460685429) == pytest.approx(1.0, rel=1e-13)
    assert orc.normal_ppf(0.001) == pytest.approx(-3.090232306167813, rel=1e-13)
    assert math.isnan(orc.normal_ppf(0.0)) and math.isnan(orc.normal_ppf(1.0))


@pytest.mark.parametrize("p", list(np.linspace(1e-6, 1 - 1e-6, 41)) + [0.9677083, 0.03, 0.5 + 1e-9])
def test_ppf_matches_scipy(orc, p):
    x = orc.normal_ppf(p)
    assert x == pytest.approx(norm.ppf(p), rel=1e-12, abs=1e-12)
    # and it inverts the CDF
    assert norm.cdf(x) == pytest.approx(p, rel=1e-13, abs=1e-16)


def test_ppf_symmetry(orc):
    for p in (0.01, 0.2, 0.37, 0.49):
        assert orc.normal_ppf(p) == pytest.approx(-orc.normal_ppf(1 - p), rel=1e-12)


def test_codebook_structure(orc):
    cb = orc.nf4_codebook()
    assert cb.dtype == np.float32 and cb.shape == (16,)
    assert np.all(np.diff(cb) > 0), "strictly increasing"
    assert cb[0] == -1.0 and cb[15] == 1.0, "normalised so the extremes are exactly +-1"
    zeros = np.flatnonzero(cb == 0.0)
    assert list(zeros) == [7], "exactly one exact zero, at index 7"
    assert (cb < 0).sum() == 7 and (cb > 0).sum() == 8, "asymmetric halves"
    assert np.all(np.abs(cb) <= 1.0)


def test_codebook_quantiles(orc):
    """Each level, scaled back by Phi^-1(delta), sits at its equal-spaced
    probability: 9 points from delta to 1/2 on the positive side, 8 on the
    negative side (the 1/2 point of each side is the shared zero)."""
    cb = orc.nf4_codebook().astype(np.float64)
    d = orc.NF4_DELTA
    z = norm.ppf(d)
    pos = [d + (0.5 - d) * i / 8 for i in range(8)]
    neg = [d + (0.5 - d) * i / 7 for i in range(7)]
    got_pos = sorted(norm.cdf(c * z) for c in cb[cb > 0])
    got_neg = sorted(norm.cdf(-c * z) for c in cb[cb < 0])
    # fp32 rounding of the levels limits agreement to ~1e-7 in probability
    np.testing.assert_allclose(got_pos, sorted(pos), atol=3e-7)
    np.testing.assert_allclose(got_neg, sorted(neg), atol=3e-7)


def test_codebook_independent_scipy_construction(orc):
    d = orc.NF4_DELTA
    z = norm.ppf(d)
    v = [norm.ppf(d + (0.5 - d) * i / 8) / z for i in range(8)]
    v += [-norm.ppf(d + (0.5 - d) * i / 7) / z for i in range(7)]
    v += [0.0]
    ref = np.sort(np.array(v, dtype=np.float64)).astype(np.float32)
    got = orc.nf4_codebook()
    ulps = np.abs(got.view(np.int32).astype(np.int64) - ref.view(np.int32).astype(np.int64))
    assert ulps.max() <= 1


def test_codebook_finer_near_zero(orc):
    """More levels near 0 than at the ends (bitsandbytes article section 6.1)."""
    cb = orc.nf4_codebook().astype(np.float64)
    gaps = np.diff(cb)
    assert gaps[6] < gaps[0] and gaps[7] < gaps[14]
    assert np.all(np.diff(gaps[7:]) > 0), "positive side spacing grows outward"
    assert np.all(np.diff(gaps[:7]) < 0), "negative side spacing grows outward"


def test_codebook_delta_variant(orc):
    """A different tail probability still yields a valid table; the library
    takes the table as an argument, so parity never depends on delta."""
    cb = orc.nf4_codebook(1 - 1 / 32)
    assert cb[0] == -1 and cb[15] == 1 and cb[7] == 0
    assert np.all(np.diff(cb) > 0)
    assert not np.array_equal(cb, orc.nf4_codebook())
