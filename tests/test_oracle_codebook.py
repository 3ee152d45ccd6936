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

from conftest import floats, read_golden


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


# ---------------------------------------------------------------- FP4 table
# bitsandbytes' other 4-bit type is a "4-bit float-style" table (bitsandbytes
# article (CSDN) 6.4-6.5, 9.3).  Reading: FP4 E2M1 of the OCP Microscaling
# formats, scaled by 1/6 into [-1, 1]; the magnitudes are the golden list.

def test_fp4_codebook_is_e2m1_over_6(orc):
    g = read_golden("fp4_e2m1_values.txt")
    mags = floats(g["magnitudes"])
    top = float(g["max_magnitude"])
    cb = orc.fp4_codebook()
    assert cb.dtype == np.float32 and cb.shape == (16,)
    want_pos = np.array([m / top for m in mags], dtype=np.float32)
    assert np.array_equal(cb[8:], want_pos)
    assert np.array_equal(cb[:8], -want_pos[::-1])
    assert cb[0] == -1 and cb[15] == 1


def test_fp4_codebook_structure(orc):
    """Non-decreasing; the one repeated level is the zero, -0 (index 7) before
    +0 (index 8); antisymmetric; each magnitude times 6 has one significant
    bit after the leading one at most (a 1-bit mantissa)."""
    cb = orc.fp4_codebook()
    assert np.all(np.diff(cb.astype(np.float64)) >= 0)
    eq = np.flatnonzero(np.diff(cb.astype(np.float64)) == 0)
    assert list(eq) == [7]
    assert cb[7] == 0 and np.signbit(cb[7]) and cb[8] == 0 and not np.signbit(cb[8])
    assert np.array_equal(cb[::-1], -cb)
    for m in np.abs(cb.astype(np.float64)) * 6:
        m = float(np.float32(m))
        if m:
            mant, _ = math.frexp(m)
            assert (mant * 4) == int(mant * 4)


def test_fp4_quantize_first_minimum(orc):
    """Quantizing with the FP4 table: every weight takes the first nearest
    level in exact arithmetic; in zero's basin that is -0 (index 7) for
    weights of either sign, and the +0 code is never produced."""
    from fractions import Fraction as Fr
    cb = orc.fp4_codebook()
    rng = np.random.default_rng(4)
    W = (rng.standard_normal((6, 64)) * 0.02).astype(np.float32)
    W[0, 1:9] = np.array([1e-9, -1e-9, 0.0, -0.0, 1e-3, -1e-3, 2e-4, -2e-4], np.float32)
    q = orc.quantize(W, cb, False)
    flat = W.reshape(-1)
    idx = np.empty(flat.size, np.int64)
    idx[0::2], idx[1::2] = q.packed >> 4, q.packed & 15
    for b in range(flat.size // 64):
        blk = flat[64 * b:64 * b + 64]
        a = Fr(float(np.max(np.abs(blk))))
        for i, w in enumerate(blk):
            d = [abs(Fr(float(w)) - Fr(float(c)) * a) for c in cb]
            assert idx[64 * b + i] == d.index(min(d))
    assert not np.any(idx == 8)
    deq = orc.dequantize(q, cb).reshape(-1)
    assert deq[2] == 0x8000 and deq[3] == 0x8000          # +-1e-9 -> -0 in bf16
