"""Pins for the oracle's NF4 codebook and thresholds (CPU only).

The pages fix the principle: 16 levels at standard-normal quantiles, equal
expected mass per bin, normalised to [-1, 1] ("QLoRA", llm-compass, 方法与公式
item 1; learn-interview-questions, section 2).  These tests check the oracle's
table against that principle with an inverse normal CDF written here
independently (bisection on math.erfc), not by re-calling the oracle's.
"""

import math
from fractions import Fraction

import numpy as np
import pytest

from oracle import nf4

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


def phi(x: float) -> float:
    return 0.5 * math.erfc(-x / math.sqrt(2.0))


def inv_phi_bisect(p: float) -> float:
    """Inverse standard normal CDF by bisection on erfc (independent of the
    oracle's statistics.NormalDist)."""
    lo, hi = -10.0, 10.0
    for _ in range(200):
        mid = 0.5 * (lo + hi)
        if phi(mid) < p:
            lo = mid
        else:
            hi = mid
    return 0.5 * (lo + hi)


def independent_levels_f32():
    delta = 1.0 - 0.5 * (1.0 / 32 + 1.0 / 30)
    norm = inv_phi_bisect(delta)
    pos = [inv_phi_bisect(delta - i * (delta - 0.5) / 8) / norm for i in range(8)]
    neg = [-inv_phi_bisect(delta - i * (delta - 0.5) / 7) / norm for i in range(7)]
    return np.array(sorted(pos + neg + [0.0]), dtype=np.float32)


def test_sixteen_levels_ascending_with_exact_zero_and_unit_extremes():
    q = nf4.codebook()
    assert q.shape == (16,)
    assert np.all(np.diff(q) > 0)
    assert q[7] == 0.0 and np.signbit(q[7]) == False  # noqa: E712
    assert q[0] == -1.0 and q[15] == 1.0
    assert np.all(np.abs(q) <= 1.0)
    # 8 positive levels, 7 negative levels (asymmetric split around the zero)
    assert (q > 0).sum() == 8 and (q < 0).sum() == 7


def test_levels_match_independent_inverse_cdf_bit_for_bit():
    ours = nf4.f32_bits(nf4.codebook())
    ref = independent_levels_f32().view(np.uint32)
    assert np.array_equal(ours, ref), (
        [hex(a) for a in ours], [hex(b) for b in ref])


def test_levels_are_not_near_an_fp32_rounding_tie():
    # Any accurate inverse CDF must give the same fp32 table: every fp64 level
    # lies well away from the midpoint between two fp32 neighbours.
    q64 = nf4.codebook_f64()
    for v in q64:
        f = np.float32(v)
        if float(f) == v:
            continue
        up = np.nextafter(f, np.float32(np.inf))
        dn = np.nextafter(f, np.float32(-np.inf))
        ulp = float(up) - float(f) if v > float(f) else float(f) - float(dn)
        assert abs(v - float(f)) < 0.49 * ulp


def test_equal_normal_mass_per_side():
    """Unnormalised levels (level * Phi^-1(delta)) cut N(0,1) into bins of
    equal mass on each side of zero; tails beyond the extremes hold 1-delta."""
    delta = 1.0 - 0.5 * (1.0 / 32 + 1.0 / 30)
    norm = inv_phi_bisect(delta)
    z = nf4.codebook() * norm
    masses = np.array([phi(z[i + 1]) - phi(z[i]) for i in range(15)])
    neg = masses[:7]     # bins between the 7 negative levels and zero
    pos = masses[7:]     # bins between zero and the 8 positive levels
    assert np.allclose(neg, (delta - 0.5) / 7, atol=1e-6)
    assert np.allclose(pos, (delta - 0.5) / 8, atol=1e-6)
    assert neg.max() - neg.min() < 1e-3 and pos.max() - pos.min() < 1e-3
    assert abs(neg.mean() / pos.mean() - 8.0 / 7.0) < 1e-5
    assert abs(phi(z[0]) - (1 - delta)) < 1e-6
    assert abs(1 - phi(z[15]) - (1 - delta)) < 1e-6
    # all masses (tails included) add to one
    assert abs(masses.sum() + 2 * (1 - delta) - 1.0) < 1e-9


def test_symmetric_sixteenths_are_not_attainable_with_exact_zero():
    """Documented consequence of the exact zero: the 16 nearest-level decision
    bins do not each hold 1/16 of N(0,1) (they range about 0.056..0.071)."""
    delta = 1.0 - 0.5 * (1.0 / 32 + 1.0 / 30)
    norm = inv_phi_bisect(delta)
    z = nf4.codebook() * norm
    cuts = [-np.inf] + list((z[:-1] + z[1:]) / 2) + [np.inf]
    bins = [phi(cuts[i + 1]) - phi(cuts[i]) for i in range(16)]
    assert abs(sum(bins) - 1.0) < 1e-12
    assert 0.05 < min(bins) < 0.06 and 0.07 < max(bins) < 0.075


def test_largest_gap_and_half_gap():
    q = nf4.codebook()
    gaps = np.diff(q)
    assert int(np.argmax(gaps)) == 0
    assert abs(gaps.max() - 0.303807) < 1e-6
    assert abs(gaps.max() / 2 - 0.151904) < 1e-6
    assert abs(gaps[7:].max() - 0.277043) < 1e-6


def test_thresholds_separate_exactly_at_midpoints():
    q = nf4.codebook()
    thr = nf4.thresholds()
    for j in range(15):
        mid = Fraction(float(q[j])) / 2 + Fraction(float(q[j + 1])) / 2
        t = np.float32(thr[j])
        assert float(t) == thr[j]
        assert Fraction(float(t)) <= mid
        # the next fp32 above the threshold is strictly above the midpoint
        nxt = np.nextafter(t, np.float32(np.inf))
        assert Fraction(float(nxt)) > mid or Fraction(float(t)) == mid
    # exactly four midpoints are fp32-representable
    exact = sum(float(np.float32(m)) == m for m in nf4.midpoints())
    assert exact == 4
