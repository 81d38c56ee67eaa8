"""Pins of the INT4 comparison oracle: the level set, brute-force nearest
level in exact arithmetic, the round-trip bound, and the pages' claim that
NF4 beats uniform INT4 on normally distributed weights."""

from fractions import Fraction

import numpy as np

from oracle import int4, nf4


def test_levels_uniform_symmetric_with_exact_zero():
    lv = int4.levels()
    assert lv.size == 16 and lv[7] == 0.0 and lv[0] == -1.0 and lv[14] == 1.0 and lv[15] == 1.0
    assert np.all(np.diff(lv[:15]) > 0)
    for k in range(15):                                     # fl32(k/7) for k = -7..7
        assert lv[k] == float(np.float32((k - 7) / 7.0))
    assert np.allclose(np.diff(lv[:15]), 1 / 7, atol=1e-7)


def test_nearest_level_brute_force_exact():
    """argmin |v - level| in exact rationals, ties to the lower index."""
    lv = [Fraction(float(x)) for x in int4.levels()]
    rng = np.random.default_rng(0)
    vs = np.concatenate([rng.uniform(-1.0, 1.0, 400).astype(np.float32),
                         np.float32(int4.midpoints()).astype(np.float32),
                         np.array([-1.0, 1.0, 0.0, np.nextafter(np.float32(1), np.float32(2))], dtype=np.float32)])
    got = int4.nearest_level(vs.astype(np.float64))
    for v, g in zip(vs, got):
        fv = Fraction(float(v))
        d = [abs(fv - x) for x in lv]
        best = min(range(16), key=lambda k: (d[k], k))
        assert lv[g] == lv[best], (v, g, best)               # code 15 and 14 share +1


def test_round_trip_bound_half_step():
    """|w - level[code] * c| <= c / 14 (half the uniform step) for every weight."""
    rng = np.random.default_rng(1)
    W = (rng.standard_normal((32, 256)) * 0.02).astype(np.float32)
    q = int4.quantize(W)
    c = q["absmax"]
    lv = int4.levels()
    approx = lv[q["codes"].reshape(-1, 64)] * c[:, None]
    err = np.abs(W.astype(np.float64).reshape(-1, 64) - approx)
    assert np.all(err <= c[:, None] / 14 * (1 + 1e-6))


def test_nf4_beats_int4_on_normal_weights():
    """The pages' comparison: on zero-mean normal weights NF4's round-trip
    error is lower than uniform INT4's at the same block size."""
    rng = np.random.default_rng(2)
    W = (rng.standard_normal((256, 1024)) * 0.02).astype(np.float32)
    qn, qi = nf4.quantize(W), int4.quantize(W)
    wn = nf4.dequantize(qn["codes"], qn["q8"], qn["step2"], qn["mean"])
    wi = nf4.bf16_to_f64(int4.dequantize_bits(qi["codes"], qi["q8"], qi["step2"], qi["mean"]))
    e_nf4 = np.linalg.norm(wn - W) / np.linalg.norm(W)
    e_int4 = np.linalg.norm(wi - W) / np.linalg.norm(W)
    assert e_nf4 < 0.9 * e_int4, (e_nf4, e_int4)
