"""Pins for the oracle's blockwise quantizer, double quantization and
dequantization (CPU only): brute force in exact rational arithmetic, exact
round trips, error bounds, zero handling and the storage arithmetic the pages
print."""

import os
import struct
from fractions import Fraction

import numpy as np
import pytest

from oracle import nf4, overhead

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")
GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def brute_nearest(v: float, levels) -> int:
    """argmin_j |v - q_j| in exact rational arithmetic, ties to the lower j."""
    fv = Fraction(float(v))
    best, best_d = 0, None
    for j, q in enumerate(levels):
        d = abs(fv - Fraction(float(q)))
        if best_d is None or d < best_d:
            best, best_d = j, d
    return best


def test_nearest_level_matches_brute_force_on_all_fp16_values():
    levels = nf4.codebook()
    h = np.arange(0, 1 << 16, dtype=np.uint16).view(np.float16).astype(np.float64)
    h = h[np.isfinite(h) & (np.abs(h) <= 1.1)]
    got = nf4.nearest_level(h)
    # brute force on a deterministic subsample plus every value within 1e-3
    # of a midpoint (where a wrong tie rule or threshold would show)
    mids = nf4.midpoints()
    near = np.min(np.abs(h[:, None] - mids[None, :]), axis=1) < 1e-3
    idx = np.unique(np.concatenate([np.nonzero(near)[0], np.arange(0, h.size, 37)]))
    for i in idx:
        assert got[i] == brute_nearest(h[i], levels), h[i]


def test_nearest_level_ties_go_to_lower_index():
    levels = nf4.codebook()
    for j, m in enumerate(nf4.midpoints()):
        if float(np.float32(m)) == m:            # representable midpoint: a true tie
            assert nf4.nearest_level(np.array([m]))[0] == j
            assert brute_nearest(m, levels) == j


def test_encode_matches_brute_force_on_tiny_blocks():
    rng = np.random.default_rng(5)
    W = (rng.standard_normal((2, 128)) * 0.02).astype(np.float32)
    W[1, 64:] = (rng.standard_t(3, 64) * 0.05).astype(np.float32)
    c = nf4.block_absmax(W)
    codes = nf4.encode(W, c)
    levels = nf4.codebook()
    for b in range(4):
        row, col0 = divmod(b * 64, 128)
        cb = np.float32(np.abs(W[row, col0:col0 + 64]).max())
        assert float(cb) == c[b]
        r = np.float32(1.0) / cb                      # fp32 reciprocal
        for k in range(64):
            v = np.float32(W[row, col0 + k]) * r      # fp32 product
            assert codes[row, col0 + k] == brute_nearest(float(v), levels)


def test_exact_levels_round_trip():
    levels = nf4.codebook()
    for c in [1.0, 0.0371, 3.5e-3, 17.25]:
        w = np.float32(c) * levels.astype(np.float32)     # includes +-c (levels 0, 15)
        W = np.tile(w, 4).reshape(1, 64)
        q = nf4.quantize(W)
        assert q["absmax"][0] == np.float32(c)
        assert np.array_equal(q["codes"][0], np.tile(np.arange(16), 4))


def test_first_level_round_trip_bound():
    """|w - q[code] * c| <= c * G/2 with G the largest codebook gap."""
    rng = np.random.default_rng(11)
    W = np.concatenate([rng.standard_normal((64, 256)) * 0.02,
                        rng.standard_t(5, (64, 256)) * 0.02]).astype(np.float32)
    q = nf4.quantize(W)
    levels = nf4.codebook()
    c = q["absmax"].repeat(64).reshape(W.shape)
    recon = levels[q["codes"]] * c
    G2 = np.diff(levels).max() / 2
    err = np.abs(W.astype(np.float64) - recon)
    # reciprocal normalisation moves v by at most a couple of fp32 ulps
    assert np.all(err <= c * (G2 + 1e-6))
    # and the bound is attained closely somewhere (it is not vacuous)
    assert (err / c).max() > 0.9 * G2


def test_dequantized_round_trip_bound_with_double_quant():
    rng = np.random.default_rng(12)
    W = (rng.standard_normal((128, 512)) * 0.02).astype(np.float32)
    q = nf4.quantize(W)
    c = q["absmax"]
    c_hat = nf4.dequant_scales(q["q8"], q["step2"], q["mean"])
    g = np.arange(c.size) // 256
    # second-level error: half a step plus fp32 rounding
    assert np.all(np.abs(c - c_hat) <= q["step2"][g] * 0.5 + 4 * np.spacing(np.float32(c.max())))
    w_hat = nf4.dequantize(q["codes"], q["q8"], q["step2"], q["mean"])
    G2 = np.diff(nf4.codebook()).max() / 2
    cb = c.repeat(64).reshape(W.shape)
    dc = np.abs(c - c_hat).repeat(64).reshape(W.shape)
    bound = cb * (G2 + 1e-6) + dc + np.abs(w_hat) * 2.0 ** -8 + 1e-30
    assert np.all(np.abs(W - w_hat) <= bound)


def test_zero_blocks_and_negative_zero():
    W = np.zeros((2, 128), dtype=np.float32)
    W[0, 64:] = np.linspace(-0.03, 0.05, 64, dtype=np.float32)
    W[1, :64] = np.float32(-0.0)
    q = nf4.quantize(W)
    assert np.all(q["codes"][0, :64] == 7)
    assert np.all(q["codes"][1] == 7)
    w_hat = nf4.dequantize(q["codes"], q["q8"], q["step2"], q["mean"])
    assert np.all(w_hat[0, :64] == 0.0) and np.all(w_hat[1] == 0.0)
    # -0.0 inside a nonzero block also maps to the zero level
    W2 = np.linspace(-1, 1, 64, dtype=np.float32).reshape(1, 64)
    W2[0, 10] = np.float32(-0.0)
    assert nf4.quantize(W2)["codes"][0, 10] == 7


def test_equal_absmax_blocks_give_zero_second_level_codes():
    # every block has absmax exactly 0.5 -> c - mean = 0 -> step 0 -> q8 = 0,
    # and the dequantized scale is exactly the mean
    rng = np.random.default_rng(3)
    W = (rng.uniform(-0.5, 0.5, (8, 256))).astype(np.float32)
    W[:, ::64] = 0.5
    q = nf4.quantize(W)
    assert q["mean"] == 0.5
    assert np.all(q["q8"] == 0) and np.all(q["step2"] == 0)
    assert np.all(nf4.dequant_scales(q["q8"], q["step2"], q["mean"]) == 0.5)


def test_second_level_codes_use_full_int8_range():
    rng = np.random.default_rng(4)
    W = (rng.standard_normal((64, 1024)) * 0.02).astype(np.float32)   # 1024 blocks = 4 groups
    q = nf4.quantize(W)
    assert q["q8"].min() >= -127 and q["q8"].max() <= 127
    for g in range(4):
        assert np.abs(q["q8"][g * 256:(g + 1) * 256]).max() == 127
    assert q["step2"].shape == (4,)


def test_partial_last_group():
    """305 blocks with absmax 1, 2, ..., 305 (a partial second group of 49),
    worked by hand: mean = 46665 / 305 = 153, d_b = b + 1 - 153 ranges over
    -152..103 in group 0 and 104..152 in group 1, so both steps are
    fl32(152/127); q8 is +-127 at the ends, 0 at d = 0, and within half a
    step (plus the fp32 roundings) of d * 127 / 152 everywhere."""
    c = np.arange(1, 306, dtype=np.float64)
    W = np.zeros((5, 64 * 61), dtype=np.float32)
    W.reshape(-1, 64)[:, 17] = c                    # one weight per block sets its absmax
    q = nf4.quantize(W)
    assert np.array_equal(q["absmax"], c)
    assert q["mean"] == 153.0
    assert q["step2"].shape == (2,) and q["q8"].shape == (305,)
    assert np.all(q["step2"] == float(np.float32(152.0 / 127.0)))
    assert q["q8"][0] == -127 and q["q8"][304] == 127 and q["q8"][152] == 0
    exact = (c - 153.0) * 127.0 / 152.0
    assert np.all(np.abs(q["q8"] - exact) <= 0.5 + 1e-4)


def _mean_fixtures():
    with open(os.path.join(GOLDEN, "scale_mean.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            bits, spec = (t.strip() for t in line.split(";"))
            tok = spec.split()
            if tok[0] == "range":
                vals = np.arange(int(tok[1]), int(tok[2]) + 1, dtype=np.float64)
            elif tok[0] == "rep":
                vals = np.full(int(tok[1]), float(tok[2]))
            else:
                vals = np.array([float(t) for t in tok])
            yield int(bits, 16), vals


def _mean_mismatches(mean_fn):
    return [(hex(b), v.size) for b, v in _mean_fixtures()
            if int(np.array([mean_fn(v)], dtype=np.float32).view(np.uint32)[0]) != b]


def test_scale_mean_fixtures():
    """Hand-worked means of block counts that are not powers of two."""
    assert _mean_mismatches(nf4.scale_mean) == []


def test_scale_mean_fixtures_through_quantize():
    for bits, vals in _mean_fixtures():
        W = np.zeros((1, 64 * vals.size), dtype=np.float32)
        W.reshape(-1, 64)[:, 5] = vals
        q = nf4.quantize(W)
        assert int(np.array([q["mean"]], dtype=np.float32).view(np.uint32)[0]) == bits


def test_scale_mean_fixtures_reject_wrong_divisors():
    """The fixtures catch a mean divided by the zero-padded tree length, by
    the number of 256-block groups, or rounded to fp32 before the division."""
    def padded(c):
        n = 1
        while n < len(c):
            n *= 2
        return float(nf4.fl32(nf4.pairwise_sum(c) / n))

    def per_group(c):
        return float(nf4.fl32(nf4.pairwise_sum(c) / ((len(c) + 255) // 256)))

    def fp32_sum(c):
        return float(nf4.fl32(float(nf4.fl32(nf4.pairwise_sum(c))) / len(c)))

    assert len(_mean_mismatches(padded)) == 5
    assert len(_mean_mismatches(per_group)) == 5
    assert len(_mean_mismatches(fp32_sum)) == 0      # all fixture sums are exact in fp32
    assert len(_mean_mismatches(lambda c: float(np.mean(c)))) == 0


def test_pairwise_tree_fixtures():
    with open(os.path.join(GOLDEN, "pairwise_tree.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            want, vals = line.split(";")
            vals = [float(v) for v in vals.split()]
            assert nf4.pairwise_sum(np.array(vals)) == float(want), line


def test_pairwise_sum_accuracy_bound():
    rng = np.random.default_rng(7)
    v = rng.uniform(0, 0.1, 100003)
    import math
    exact = math.fsum(v)
    # pairwise summation error <= ceil(log2 n) * eps * sum|v|
    assert abs(nf4.pairwise_sum(v) - exact) <= 17 * 2.0 ** -53 * exact


def test_pack_unpack_nibble_order():
    codes = np.arange(32, dtype=np.uint8).reshape(1, 32) % 16
    p = nf4.pack(codes)
    assert p[0, 0] == (0 | (1 << 4)) and p[0, 1] == (2 | (3 << 4))
    assert np.array_equal(nf4.unpack(p), codes)


def test_bf16_rounding_matches_torch():
    import torch
    rng = np.random.default_rng(8)
    x = np.concatenate([rng.standard_normal(20000).astype(np.float32),
                        np.array([1.00390625, 1.01171875, -1.00390625, 0.0, -0.0,
                                  3.0e-39, 1e-45], dtype=np.float32)])
    ours = nf4.bf16_bits_from_f32(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)


def _golden_figures():
    out = {}
    with open(os.path.join(GOLDEN, "pages_figures.txt")) as f:
        for line in f:
            if line.strip() and not line.startswith("#"):
                name, val, tol = line.split()[:3]
                out[name] = (float(val), float(tol))
    return out


def test_overhead_arithmetic_matches_pages():
    fig = _golden_figures()

    def near(name, x):
        v, tol = fig[name]
        assert abs(x - v) <= tol, (name, x, v)

    fp32 = overhead.scale_bits_per_param(64, 32)
    dq = overhead.dq_bits_per_param(64, 256)
    assert fp32 == 0.5
    assert abs(dq - (8 / 64 + 32 / (64 * 256))) < 1e-15
    near("fp32_const_bits_per_param", fp32)
    near("dq_const_bits_per_param", dq)
    near("dq_saving_bits_per_param", fp32 - dq)
    near("dq_saving_bits_rounded", fp32 - dq)
    near("nf4_base_bytes_per_param", overhead.bits_per_param() / 8)
    near("base_7b_gigabytes", 7e9 * 4 / 8 / 1e9)


def test_stored_bytes_match_oracle_arrays():
    rng = np.random.default_rng(9)
    W = (rng.standard_normal((64, 64 * 40)) * 0.02).astype(np.float32)   # 2560 blocks
    q = nf4.quantize(W)
    nbytes = q["packed"].nbytes + q["q8"].nbytes + 4 * q["step2"].size + 4
    assert nbytes == overhead.stored_bytes(*W.shape)
    bits = 8.0 * nbytes / W.size
    assert abs(bits - overhead.bits_per_param(n_params=W.size)) < 1e-12


def test_quantize_rows_equals_full_quantize_rows():
    rng = np.random.default_rng(10)
    W = (rng.standard_normal((40, 640)) * 0.02).astype(np.float32)   # 400 blocks, 2 groups
    full = nf4.quantize(W)
    rows = np.array([0, 7, 39])
    sub = nf4.quantize_rows(W, rows)
    assert np.array_equal(sub["codes"], full["codes"][rows])
    assert np.array_equal(sub["q8"], full["q8"]) and sub["mean"] == full["mean"]
    d_full = nf4.dequantize(full["codes"], full["q8"], full["step2"], full["mean"])
    d_sub = nf4.dequantize(sub["codes"], sub["q8"], sub["step2"], sub["mean"], blocks=sub["blocks"])
    assert np.array_equal(d_sub, d_full[rows])


def test_reciprocal_overflow_block():
    """Absmax below ~2.9e-39: fl32(1/c) overflows, so every weight of the
    block is normalised by one correctly rounded division and gets its
    nearest level (brute force in exact rationals); zero weights stay at the
    zero level."""
    tiny = np.float32(2.0 ** -149)                  # smallest subnormal
    W = np.zeros((1, 64), dtype=np.float32)
    W[0, :8] = [2e-39, -2e-39, 0.0, -0.0, 1e-39, 3 * tiny, -5 * tiny, 1.3e-39]
    W[0, 8] = np.float32(1.9e-39)
    q = nf4.quantize(W)
    c = np.float32(2e-39)
    assert q["absmax"][0] == c
    assert not np.isfinite(np.float32(1.0) / c)     # the reciprocal really overflows
    levels = nf4.codebook()
    for k in range(64):
        quotient = Fraction(float(W[0, k])) / Fraction(float(c))
        v = float(np.float32(float(quotient)))      # the correctly rounded fp32 quotient
        assert q["codes"][0, k] == brute_nearest(v, levels), k
    assert list(q["codes"][0, :5]) == [15, 0, 7, 7, 12]   # 1e-39 / 2e-39 = 0.5 -> level 12


def test_second_level_reciprocal_overflow():
    """A group whose step's fp32 reciprocal overflows (max |c - mean| below
    ~3.7e-37) is coded by division: q8 = rint(fl32(d / step2)), checked in
    exact rationals, instead of saturating every nonzero d to +-127."""
    mu = float(np.float32(3e-38))
    scales = nf4.fl32(mu + np.array([1e-38, -1e-38, 5e-39, 2.5e-39, 0.0]))
    q8, step2 = nf4.second_level(scales, mu)
    d = nf4.fl32(scales - mu)
    st = float(np.float32(np.abs(d).max() / 127.0))
    assert step2[0] == st and not np.isfinite(np.float32(1.0) / np.float32(st))
    want = np.clip(np.rint([float(np.float32(float(Fraction(x) / Fraction(st)))) for x in d]), -127, 127)
    assert np.array_equal(q8, want.astype(np.int8))
    assert q8[0] == 127 and q8[1] == -127 and 0 < abs(int(q8[2])) < 127 and q8[4] == 0


# ---------------------------------------------------------------- rounding order of readings R3 and R6
# Independent IEEE binary32 rounding (round to nearest, ties to even; normal
# range) on exact rationals, to pin which operations the readings round.
def _round32(q: Fraction) -> Fraction:
    if q == 0:
        return Fraction(0)
    sign, a = (-1 if q < 0 else 1), abs(q)
    e = a.numerator.bit_length() - a.denominator.bit_length()
    while Fraction(2) ** e > a:
        e -= 1
    while Fraction(2) ** (e + 1) <= a:
        e += 1
    ulp = Fraction(2) ** (e - 23)
    m = a / ulp
    n = m.numerator // m.denominator
    rem = m - n
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and n % 2 == 1):
        n += 1
    return sign * n * ulp


def _from_bits(h: int) -> Fraction:
    return Fraction(struct.unpack("<f", struct.pack("<I", h))[0])


def _bits(q: Fraction) -> int:
    return struct.unpack("<I", struct.pack("<f", float(q)))[0]


@pytest.mark.parametrize("w_hex,c_hex,code_recip,code_div", [
    (0xBEE8D8AC, 0x3FF81F9C, 5, 4), (0xBEFF6C6F, 0x3FBBFD1D, 3, 4), (0xBDB60F98, 0x3FF9F248, 7, 6)])
def test_normalisation_multiplies_by_the_fp32_reciprocal(w_hex, c_hex, code_recip, code_div):
    """Reading R3: v = fl32(w * fl32(1/c)), not fl32(w / c).  Blocks where the
    two normalisations fall on different sides of a decision midpoint."""
    w, c = _from_bits(w_hex), _from_bits(c_hex)
    levels = [Fraction(float(v)) for v in nf4.codebook()]
    mids = [(levels[i] + levels[i + 1]) / 2 for i in range(15)]
    v_recip = _round32(w * _round32(1 / c))
    v_div = _round32(w / c)
    assert sum(m < v_recip for m in mids) == code_recip
    assert sum(m < v_div for m in mids) == code_div
    W = np.zeros((1, 64), dtype=np.float32)
    W[0, 0], W[0, 1] = float(c), float(w)               # c is the block's absmax
    assert nf4.quantize(W)["codes"][0, 1] == code_recip


def test_block_scale_rounds_the_product_then_the_sum():
    """Reading R6: c_hat = fl32(fl32(q8 * step2) + mean), two roundings; a
    case where one rounding of the exact sum gives the neighbouring float."""
    q, st, mu = -67, _from_bits(0x3C4DA4F9), _from_bits(0x3E1A6916)
    twice = _round32(_round32(q * st) + mu)
    once = _round32(q * st + mu)
    assert _bits(twice) == 0xBF30AE70 and _bits(once) == 0xBF30AE6F
    got = nf4.dequant_scales(np.array([q], dtype=np.int8), np.array([float(st)]), float(mu))
    assert _bits(Fraction(float(got[0]))) == 0xBF30AE70
