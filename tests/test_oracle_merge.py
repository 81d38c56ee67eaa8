"""Pins of the adapter-merge and 16-bit-input oracles against facts that do
not come from the oracle itself: torch's bf16 widening, exact arithmetic,
error bounds and the linear-layer identity."""

import numpy as np
import torch

from oracle import linear, merge, nf4


def _bf16_bits(t: torch.Tensor) -> np.ndarray:
    return t.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def test_bf16_widening_matches_torch():
    rng = np.random.default_rng(0)
    bits = rng.integers(0, 1 << 16, 4096, dtype=np.uint32).astype(np.uint16)
    bits = bits[(bits & 0x7F80) != 0x7F80]                    # finite values only
    ours = nf4.bf16_to_f64(bits)
    ref = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).float().double().numpy()
    assert np.array_equal(ours, ref)


def test_bf16_quantizer_input_levels_round_trip():
    """A block holding bf16(c * level[j]) for every j (c a power of two, so
    the products are exact) encodes to j: the bf16 rounding of a level moves
    it by at most 2^-9 relative, far less than half of any level gap."""
    lv = nf4.codebook()
    vals = np.tile(np.repeat(lv, 4), 1)                       # 64 values, codes 0..15 four times
    W = (0.25 * vals).astype(np.float32).reshape(1, 64)
    bits = _bf16_bits(torch.from_numpy(W))
    q = nf4.quantize_bf16(bits)
    assert np.array_equal(q["codes"].ravel(), np.repeat(np.arange(16), 4))


def _rand_bf16(rng, shape, scale):
    return _bf16_bits(torch.from_numpy((rng.standard_normal(shape) * scale).astype(np.float32)))


def test_merge_with_zero_B_is_the_base():
    rng = np.random.default_rng(1)
    w = _rand_bf16(rng, (32, 128), 0.02)
    A = _rand_bf16(rng, (8, 128), 0.1)
    B = np.zeros((32, 8), dtype=np.uint16)
    assert np.array_equal(merge.merge_adapter_bits(w, A, B, 16.0), w)


def test_merge_rank_one_exact_sum():
    """r = 1, alpha = r: one exact product, s = 1; the merged value is the
    correctly rounded (fp32, then bf16) exact sum w + b * a."""
    rng = np.random.default_rng(2)
    w = _rand_bf16(rng, (16, 64), 0.02)
    A = _rand_bf16(rng, (1, 64), 0.5)
    B = _rand_bf16(rng, (16, 1), 0.05)
    got = merge.merge_adapter_bits(w, A, B, 1.0)
    exact = nf4.bf16_to_f64(w) + np.outer(nf4.bf16_to_f64(B)[:, 0], nf4.bf16_to_f64(A)[0])
    want = nf4.bf16_bits_from_f32(exact.astype(np.float32).astype(np.float64))
    assert np.array_equal(got, want)


def test_merge_error_bound_and_orientation():
    """|W' - (W0 + s B A)| <= half a bf16 ulp of W' + the fp32 accumulation
    bound; a transposed or mis-scaled product fails it."""
    rng = np.random.default_rng(3)
    out_f, in_f, r, alpha = 48, 192, 16, 32.0
    w = _rand_bf16(rng, (out_f, in_f), 0.02)
    A = _rand_bf16(rng, (r, in_f), 1 / np.sqrt(in_f))
    B = _rand_bf16(rng, (out_f, r), 0.01)
    s = alpha / r
    got = nf4.bf16_to_f64(merge.merge_adapter_bits(w, A, B, alpha))
    Af, Bf = nf4.bf16_to_f64(A), nf4.bf16_to_f64(B)
    exact = nf4.bf16_to_f64(w) + s * (Bf @ Af)
    half_ulp = np.abs(got) * 2.0 ** -8
    acc_bound = s * r * 2.0 ** -23 * (np.abs(Bf) @ np.abs(Af)) + np.abs(exact) * 2.0 ** -23
    assert np.all(np.abs(got - exact) <= half_ulp + acc_bound + 1e-30)
    wrong = nf4.bf16_to_f64(w) + s * (Bf @ Af)[:, ::-1]           # permuted columns
    assert not np.all(np.abs(got - wrong) <= half_ulp + acc_bound + 1e-30)


def test_merged_weight_reproduces_the_layer():
    """x W'^T equals the layer forward x W0^T + s (x A^T) B^T up to the bf16
    rounding of W' (llm-compass formula, merged form)."""
    rng = np.random.default_rng(4)
    M, out_f, in_f, r, alpha = 8, 64, 128, 8, 16.0
    w = _rand_bf16(rng, (out_f, in_f), 0.02)
    A = _rand_bf16(rng, (r, in_f), 1 / np.sqrt(in_f))
    B = _rand_bf16(rng, (out_f, r), 0.01)
    x = nf4.bf16_to_f64(_rand_bf16(rng, (M, in_f), 1.0))
    Wm = nf4.bf16_to_f64(merge.merge_adapter_bits(w, A, B, alpha))
    h_ref, _ = linear.linear_fwd(x, nf4.bf16_to_f64(w), nf4.bf16_to_f64(A), nf4.bf16_to_f64(B), alpha)
    h = x @ Wm.T
    assert np.linalg.norm(h - h_ref) <= 2.0 ** -8 * np.linalg.norm(np.abs(x) @ np.abs(Wm).T)


def _bf16_exact_bits(x: float) -> int:
    """bf16 bit pattern of a value that bf16 represents exactly."""
    b = int(np.float32(x).view(np.uint32))
    assert b & 0xFFFF == 0
    return b >> 16


def test_merge_accumulates_in_fp32_in_rank_order():
    """Reading M1: acc is the in-order fp32 sum of the exact products.  Here
    the first product is 1 + 2^-3 + 2^-8 (a bf16 tie) and the next two,
    0.75 * 2^-24 each, are dropped one by one in fp32, so W' rounds the tie
    to even (0x3F90); the exact sum (1.5 * 2^-24 more) would round up."""
    B = np.array([[_bf16_exact_bits(1 + 2 ** -4), _bf16_exact_bits(1.5 * 2 ** -12), _bf16_exact_bits(1.5 * 2 ** -12)]], dtype=np.uint16)
    A = np.array([[_bf16_exact_bits(1 + 2 ** -4)], [_bf16_exact_bits(2 ** -13)], [_bf16_exact_bits(2 ** -13)]], dtype=np.uint16)
    acc = merge.lora_product_f32(A, B)
    assert acc[0, 0] == 1 + 2 ** -3 + 2 ** -8
    w_hat = np.array([[0]], dtype=np.uint16)
    assert merge.merge_adapter_bits(w_hat, A, B, 3.0)[0, 0] == 0x3F90         # s = fl32(3 / 3) = 1
    assert nf4.bf16_bits_from_f32(1 + 2 ** -3 + 2 ** -8 + 1.5 * 2 ** -24) == 0x3F91   # the exact sum's bf16


def test_merge_rounds_the_scaled_product_before_adding_the_base():
    """Reading M1: W' = bf16(fl32(w_hat + fl32(s * acc))).  With r = 1,
    s = 16647415 * 2^-24, acc = 2^-8 (1 + 2^-7): s * acc = 2^-8 + 2^-24 +
    119 * 2^-39 rounds to 2^-8 + 2^-24 in fp32, so 1 + that is an fp32 tie
    (to 1 + 2^-8, then a bf16 tie to 1.0); without the inner rounding the sum
    lies above both ties and W' would be 1 + 2^-7."""
    alpha = 16647415 * 2.0 ** -24
    B = np.array([[_bf16_exact_bits(2 ** -4 * (1 + 2 ** -7))]], dtype=np.uint16)
    A = np.array([[_bf16_exact_bits(2 ** -4)]], dtype=np.uint16)
    w_hat = np.array([[_bf16_exact_bits(1.0)]], dtype=np.uint16)
    assert merge.merge_adapter_bits(w_hat, A, B, alpha)[0, 0] == 0x3F80
    exact = 1 + (16647415 * 2.0 ** -24) * (2 ** -8 * (1 + 2 ** -7))          # exact in fp64 (41 bits)
    assert nf4.bf16_bits_from_f32(nf4.fl32(exact)) == 0x3F81                   # one rounding only


def test_merge_rounds_the_scale_alpha_over_r_to_fp32():
    """Reading M1: s = fl32(alpha / r).  With alpha = 11107844 * 2^-22 and
    r = 3, alpha / 3 = 14810458.67 * 2^-24 rounds up to s = 14810459 * 2^-24.
    One rank carries acc = 2^-4 * 145 * 2^-11 (the other two are zero), and
    s * acc = 8388736.54 * 2^-31 rounds to 2^-8 + 2^-24 + 2^-31: above the
    fp32 tie of 1 + 2^-8 + 2^-24, so W' = bf16(1 + 2^-8 + 2^-23) = 1 + 2^-7.
    With the quotient left unrounded the product, 8388736.36 * 2^-31, rounds to
    2^-8 + 2^-24, both ties round to even and W' would be 1.0."""
    alpha = 11107844 * 2.0 ** -22
    assert float(np.float32(alpha)) == alpha
    s = np.float32(alpha) / np.float32(3)                                      # IEEE fp32 division
    assert float(s) == 14810459 * 2.0 ** -24
    B = np.array([[_bf16_exact_bits(2 ** -4), 0, 0]], dtype=np.uint16)
    A = np.array([[_bf16_exact_bits(145 * 2.0 ** -11)], [0], [0]], dtype=np.uint16)
    w_hat = np.array([[_bf16_exact_bits(1.0)]], dtype=np.uint16)
    prod = np.float32(float(s) * (145 * 2.0 ** -15))                            # the fp64 product is exact
    assert float(prod) == 2 ** -8 + 2 ** -24 + 2 ** -31
    assert int((np.float32(1) + prod).view(np.uint32)) == 0x3F808001           # 1 + 2^-8 + 2^-23
    assert merge.merge_adapter_bits(w_hat, A, B, alpha)[0, 0] == 0x3F81
    unrounded = np.float32((alpha / 3) * (145 * 2.0 ** -15))
    assert float(unrounded) == 2 ** -8 + 2 ** -24
    assert int((np.float32(1) + unrounded).view(np.uint32)) == 0x3F808000      # tie to even: 1 + 2^-8
