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
