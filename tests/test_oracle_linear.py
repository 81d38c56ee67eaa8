"""Pins for the oracle's QLoRA linear forward/backward (CPU only).

The loss L = sum(dh * h) is linear in x, in A and in B separately, so central
differences with any step are exact up to fp64 rounding: they pin the
analytic dx, dA, dB (catching dropped terms, wrong scale, transposed
operands).  Brute-force triple loops pin the forward independently of
NumPy's matmul, and the merged-weight identity pins the LoRA term's operand
order.
"""

import itertools

import numpy as np
import pytest

from oracle import linear, nf4


def _problem(M=3, n_in=7, n_out=5, r=2, seed=0):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((M, n_in))
    W = rng.standard_normal((n_out, n_in)) * 0.1
    A = rng.uniform(-0.5, 0.5, (r, n_in))
    B = rng.standard_normal((n_out, r)) * 0.1
    dh = rng.standard_normal((M, n_out))
    return x, W, A, B, dh


def _loss(x, W, A, B, dh, alpha):
    h, _ = linear.linear_fwd(x, W, A, B, alpha)
    return float((dh * h).sum())


def _fd(fun, P, eps=0.5):
    G = np.zeros_like(P)
    for idx in itertools.product(*[range(n) for n in P.shape]):
        Pp = P.copy(); Pp[idx] += eps
        Pm = P.copy(); Pm[idx] -= eps
        G[idx] = (fun(Pp) - fun(Pm)) / (2 * eps)
    return G


@pytest.mark.parametrize("alpha", [4.0, 0.5])
def test_backward_matches_central_differences(alpha):
    x, W, A, B, dh = _problem()
    dx, dA, dB = linear.linear_bwd(dh, x, W, A, B, alpha)
    gx = _fd(lambda P: _loss(P, W, A, B, dh, alpha), x)
    gA = _fd(lambda P: _loss(x, W, P, B, dh, alpha), A)
    gB = _fd(lambda P: _loss(x, W, A, P, dh, alpha), B)
    for g, a in [(gx, dx), (gA, dA), (gB, dB)]:
        assert g.shape == a.shape
        assert np.allclose(g, a, rtol=1e-9, atol=1e-11)


def test_forward_matches_brute_force_loops():
    x, W, A, B, _ = _problem(M=2, n_in=4, n_out=3, r=2, seed=1)
    alpha = 3.0
    s = alpha / 2
    h, u = linear.linear_fwd(x, W, A, B, alpha)
    for m in range(2):
        for o in range(3):
            base = sum(x[m, k] * W[o, k] for k in range(4))
            lora = sum(B[o, j] * sum(A[j, k] * x[m, k] for k in range(4)) for j in range(2))
            assert abs(h[m, o] - (base + s * lora)) < 1e-12
        for j in range(2):
            assert abs(u[m, j] - sum(A[j, k] * x[m, k] for k in range(4))) < 1e-12


def test_merged_weight_identity():
    """h = x (W + s B A)^T and dx = dh (W + s B A): the adapter merge."""
    x, W, A, B, dh = _problem(M=4, n_in=9, n_out=6, r=3, seed=2)
    alpha = 6.0
    Wm = W + (alpha / 3) * (B @ A)
    h, _ = linear.linear_fwd(x, W, A, B, alpha)
    dx, _, _ = linear.linear_bwd(dh, x, W, A, B, alpha)
    assert np.allclose(h, x @ Wm.T, rtol=1e-12, atol=1e-12)
    assert np.allclose(dx, dh @ Wm, rtol=1e-12, atol=1e-12)


def test_zero_adapter_reduces_to_plain_matmul():
    x, W, A, B, dh = _problem(M=3, n_in=6, n_out=4, r=2, seed=3)
    for (AA, BB, alpha) in [(A, np.zeros_like(B), 2.0), (A, B, 0.0)]:
        h, _ = linear.linear_fwd(x, W, AA, BB, alpha)
        ref = np.array([[sum(x[m, k] * W[o, k] for k in range(6)) for o in range(4)]
                        for m in range(3)])
        assert np.allclose(h, ref, rtol=1e-12, atol=1e-12)
    _, dA, dB = linear.linear_bwd(dh, x, W, np.zeros_like(A), B, 2.0)
    assert np.all(dB == 0.0)
    _, dA, _ = linear.linear_bwd(dh, x, W, A, np.zeros_like(B), 2.0)
    assert np.all(dA == 0.0)


def test_row_restricted_helpers_agree_with_full():
    x, W, A, B, dh = _problem(M=6, n_in=8, n_out=5, r=2, seed=4)
    rows = np.array([0, 3, 5])
    h, _ = linear.linear_fwd(x, W, A, B, 2.0)
    dx, _, _ = linear.linear_bwd(dh, x, W, A, B, 2.0)
    assert np.array_equal(linear.linear_fwd_rows(x, W, A, B, 2.0, rows), h[rows])
    assert np.allclose(linear.linear_dx_rows(dh, W, A, B, 2.0, rows), dx[rows],
                       rtol=1e-13, atol=1e-13)


def test_quantized_base_forward_uses_dequantized_weight():
    """The base term of h uses dequant(W0): with B = 0 the layer output equals
    x times the oracle's dequantized weight, and the quantization error of
    the output is bounded by the weight round-trip bound."""
    rng = np.random.default_rng(5)
    W0 = (rng.standard_normal((8, 128)) * 0.02).astype(np.float32)
    q = nf4.quantize(W0)
    Wd = nf4.dequantize(q["codes"], q["q8"], q["step2"], q["mean"])
    x = rng.standard_normal((3, 128))
    A = np.zeros((2, 128)); B = np.zeros((8, 2))
    h, _ = linear.linear_fwd(x, Wd, A, B, 4.0)
    assert np.allclose(h, x @ Wd.T)
    err = np.abs(h - x @ W0.astype(np.float64).T)
    assert np.all(err <= np.abs(x).sum(axis=1, keepdims=True) * 0.2 * np.abs(W0).max())


@pytest.mark.parametrize("alpha", [3.0, 16.0])
def test_lora_grads_equal_linear_bwd(alpha):
    # alpha != r as well, so that the scale s = alpha / r is visible
    x, W, A, B, dh = _problem(M=5, n_in=6, n_out=4, r=3, seed=6)
    _, dA, dB = linear.linear_bwd(dh, x, W, A, B, alpha)
    gA, gB = linear.lora_grads(dh, x, A, B, alpha)
    assert np.allclose(gA, dA, rtol=1e-13, atol=1e-14) and np.allclose(gB, dB, rtol=1e-13, atol=1e-14)


# ---------------------------------------------------------------- LoRA dropout (reading D1)
def _keep(M, n, seed, p=0.3):
    return (np.random.default_rng(seed).random((M, n)) >= p).astype(np.float64)


def test_keep_mask_unpacking_matches_numpy_bit_order():
    rng = np.random.default_rng(5)
    bits = rng.integers(0, 256, (3, 4), dtype=np.uint8)
    want = np.unpackbits(bits, axis=1, bitorder="little").astype(np.float64)
    assert np.array_equal(linear.unpack_keep(bits, 32), want)


@pytest.mark.parametrize("p", [0.05, 0.5])
def test_dropout_backward_matches_central_differences(p):
    x, W, A, B, dh = _problem(seed=6)
    keep = _keep(*x.shape, seed=7)
    alpha = 4.0

    def loss(xx, AA, BB):
        h, _ = linear.linear_fwd_dropout(xx, W, AA, BB, alpha, keep, p)
        return float((dh * h).sum())

    dx, dA, dB = linear.linear_bwd_dropout(dh, x, W, A, B, alpha, keep, p)
    for g, a in [(_fd(lambda P: loss(P, A, B), x), dx), (_fd(lambda P: loss(x, P, B), A), dA),
                 (_fd(lambda P: loss(x, A, P), B), dB)]:
        assert np.allclose(g, a, rtol=1e-9, atol=1e-11)


def test_dropout_forward_brute_force_loops():
    x, W, A, B, _ = _problem(M=2, n_in=4, n_out=3, r=2, seed=8)
    keep = _keep(2, 4, seed=9, p=0.5)
    alpha, p = 3.0, 0.25
    s = alpha / 2
    h, _ = linear.linear_fwd_dropout(x, W, A, B, alpha, keep, p)
    for m in range(2):
        for o in range(3):
            v = sum(x[m, i] * W[o, i] for i in range(4))
            for j in range(2):
                v += s * B[o, j] * sum(x[m, i] * keep[m, i] / (1 - p) * A[j, i] for i in range(4))
            assert abs(h[m, o] - v) < 1e-12


def test_dropout_limits():
    """All kept with p = 0 is the plain layer; nothing kept leaves the base
    matmul and zero adapter gradients."""
    x, W, A, B, dh = _problem(seed=10)
    ones, zeros = np.ones_like(x), np.zeros_like(x)
    h0, _ = linear.linear_fwd(x, W, A, B, 2.0)
    h1, _ = linear.linear_fwd_dropout(x, W, A, B, 2.0, ones, 0.0)
    assert np.allclose(h0, h1, rtol=0, atol=1e-13)
    h2, _ = linear.linear_fwd_dropout(x, W, A, B, 2.0, zeros, 0.3)
    assert np.allclose(h2, x @ W.T, rtol=0, atol=1e-13)
    dx, dA, dB = linear.linear_bwd_dropout(dh, x, W, A, B, 2.0, zeros, 0.3)
    assert np.allclose(dx, dh @ W) and not dA.any() and not dB.any()
