"""GPU parity of the layer with LoRA dropout (keep mask drawn on the host,
passed as bits) against the fp64 oracle, with the tolerance of the plain
layer: relative Frobenius <= 2e-2 and max-abs <= 5e-2 x RMS(reference)."""

import numpy as np
import pytest
import torch

import bit_nf4_quantized_11_b200 as qmod
from bit_nf4_quantized_11_b200 import synth
from oracle import linear, nf4
from parity import assert_close, to_np

pytestmark = [pytest.mark.gpu, pytest.mark.filterwarnings("ignore::RuntimeWarning")]


def _run(q, M, n_in, n_out, r, alpha, p, seed=0, sample_rows=None):
    prob = synth.problem(M, n_in, n_out, r, seed=seed)
    keep = torch.from_numpy(np.random.default_rng(seed + 99).random((M, n_in)) >= p)
    dev = torch.device("cuda")
    keep_bits = qmod.pack_keep_mask(keep.to(dev))
    w = q.quantize_nf4(prob["W"].to(dev))
    x, A, B, dh = (prob[k].to(dev) for k in ("x", "A", "B", "dh"))
    h, us = q.linear_fwd_dropout(x, w, A, B, alpha, keep_bits, p)
    dx, dA, dB = q.linear_bwd_dropout(dh, x, us, w, A, B, alpha, keep_bits, p)
    assert q.last_device_status() == 0

    k = keep.numpy().astype(np.float64)
    assert np.array_equal(linear.unpack_keep(keep_bits.cpu().numpy(), n_in), k)
    qo = nf4.quantize(prob["W"].numpy())
    Wd = nf4.dequantize(qo["codes"], qo["q8"], qo["step2"], qo["mean"])
    xn, An, Bn, dhn = (to_np(prob[t]) for t in ("x", "A", "B", "dh"))
    rows = np.arange(M) if sample_rows is None else np.asarray(sample_rows)
    h_ref, u_ref = linear.linear_fwd_dropout(xn[rows], Wd, An, Bn, alpha, k[rows], p)
    assert_close(to_np(h)[rows], h_ref, "h")
    assert_close(to_np(us)[rows], (alpha / r) * u_ref, "us")
    dx_ref, dA_ref, dB_ref = linear.linear_bwd_dropout(dhn, xn, Wd, An, Bn, alpha, k, p)
    assert_close(to_np(dx)[rows], dx_ref[rows], "dx")
    assert_close(to_np(dA), dA_ref, "dA")
    assert_close(to_np(dB), dB_ref, "dB")


@pytest.mark.parametrize("M,n_in,n_out,r,alpha,p", [
    (64, 512, 512, 8, 16.0, 0.05),
    (300, 640, 320, 16, 32.0, 0.5),
    (129, 256, 768, 32, 8.0, 0.05),
    (200, 256, 192, 136, 16.0, 0.2),
    (9, 1024, 768, 16, 32.0, 0.05),      # few-token path
    (300, 640, 320, 12, 24.0, 0.1),      # rank not a multiple of 8 (padded copies)
    (130, 576, 320, 8, 16.0, 0.1),       # in % 128 == 64: a half-width column tile in the dx pass
    (7, 512, 384, 5, 10.0, 0.1),
])
def test_dropout_layer_small(cuda_lib, M, n_in, n_out, r, alpha, p):
    _run(cuda_lib, M, n_in, n_out, r, alpha, p, seed=M)


def test_dropout_p0_all_kept_equals_plain_layer(cuda_lib):
    """p = 0 with every element kept is the plain layer, bit for bit in the
    forward and in dA, dB (the same rank-r kernels run, the mask changes
    nothing); dx takes one more bf16 rounding (the masked rank-r term is
    added after the base GEMM)."""
    q = cuda_lib
    prob = synth.problem(256, 512, 384, 16, seed=3)
    dev = torch.device("cuda")
    w = q.quantize_nf4(prob["W"].to(dev))
    x, A, B, dh = (prob[k].to(dev) for k in ("x", "A", "B", "dh"))
    keep_bits = torch.full((256, 64), 255, dtype=torch.uint8, device=dev)
    h0, us0 = q.linear_fwd(x, w, A, B, 32.0)
    h1, us1 = q.linear_fwd_dropout(x, w, A, B, 32.0, keep_bits, 0.0)
    assert torch.equal(h0, h1) and torch.equal(us0, us1)
    dx0, dA0, dB0 = q.linear_bwd(dh, x, us0, w, A, B, 32.0)
    dx1, dA1, dB1 = q.linear_bwd_dropout(dh, x, us1, w, A, B, 32.0, keep_bits, 0.0)
    assert torch.equal(dA0, dA1) and torch.equal(dB0, dB1)
    assert_close(to_np(dx1), to_np(dx0).astype(np.float64), "dx")   # dx differs by one extra rounding


def test_dropout_full_size_7b_attention(cuda_lib):
    rng = np.random.default_rng(0)
    rows = np.sort(rng.choice(4096, 64, replace=False))
    _run(cuda_lib, 4096, 4096, 4096, 16, 32.0, 0.05, seed=1, sample_rows=rows)
