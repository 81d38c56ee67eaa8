"""GPU parity of the QLoRA linear forward/backward against the fp64 oracle.

The GPU result is compared element by element with the oracle on the same
seeded inputs: h, us, dx, dA, dB within relative Frobenius error <= 2e-2 and
max-abs error <= 5e-2 x RMS(reference).  The oracle runs on its own
dequantized weight (bit-identical to the GPU's, checked in
test_gpu_quant.py) and exact fp64 arithmetic.

Small cases cover several tiles, ragged token counts, output widths that are
not a multiple of the 256-wide tile, ranks spanning more than one 64-wide
LoRA stage, both token-tile sizes (128 and 256 rows) and the few-token GEMV
path (M <= 16).  Full-size cases check sampled token rows of h and dx and the
complete dA, dB at the pages' Llama-shaped workloads, in the launch
configuration the benchmark times.
"""

import numpy as np
import pytest
import torch

from bit_nf4_quantized_11_b200 import synth
from oracle import linear, nf4
from parity import assert_close, to_np

pytestmark = [pytest.mark.gpu, pytest.mark.filterwarnings("ignore::RuntimeWarning")]


def _run(q, M, n_in, n_out, r, alpha, w_std=0.02, w_dist="normal", seed=0, backward=True,
         sample_rows=None, sample_out=None):
    """Run fwd (+bwd) on the GPU and compare with the oracle.  sample_rows
    restricts h/dx to those token rows; sample_out restricts h to those output
    features (forward only: dx needs every row of W0)."""
    p = synth.problem(M, n_in, n_out, r, w_std, w_dist, seed)
    dev = torch.device("cuda")
    w = q.quantize_nf4(p["W"].to(dev))
    x, A, B, dh = (p[k].to(dev) for k in ("x", "A", "B", "dh"))
    h, us = q.linear_fwd(x, w, A, B, alpha)
    if backward:
        dx, dA, dB = q.linear_bwd(dh, x, us, w, A, B, alpha)
    assert q.last_device_status() == 0

    # oracle on the same inputs and its own dequantized weight
    Wn = p["W"].numpy()
    outs = np.arange(n_out) if sample_out is None else np.asarray(sample_out)
    qo = nf4.quantize_rows(Wn, outs)
    Wd = nf4.dequantize(qo["codes"], qo["q8"], qo["step2"], qo["mean"], blocks=qo["blocks"])
    xn, An, Bn, dhn = (to_np(p[k]) for k in ("x", "A", "B", "dh"))
    s = alpha / r
    rows = np.arange(M) if sample_rows is None else np.asarray(sample_rows)
    h_ref = linear.linear_fwd_rows(xn, Wd, An, Bn[outs], alpha, rows)
    assert_close(to_np(h)[np.ix_(rows, outs)], h_ref, "h")
    assert_close(to_np(us)[rows], s * (xn[rows] @ An.T), "us")
    if backward:
        assert sample_out is None
        dx_ref = linear.linear_dx_rows(dhn, Wd, An, Bn, alpha, rows)
        assert_close(to_np(dx)[rows], dx_ref, "dx")
        dA_ref, dB_ref = linear.lora_grads(dhn, xn, An, Bn, alpha)
        assert_close(to_np(dA), dA_ref, "dA")
        assert_close(to_np(dB), dB_ref, "dB")


@pytest.mark.parametrize("M,n_in,n_out,r,alpha", [
    (64, 512, 512, 8, 16.0),        # the small parity layer
    (300, 640, 320, 16, 32.0),      # ragged M, 320 = 256 + 64 output columns, 10 K stages
    (129, 256, 768, 32, 8.0),       # one row past a 128-row tile
    (200, 256, 192, 136, 16.0),     # rank spanning three 64-wide LoRA stages
    (1100, 512, 768, 64, 16.0),     # 256-row token tiles, ragged
])
def test_linear_small_shapes(cuda_lib, M, n_in, n_out, r, alpha):
    _run(cuda_lib, M, n_in, n_out, r, alpha, seed=M)


@pytest.mark.parametrize("M", [1, 4, 9, 16])
def test_few_token_gemv(cuda_lib, M):
    _run(cuda_lib, M, 1024, 768, 16, 32.0, seed=M, backward=True)


@pytest.mark.parametrize("M,r", [(9, 256), (16, 136), (2, 64)])
def test_few_token_ranks(cuda_lib, M, r):
    # the few-token rank-r kernel at the largest rank, a rank spanning three
    # 64-wide stages, and with its partials over four K chunks
    _run(cuda_lib, M, 1024, 768, r, 16.0, seed=300 + r, backward=True)


@pytest.mark.parametrize("M,n_in,n_out", [(3, 576, 320), (12, 192, 448), (1, 64, 64), (16, 64, 1088),
                                           (7, 4160, 576)])
def test_few_token_ragged(cuda_lib, M, n_in, n_out):
    # K with a half 128-column unit (in % 128 == 64), a partial last row tile,
    # a single unit, and more row tiles than a CTA range spans
    _run(cuda_lib, M, n_in, n_out, 8, 16.0, seed=100 + M, backward=False)


@pytest.mark.parametrize("M,n_in,n_out,alpha", [
    (520, 512, 640, 16.0),    # CTA-pair GEMM: four 64-wide LoRA stages in the K loop
    (100, 256, 320, 8.0),     # one-CTA GEMM
    (5, 512, 384, 16.0),      # few-token GEMV forward, GEMM backward
])
def test_largest_rank(cuda_lib, M, n_in, n_out, alpha):
    # r = 256, the largest rank the library takes
    _run(cuda_lib, M, n_in, n_out, 256, alpha, seed=M + 7)


@pytest.mark.parametrize("r", [1, 4, 12, 20])
@pytest.mark.parametrize("M,n_in,n_out", [
    (520, 512, 640),      # CTA-pair GEMM
    (100, 256, 320),      # one-CTA GEMM
    (5, 576, 384),        # few-token GEMV forward, GEMM backward
])
def test_rank_not_multiple_of_8(cuda_lib, M, n_in, n_out, r):
    # any rank 1 <= r <= 256: the layer runs on zero-padded copies at r rounded up to 8
    _run(cuda_lib, M, n_in, n_out, r, 2.0 * r, seed=M + r)


@pytest.mark.parametrize("M,n_in,n_out", [(4096, 512, 2560), (4096, 2560, 512)])
def test_two_waves_short_k(cuda_lib, M, n_in, n_out):
    # 80 output tiles of 512 x 256: more tiles than co-resident CTA pairs, so
    # pairs take a second tile; short K on one side, forward and dx in turn
    _run(cuda_lib, M, n_in, n_out, 16, 32.0, seed=M + n_in)


def test_zero_adapter_is_plain_quantized_matmul(cuda_lib):
    """B = 0: h equals x dequant(W0)^T, dA = 0 exactly."""
    q = cuda_lib
    p = synth.problem(256, 512, 384, 16, seed=5)
    dev = torch.device("cuda")
    w = q.quantize_nf4(p["W"].to(dev))
    Wd = q.dequantize_nf4(w)
    x, A, dh = p["x"].to(dev), p["A"].to(dev), p["dh"].to(dev)
    B = torch.zeros(384, 16, dtype=torch.bfloat16, device=dev)
    h, us = q.linear_fwd(x, w, A, B, 32.0)
    ref = (x.double() @ Wd.double().T)
    assert_close(to_np(h), ref.cpu().numpy(), "h")
    _, dA, _ = q.linear_bwd(dh, x, us, w, A, B, 32.0)
    assert torch.all(dA == 0)


def _sample(M, k=256, seed=0):
    rng = np.random.default_rng(seed)
    rows = np.sort(rng.choice(M, k, replace=False))
    rows[0], rows[-1] = 0, M - 1
    return rows


def test_full_size_7b_attention(cuda_lib):
    _run(cuda_lib, 4096, 4096, 4096, 16, 32.0, sample_rows=_sample(4096))


def test_full_size_7b_mlp_gate(cuda_lib):
    _run(cuda_lib, 8192, 4096, 11008, 16, 32.0, w_dist="student_t5", sample_rows=_sample(8192, 128))


def test_full_size_65b_down(cuda_lib):
    _run(cuda_lib, 2048, 22016, 8192, 64, 16.0, w_std=0.01, sample_rows=_sample(2048, 128))


def test_full_size_7b_mlp_down(cuda_lib):
    _run(cuda_lib, 8192, 11008, 4096, 16, 32.0, w_dist="student_t5", sample_rows=_sample(8192, 128))


@pytest.mark.parametrize("n_in,n_out", [(8192, 8192), (8192, 22016)])
def test_full_size_65b_layer(cuda_lib, n_in, n_out):
    # q/k/v/o share the 8192 x 8192 shape; gate and up share 8192 -> 22016
    _run(cuda_lib, 2048, n_in, n_out, 64, 16.0, w_std=0.01, seed=n_out, sample_rows=_sample(2048, 128))


@pytest.mark.parametrize("M,n_in,n_out", [(1, 8192, 28672), (4, 8192, 28672), (16, 8192, 28672),
                                           (1, 28672, 8192), (4, 28672, 8192), (16, 28672, 8192)])
def test_full_size_70b_gemv(cuda_lib, M, n_in, n_out):
    _run(cuda_lib, M, n_in, n_out, 16, 32.0, w_std=0.015, backward=False,
         sample_out=_sample(n_out, 512, seed=M))
