"""GPU parity of the uniform INT4 comparison code (same kernels, INT4 level
table) against the oracle, bit for bit, and the NF4 < INT4 error ordering on
normally distributed weights measured on the GPU outputs."""

import numpy as np
import pytest
import torch

from bit_nf4_quantized_11_b200 import synth
from oracle import int4, nf4
from parity import bf16_bits, f32_bits

pytestmark = [pytest.mark.gpu, pytest.mark.filterwarnings("ignore::RuntimeWarning")]


def _check_int4(q, W_cpu):
    Wn = W_cpu.numpy()
    w = q.quantize_codebook(W_cpu.cuda(), q.CODEBOOK_INT4)
    deq = q.dequantize_codebook(w, q.CODEBOOK_INT4)
    assert q.last_device_status() == 0
    ref = int4.quantize(Wn)
    assert np.array_equal(w.codes.cpu().numpy(), ref["packed"])
    assert np.array_equal(w.q8.cpu().numpy(), ref["q8"])
    assert np.array_equal(f32_bits(w.step2), nf4.f32_bits(ref["step2"]))
    assert f32_bits(w.mean)[0] == nf4.f32_bits(ref["mean"])
    assert np.array_equal(bf16_bits(deq), int4.dequantize_bits(ref["codes"], ref["q8"], ref["step2"], ref["mean"]))
    return w, deq


@pytest.mark.parametrize("rows,cols,dist,seed", [(1, 64, "normal", 0), (300, 640, "normal", 1),
                                                 (512, 512, "student_t5", 2), (1024, 1024, "normal", 3)])
def test_int4_bit_exact(cuda_lib, rows, cols, dist, seed):
    _check_int4(cuda_lib, synth.weight(rows, cols, 0.02, dist, seed))


def test_int4_degenerate_blocks(cuda_lib):
    W = synth.weight(64, 512, 0.02, "normal", 7).numpy().copy()
    W[0, :64] = 0.0
    W[1, :] = -0.0
    W[2, 64:128] = np.float32(1e-40)
    W[3, :64] = 1e4 * np.sign(W[3, :64])
    W[4, :64] = 0.0
    W[4, :5] = [2e-39, -2e-39, 0.0, -0.0, 1e-39]
    _check_int4(cuda_lib, torch.from_numpy(W))


def test_nf4_error_below_int4_on_gpu(cuda_lib):
    W = synth.weight(4096, 4096, 0.02, "normal", 0).cuda()
    e_nf4 = (cuda_lib.dequantize_nf4(cuda_lib.quantize_nf4(W)).float() - W).norm() / W.norm()
    w4 = cuda_lib.quantize_codebook(W, cuda_lib.CODEBOOK_INT4)
    e_int4 = (cuda_lib.dequantize_codebook(w4, cuda_lib.CODEBOOK_INT4).float() - W).norm() / W.norm()
    assert float(e_nf4) < 0.9 * float(e_int4)
