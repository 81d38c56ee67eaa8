"""GPU parity of the bf16-input quantizer and of the adapter merge (and its
lossy re-quantization) against the oracle, bit for bit."""

import numpy as np
import pytest
import torch

from bit_nf4_quantized_11_b200 import synth
from oracle import merge, nf4
from parity import bf16_bits, f32_bits

pytestmark = [pytest.mark.gpu, pytest.mark.filterwarnings("ignore::RuntimeWarning")]


def _check_quant_bf16(q, Wb, sample_rows=None):
    bits = bf16_bits(Wb)
    w = q.quantize_nf4(Wb.cuda())
    assert q.last_device_status() == 0
    if sample_rows is None:
        ref = nf4.quantize_bf16(bits)
        assert np.array_equal(w.codes.cpu().numpy(), ref["packed"])
        q8, step2, mean = ref["q8"], ref["step2"], ref["mean"]
    else:
        Wn = nf4.bf16_to_f64(bits)
        rows = np.asarray(sample_rows)
        c = nf4.block_absmax(Wn)
        q8, step2, mean = nf4.double_quantize(c)
        nbr = Wn.shape[1] // 64
        blk = (rows[:, None] * nbr + np.arange(nbr)[None, :]).ravel()
        assert np.array_equal(w.codes.cpu().numpy()[rows], nf4.pack(nf4.encode(Wn[rows], c[blk])))
    assert f32_bits(w.mean)[0] == nf4.f32_bits(mean)
    assert np.array_equal(f32_bits(w.step2), nf4.f32_bits(step2))
    assert np.array_equal(w.q8.cpu().numpy(), q8)
    return w


@pytest.mark.parametrize("rows,cols,std,seed", [(1, 64, 0.02, 0), (300, 640, 0.02, 1), (512, 512, 0.02, 2),
                                               (1024, 1024, 0.015, 3)])
def test_quantize_bf16_input_bit_exact(cuda_lib, rows, cols, std, seed):
    _check_quant_bf16(cuda_lib, synth.weight(rows, cols, std, "normal", seed).to(torch.bfloat16))


def test_quantize_bf16_degenerate_blocks(cuda_lib):
    W = synth.weight(64, 512, 0.02, "normal", 7).numpy().copy()
    W[0, :64] = 0.0
    W[1, :] = -0.0
    W[2, 64:128] = np.float32(1e-38)
    W[3, :64] = 1e4 * np.sign(W[3, :64])
    _check_quant_bf16(cuda_lib, torch.from_numpy(W).to(torch.bfloat16))


def test_quantize_bf16_equals_fp32_of_widened(cuda_lib):
    Wb = synth.weight(256, 1024, 0.02, "student_t5", 4).to(torch.bfloat16)
    a = cuda_lib.quantize_nf4(Wb.cuda())
    b = cuda_lib.quantize_nf4(Wb.float().cuda())
    for x, y in ((a.codes, b.codes), (a.q8, b.q8), (a.step2, b.step2), (a.mean, b.mean)):
        assert torch.equal(x, y)


def _merge_case(q, out_f, in_f, r, alpha, seed, sample_rows=None):
    p = synth.problem(8, in_f, out_f, r, seed=seed)
    W, A, B = p["W"], p["A"], p["B"]
    w = q.quantize_nf4(W.cuda())
    got = q.merge_adapter(w, A.cuda(), B.cuda(), alpha)
    assert q.last_device_status() == 0
    ref_q = nf4.quantize(W.numpy())
    w_hat = nf4.dequantize_bits(ref_q["codes"], ref_q["q8"], ref_q["step2"], ref_q["mean"])
    rows = np.arange(out_f) if sample_rows is None else np.asarray(sample_rows)
    want = merge.merge_adapter_bits(w_hat[rows], bf16_bits(A), bf16_bits(B)[rows], alpha)
    assert np.array_equal(bf16_bits(got)[rows], want)
    return got


@pytest.mark.parametrize("out_f,in_f,r,alpha", [(64, 128, 8, 16.0), (320, 640, 16, 32.0), (128, 256, 64, 16.0),
                                                (64, 64, 1, 1.0), (192, 512, 136, 8.0)])
def test_merge_adapter_bit_exact(cuda_lib, out_f, in_f, r, alpha):
    _merge_case(cuda_lib, out_f, in_f, r, alpha, seed=r)


def test_merge_adapter_full_size_sampled_rows(cuda_lib):
    rng = np.random.default_rng(0)
    rows = np.sort(rng.choice(4096, 32, replace=False))
    _merge_case(cuda_lib, 4096, 4096, 16, 32.0, seed=11, sample_rows=rows)


def test_requantize_merged_weight_bit_exact(cuda_lib):
    """The lossy merge back into 4 bit: the bf16 merged weight re-quantized."""
    merged = _merge_case(cuda_lib, 256, 1024, 16, 32.0, seed=5)
    _check_quant_bf16(cuda_lib, merged.cpu())
