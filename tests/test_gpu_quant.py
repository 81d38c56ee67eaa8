"""GPU parity of the NF4 quantizer and dequantizer against the oracle:
bit-exact packed codes, second-level int8 codes, steps, mean and bf16
dequantized weights, on seeded synthetic weights and on the degenerate cases
(zero blocks, equal-absmax blocks, signed zeros, subnormals, a partial last
scale group, multi-pass summation trees), through the C ABI."""

import numpy as np
import pytest
import torch

from bit_nf4_quantized_11_b200 import synth
from oracle import nf4
from parity import bf16_bits, f32_bits

pytestmark = [pytest.mark.gpu, pytest.mark.filterwarnings("ignore::RuntimeWarning")]


def _check_quant(q, W_cpu, sample_rows=None):
    """Quantize on the GPU and compare every stored array with the oracle.
    With sample_rows, the first-level codes and dequantized weights are
    compared on those rows only (the scale statistics are still global)."""
    Wn = W_cpu.numpy()
    w = q.quantize_nf4(W_cpu.cuda())
    deq = q.dequantize_nf4(w)
    assert q.last_device_status() == 0
    c = nf4.block_absmax(Wn)
    q8, step2, mean = nf4.double_quantize(c)
    assert f32_bits(w.mean)[0] == nf4.f32_bits(mean)
    assert np.array_equal(f32_bits(w.step2), nf4.f32_bits(step2))
    assert np.array_equal(w.q8.cpu().numpy(), q8)
    rows = np.arange(Wn.shape[0]) if sample_rows is None else np.asarray(sample_rows)
    nbr = Wn.shape[1] // 64
    blk = (rows[:, None] * nbr + np.arange(nbr)[None, :]).ravel()
    codes = nf4.encode(Wn[rows], c[blk])
    assert np.array_equal(w.codes.cpu().numpy()[rows], nf4.pack(codes))
    assert np.array_equal(bf16_bits(deq)[rows], nf4.dequantize_bits(codes, q8, step2, mean, blocks=blk))
    return w


@pytest.mark.parametrize("rows,cols,dist,std,seed", [
    (1, 64, "normal", 0.02, 0),          # one block
    (64, 64, "normal", 0.02, 1),
    (300, 640, "normal", 0.02, 2),       # 3000 blocks: partial last group (3000 % 256 = 184)
    (512, 512, "normal", 0.02, 0),       # the small parity layer
    (257, 1088, "student_t5", 0.02, 3),  # heavy tails, odd row count
    (1024, 1024, "normal", 0.015, 4),    # 16384 blocks: 4 tree chunks finished by the last CTA
])
def test_quantize_bit_exact(cuda_lib, rows, cols, dist, std, seed):
    _check_quant(cuda_lib, synth.weight(rows, cols, std, dist, seed))


def test_degenerate_blocks_bit_exact(cuda_lib):
    W = synth.weight(64, 512, 0.02, "normal", 7).numpy().copy()
    W[0, :64] = 0.0                                  # all-zero block
    W[1, :] = -0.0                                   # a row of negative zeros
    W[2, 64:128] = np.float32(1e-40)                 # subnormal block
    W[3, 128:192] = np.linspace(-1e-38, 1e-38, 64, dtype=np.float32)
    W[4, :64] = 1e4 * np.sign(W[4, :64])             # large magnitude
    W[6, :64] = 0.0                                  # absmax whose reciprocal overflows
    W[6, :5] = [2e-39, -2e-39, 0.0, -0.0, 1e-39]
    W[5, 3] = -0.0
    w = _check_quant(cuda_lib, torch.from_numpy(W))
    codes = w.codes.cpu().numpy()
    assert np.all(codes[0, :32] == 0x77) and np.all(codes[1] == 0x77)


def test_subnormal_tensor_divides_at_both_levels(cuda_lib):
    """Weights ~1e-39: most blocks' absmax reciprocals overflow (first-level
    division path) and every group's step is subnormal, so the second-level
    codes take the division path too."""
    W = (synth.weight(64, 1024, 1.0, "normal", 8).numpy() * np.float32(1e-39)).astype(np.float32)
    c = nf4.block_absmax(W)
    _, step2, _ = nf4.double_quantize(c)
    with np.errstate(over="ignore", divide="ignore"):
        assert np.any(~np.isfinite(np.float32(1.0) / c.astype(np.float32)))
        assert np.all(~np.isfinite(np.float32(1.0) / step2.astype(np.float32)))
    _check_quant(cuda_lib, torch.from_numpy(W))


def test_equal_absmax_gives_zero_second_level(cuda_lib):
    rng = np.random.default_rng(3)
    W = rng.uniform(-0.5, 0.5, (16, 1024)).astype(np.float32)
    W[:, ::64] = 0.5
    w = _check_quant(cuda_lib, torch.from_numpy(W))
    assert torch.all(w.q8 == 0) and torch.all(w.step2 == 0)
    assert w.mean.item() == 0.5


@pytest.mark.parametrize("shape,dist,std", [
    ((4096, 4096), "normal", 0.02),        # 7B attention projection, full tensor
    ((11008, 4096), "student_t5", 0.02),   # 7B MLP gate/up, full tensor
])
def test_quantize_full_size_bit_exact(cuda_lib, shape, dist, std):
    _check_quant(cuda_lib, synth.weight(shape[0], shape[1], std, dist, 0))


@pytest.mark.parametrize("shape,std", [((28672, 8192), 0.015), ((8192, 22016), 0.01)])
def test_quantize_70b_65b_shapes_sampled_rows(cuda_lib, shape, std):
    rng = np.random.default_rng(0)
    rows = np.sort(rng.choice(shape[0], 48, replace=False))
    rows[0], rows[-1] = 0, shape[0] - 1
    _check_quant(cuda_lib, synth.weight(shape[0], shape[1], std, "normal", 0), sample_rows=rows)


def test_quantize_extra_tree_pass_sampled_rows(cuda_lib):
    """8200 x 32768: 4 198 400 blocks leave 1025 sums of 4096-leaf subtrees,
    more than the 1024 that the last CTA of a tree pass finishes, so a second
    pass over them runs (and its last CTA writes the mean)."""
    rng = np.random.default_rng(1)
    rows = np.sort(rng.choice(8200, 16, replace=False))
    rows[0], rows[-1] = 0, 8199
    _check_quant(cuda_lib, synth.weight(8200, 32768, 0.02, "normal", 5), sample_rows=rows)


def test_dequantize_matches_codebook_levels_exactly(cuda_lib):
    """A block whose values are exactly c * level[j] reproduces its codes."""
    lv, _ = cuda_lib.codebook()
    c = np.float32(0.0371)
    w = (c * np.array(lv, dtype=np.float32)).astype(np.float32)
    W = np.tile(w, 8).reshape(2, 64)
    qw = cuda_lib.quantize_nf4(torch.from_numpy(W).cuda())
    codes = nf4.unpack(qw.codes.cpu().numpy())
    assert np.array_equal(codes, np.tile(np.arange(16, dtype=np.uint8), 8).reshape(2, 64))


def _sharded(q, W, world):
    """Quantize W as `world` ranks would, the ranks run one after another on
    this GPU (independent launches; the all-gather is a concatenation in rank
    order), and assemble the whole weight."""
    flat = W.reshape(-1)
    n_total = flat.numel() // 64
    locals_ = []
    for k in range(world):
        b0, b1, cpr = q.quantize_shard_plan(n_total, world, k)
        codes, roots, ws = q.quantize_nf4_shard_local(flat[b0 * 64:b1 * 64], cpr, world * cpr)
        locals_.append((b0, b1, codes, roots, ws))
    roots_all = torch.cat([l[3] for l in locals_])
    parts = [q.quantize_nf4_shard_finish(roots_all, n_total, b1 - b0, ws) for b0, b1, _, _, ws in locals_]
    assert q.last_device_status() == 0
    means = [p[2] for p in parts]
    assert all(torch.equal(m, means[0]) for m in means)
    return (torch.cat([l[2] for l in locals_]), torch.cat([p[0] for p in parts]),
            torch.cat([p[1] for p in parts]), means[0])


@pytest.mark.parametrize("rows,cols,dist,world", [
    (37, 8192, "student_t5", 2),    # a whole 4096-block chunk and a partial one
    (37, 8192, "normal", 3),        # the third rank holds no block
    (300, 640, "normal", 4),        # one partial chunk: ranks 1..3 empty
    (4096, 11008, "student_t5", 8), # 172 chunks, 22 per rank, the last rank short
])
def test_sharded_quantize_equals_single_call(cuda_lib, rows, cols, dist, world):
    q = cuda_lib
    W = synth.weight(rows, cols, 0.02, dist, 21).cuda()
    codes, q8, step2, mean = _sharded(q, W, world)
    w = q.quantize_nf4(W)
    assert torch.equal(codes, w.codes.reshape(-1))
    assert torch.equal(q8, w.q8)
    assert torch.equal(step2.view(torch.int32), w.step2.view(torch.int32))
    assert torch.equal(mean.view(torch.int32), w.mean.view(torch.int32))
    if rows * cols <= 37 * 8192:
        ref = nf4.quantize(W.cpu().numpy())
        assert np.array_equal(codes.cpu().numpy(), ref["packed"].reshape(-1))
        assert np.array_equal(q8.cpu().numpy(), ref["q8"])
        assert np.array_equal(f32_bits(step2), nf4.f32_bits(ref["step2"]))
        assert f32_bits(mean)[0] == nf4.f32_bits(ref["mean"])


def test_sharded_quantize_extra_tree_pass(cuda_lib):
    """8200 x 32768 over 2 ranks: 2 x 513 gathered chunk sums, more than one
    finishing CTA takes, so the finishing call runs a second tree pass."""
    q = cuda_lib
    W = synth.weight(8200, 32768, 0.02, "normal", 5).cuda()
    codes, q8, step2, mean = _sharded(q, W, 2)
    w = q.quantize_nf4(W)
    assert torch.equal(codes, w.codes.reshape(-1))
    assert torch.equal(q8, w.q8)
    assert torch.equal(step2.view(torch.int32), w.step2.view(torch.int32))
    assert torch.equal(mean.view(torch.int32), w.mean.view(torch.int32))
