"""Data-parallel step on CPU: two gloo ranks, each with its token shard,
sum their adapter gradients; the sum must equal the whole batch's gradient
(the oracle on all tokens).  Shard bounds cover every token exactly once."""

import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from bit_nf4_quantized_11_b200 import dp, synth
from oracle.linear import lora_grads


def test_shard_bounds_cover_batch():
    for M in (0, 1, 7, 64, 4097):
        for world in (1, 2, 3, 8):
            spans = [dp.shard_bounds(M, world, k) for k in range(world)]
            assert spans[0][0] == 0 and spans[-1][1] == M
            for (a0, a1), (b0, b1) in zip(spans, spans[1:]):
                assert a1 == b0
            sizes = [b - a for a, b in spans]
            assert max(sizes) - min(sizes) <= 1
    with pytest.raises(ValueError):
        dp.shard_bounds(4, 2, 2)


def test_adapter_grad_buffers_are_views():
    flat, dA, dB = dp.adapter_grad_buffers(8, 64, 128, "cpu")
    assert dA.shape == (8, 64) and dB.shape == (128, 8)
    dA.fill_(1.0)
    dB.fill_(2.0)
    assert float(flat.sum()) == 8 * 64 + 2 * 128 * 8


M, N_IN, N_OUT, R, ALPHA = 37, 128, 64, 8, 16.0


def _rank(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    torch.distributed.init_process_group("gloo", rank=rank, world_size=world)
    try:
        p = synth.problem(M, N_IN, N_OUT, R, seed=3)
        b, e = dp.shard_bounds(M, world, rank)
        dA, dB = lora_grads(p["dh"][b:e].double().numpy(), p["x"][b:e].double().numpy(),
                            p["A"].double().numpy(), p["B"].double().numpy(), ALPHA)
        flat = torch.cat([torch.from_numpy(dA).reshape(-1), torch.from_numpy(dB).reshape(-1)]).float()
        dp.allreduce_adapter_grads(flat)
        if rank == 0:
            out.put(flat.numpy().copy())
    finally:
        torch.distributed.destroy_process_group()


def test_layer_grad_buffers_are_disjoint_views():
    shapes = [(64, 128), (128, 96), (96, 64)]
    flat, views = dp.layer_grad_buffers(8, shapes, "cpu")
    assert flat.numel() == sum(8 * a + b * 8 for a, b in shapes)
    flat.zero_()
    for i, ((dA, dB), (n_in, n_out)) in enumerate(zip(views, shapes)):
        assert dA.shape == (8, n_in) and dB.shape == (n_out, 8)
        dA.fill_(2 * i + 1)
        dB.fill_(2 * i + 2)
    # every element of the flat buffer belongs to exactly one view, in order
    want = torch.cat([torch.full((8 * a,), 2.0 * i + 1) if j == 0 else torch.full((b * 8,), 2.0 * i + 2)
                      for i, (a, b) in enumerate(shapes) for j in (0, 1)])
    assert torch.equal(flat, want)


def test_two_rank_adapter_gradient_sum():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    procs = [ctx.Process(target=_rank, args=(k, 2, port, out)) for k in range(2)]
    for p in procs:
        p.start()
    got = out.get(timeout=120)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    p = synth.problem(M, N_IN, N_OUT, R, seed=3)
    dA, dB = lora_grads(p["dh"].double().numpy(), p["x"].double().numpy(),
                        p["A"].double().numpy(), p["B"].double().numpy(), ALPHA)
    want = np.concatenate([dA.reshape(-1), dB.reshape(-1)])
    # fp32 all-reduce of two fp32-rounded partial sums against the fp64 whole
    np.testing.assert_allclose(got, want, rtol=1e-5, atol=1e-6 * np.abs(want).max())


# ---------------------------------------------------------------------------
# sharded quantization: the host side (shard plan from the C library, the
# all-gathers, padding and assembly) on gloo ranks, with the per-rank compute
# done by the oracle; the assembled weight must equal the oracle's
# quantization of the whole tensor, bit for bit.

class _OracleShardLib:
    """The per-rank calls of the sharded quantizer computed by the oracle (test only)."""

    def quantize_shard_plan(self, n, world, rank):
        import bit_nf4_quantized_11_b200 as q
        return q.quantize_shard_plan(n, world, rank)

    def quantize_nf4_shard_local(self, W_shard, cpr, n_roots_total):
        from oracle import nf4
        Wn = W_shard.numpy().astype(np.float32).astype(np.float64).reshape(-1, 64)
        c = nf4.block_absmax(Wn) if Wn.size else np.zeros(0)
        codes = nf4.pack(nf4.encode(Wn, c)).reshape(-1) if Wn.size else np.zeros(0, np.uint8)
        roots = np.array([nf4.pairwise_sum(c[i * 4096:(i + 1) * 4096]) if i * 4096 < c.size else 0.0
                          for i in range(cpr)])
        return torch.from_numpy(codes.astype(np.uint8)), torch.from_numpy(roots), c

    def quantize_nf4_shard_finish(self, roots_all, n_total, n_shard, ws):
        from oracle import nf4
        mean = float(nf4.fl32(nf4.pairwise_sum(roots_all.numpy()) / float(n_total)))
        q8, step2 = nf4.second_level(ws, mean) if n_shard else (np.zeros(0, np.int8), np.zeros(0))
        return (torch.from_numpy(q8), torch.from_numpy(step2.astype(np.float32)),
                torch.tensor([mean], dtype=torch.float32))


QROWS, QCOLS = 37, 8192          # 4736 blocks: one whole 4096-block chunk and a partial one


def _quant_rank(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    torch.distributed.init_process_group("gloo", rank=rank, world_size=world)
    try:
        W = synth.weight(QROWS, QCOLS, 0.02, "student_t5", 11).reshape(-1)
        n_total = W.numel() // 64
        lib = _OracleShardLib()
        b0, b1, _ = lib.quantize_shard_plan(n_total, world, rank)
        shard = dp.quantize_nf4_sharded(W[b0 * 64:b1 * 64].contiguous(), n_total, lib=lib)
        codes, q8, step2, mean = dp.gather_nf4_replica(shard, n_total)
        if rank == 0:
            out.put((codes.numpy().copy(), q8.numpy().copy(), step2.numpy().copy(), float(mean[0])))
    finally:
        torch.distributed.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_sharded_quantize_assembles_the_whole_weight(world):
    from oracle import nf4
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    procs = [ctx.Process(target=_quant_rank, args=(k, world, port, out)) for k in range(world)]
    for p in procs:
        p.start()
    codes, q8, step2, mean = out.get(timeout=180)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    W = synth.weight(QROWS, QCOLS, 0.02, "student_t5", 11).numpy()
    ref = nf4.quantize(W)
    assert np.float32(mean).view(np.uint32) == nf4.f32_bits(ref["mean"])
    assert np.array_equal(q8, ref["q8"])
    assert np.array_equal(nf4.f32_bits(step2.astype(np.float64)), nf4.f32_bits(ref["step2"]))
    assert np.array_equal(codes, ref["packed"].reshape(-1))


def test_shard_plan_aligns_chunks_and_covers_blocks():
    import bit_nf4_quantized_11_b200 as q
    for n in (1, 4095, 4096, 4097, 4736, 704512, 3 * 4096 + 5):
        for world in (1, 2, 3, 8):
            spans = [q.quantize_shard_plan(n, world, k) for k in range(world)]
            cpr = spans[0][2]
            assert all(s[2] == cpr for s in spans) and world * cpr * 4096 >= n
            assert spans[0][0] == 0 and spans[-1][1] == n
            for (a0, a1, _), (c0, c1, _) in zip(spans, spans[1:]):
                assert a1 == c0
            for b0, b1, _ in spans:
                assert (b0 == b1 == n or b0 % 4096 == 0) and b1 - b0 <= cpr * 4096   # empty trailing ranks sit at n
    with pytest.raises(q.QLoRAError):
        q.quantize_shard_plan(10, 2, 2)


def test_sharded_quantize_single_process_is_the_whole_weight():
    """World of one (no process group): the plan gives rank 0 every block and
    the gather returns the shard itself."""
    from oracle import nf4
    W = synth.weight(37, 8192, 0.02, "normal", 12).reshape(-1)
    n_total = W.numel() // 64
    shard = dp.quantize_nf4_sharded(W, n_total, lib=_OracleShardLib())
    assert (shard.block_begin, shard.block_end) == (0, n_total)
    codes, q8, step2, mean = dp.gather_nf4_replica(shard, n_total)
    ref = nf4.quantize(W.numpy().reshape(37, 8192))
    assert np.array_equal(codes.numpy(), ref["packed"].reshape(-1))
    assert np.array_equal(q8.numpy(), ref["q8"])
    assert np.array_equal(nf4.f32_bits(step2.numpy().astype(np.float64)), nf4.f32_bits(ref["step2"]))
    assert np.float32(mean[0]).view(np.uint32) == nf4.f32_bits(ref["mean"])
