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
