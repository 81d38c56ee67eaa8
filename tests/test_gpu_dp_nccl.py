"""The data-parallel helpers over a real NCCL process group on one GPU.

A single rank cannot show the exchange itself (that needs several GPUs, whose
collectives would wait on one another on one device), but it runs
`bit_nf4_quantized_11_b200.dp` inside an NCCL process group on the device:
the one-rank sharded quantizer (its all-gather is the identity at one rank)
must equal the single call bit for bit, and the adapter-gradient NCCL
all-reduce must leave one rank's gradients unchanged.  The process
group lives in a child process (bounded by a timeout) so that it does not
outlast the test.
"""

import os
import subprocess
import sys
import textwrap

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = textwrap.dedent("""
    import datetime, os, sys, torch
    sys.path.insert(0, os.environ["QLORA_TEST_ROOT"])
    import bit_nf4_quantized_11_b200 as q
    from bit_nf4_quantized_11_b200 import dp, synth
    torch.cuda.set_device(0)
    torch.distributed.init_process_group("nccl", init_method="tcp://127.0.0.1:" + os.environ["QLORA_TEST_PORT"],
                                         world_size=1, rank=0, timeout=datetime.timedelta(seconds=60))
    try:
        dev = torch.device("cuda", 0)
        W = synth.weight(384, 1024, 0.02, seed=5).to(dev)
        n_blocks = W.numel() // 64
        shard = dp.quantize_nf4_sharded(W.reshape(-1), n_blocks)
        codes, q8, step2, mean = dp.gather_nf4_replica(shard, n_blocks)
        ref = q.quantize_nf4(W)
        torch.cuda.synchronize()
        assert torch.equal(codes.cpu(), ref.codes.reshape(-1).cpu()), "codes"
        assert torch.equal(q8.cpu(), ref.q8.cpu()), "q8"
        assert torch.equal(step2.cpu(), ref.step2.cpu()), "step2"
        assert torch.equal(mean.cpu(), ref.mean.cpu()), "mean"
        flat, views = dp.layer_grad_buffers(16, [(1024, 384), (384, 1024)], dev)
        flat.copy_(torch.randn(flat.numel(), device=dev))
        before = flat.clone()
        dp.allreduce_adapter_grads(flat)
        torch.cuda.synchronize()
        assert torch.equal(flat, before), "one rank's all-reduce changed the gradients"
        print("nccl ok")
    finally:
        torch.distributed.destroy_process_group()
""")


def test_dp_helpers_over_nccl_one_rank(cuda_lib):
    env = dict(os.environ, QLORA_TEST_ROOT=ROOT, QLORA_TEST_PORT=str(29500 + os.getpid() % 1000),
               NCCL_NVLS_ENABLE="0")
    res = subprocess.run([sys.executable, "-c", CHILD], env=env, capture_output=True, text=True, timeout=300)
    assert res.returncode == 0, res.stdout[-2000:] + res.stderr[-2000:]
    assert "nccl ok" in res.stdout
