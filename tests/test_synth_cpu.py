"""The seeded synthetic inputs: reproducible from their seed, one generator
per tensor, and with the stated distributions (so the workloads stand in for
the pages' normal-like Llama weights as described)."""

import math

import torch

from bit_nf4_quantized_11_b200 import synth


def test_same_seed_same_tensors_and_independent_streams():
    a = synth.problem(64, 256, 128, 8, seed=5)
    b = synth.problem(64, 256, 128, 8, seed=5)
    for k in a:
        assert torch.equal(a[k], b[k]), k
    c = synth.problem(64, 256, 128, 8, seed=6)
    assert not torch.equal(a["W"], c["W"])
    # x and dh come from different generators even with equal shapes
    p = synth.problem(32, 128, 128, 8, seed=0)
    assert not torch.equal(p["x"], p["dh"])


def test_distributions():
    W = synth.weight(512, 1024, 0.02, "normal", 1)
    assert abs(float(W.std()) - 0.02) < 0.02 * 0.01 and abs(float(W.mean())) < 1e-4
    T = synth.weight(512, 1024, 0.02, "student_t5", 2)
    assert abs(float(T.std()) - 0.02) < 0.02 * 0.05
    # heavier tails than the normal weight of the same deviation
    assert float((T.abs() > 4 * 0.02).float().mean()) > 2 * float((W.abs() > 4 * 0.02).float().mean())
    A = synth.lora_A(16, 4096, 3).float()
    bound = 1.0 / math.sqrt(4096)
    assert float(A.abs().max()) <= bound * (1 + 2 ** -8) and abs(float(A.std()) - bound / math.sqrt(3)) < 0.02 * bound
    B = synth.lora_B(4096, 16, seed=4).float()
    assert abs(float(B.std()) - 0.01) < 0.01 * 0.03
    x = synth.activations(256, 1024, 5).float()
    assert abs(float(x.std()) - 1.0) < 0.01
    assert synth.activations(4, 8).dtype == torch.bfloat16
