"""Grouped projections: the grouped forward and backward issue the same
kernels as the single calls, with the rank-r products on a second stream, so
every output must equal the single calls' bit for bit (the single calls are
checked against the oracle in test_gpu_linear.py).  The mixes include
projections that stay on the single-call path inside a group (few tokens,
a rank that is not a multiple of 8), different token counts per projection
and the seven projections of the 65B decoder layer."""

import pytest
import torch

from bit_nf4_quantized_11_b200 import synth, workloads

pytestmark = pytest.mark.gpu


def _setup(q, specs, seed):
    dev = torch.device("cuda")
    out = []
    for i, (M, n_in, n_out, r) in enumerate(specs):
        p = synth.problem(M, n_in, n_out, r, seed=seed + i)
        c = {k: p[k].to(dev) for k in ("x", "A", "B", "dh")}
        c["w"] = q.quantize_nf4(p["W"].to(dev))
        out.append(c)
    return out


def _singles(q, cs, alpha):
    res = []
    for c in cs:
        h, us = q.linear_fwd(c["x"], c["w"], c["A"], c["B"], alpha)
        dx, dA, dB = q.linear_bwd(c["dh"], c["x"], us, c["w"], c["A"], c["B"], alpha)
        res.append((h, us, dx, dA, dB))
    return res


def _grouped(q, cs, alpha):
    probs = [q.LinearProblem(x=c["x"], w=c["w"], A=c["A"], B=c["B"], alpha=alpha, dh=c["dh"]) for c in cs]
    q.linear_fwd_group(probs)
    q.linear_bwd_group(probs)
    return [(p.h, p.us, p.dx, p.dA, p.dB) for p in probs]


def _check(q, specs, alpha=16.0, seed=0, stream=None):
    cs = _setup(q, specs, seed)
    ref = _singles(q, cs, alpha)
    if stream is None:
        got = _grouped(q, cs, alpha)
    else:
        stream.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(stream):
            got = _grouped(q, cs, alpha)
            # ordered after the grouped calls on the caller's stream, no host sync
            sums = [g[2].float().sum() for g in got]
        torch.cuda.current_stream().wait_stream(stream)
        for s_, g in zip(sums, got):
            assert torch.equal(s_, g[2].float().sum())
    torch.cuda.synchronize()
    assert q.last_device_status() == 0
    for i, (a, b) in enumerate(zip(ref, got)):
        for name, x, y in zip(("h", "us", "dx", "dA", "dB"), a, b):
            assert torch.equal(x, y), f"projection {i} {specs[i]}: {name} differs from the single call"


@pytest.mark.parametrize("specs", [
    [(300, 640, 320, 16), (1100, 512, 768, 64), (129, 256, 768, 32)],
    # few tokens (GEMV path) and r = 12 (padded rank) stay on the single-call path inside the group
    [(64, 512, 512, 8), (7, 512, 384, 8), (200, 256, 192, 12), (520, 1024, 1536, 24)],
    [(1024, 2048, 2048, 16)],
])
def test_group_equals_single_calls(cuda_lib, specs):
    _check(cuda_lib, specs, seed=len(specs))


def test_group_on_a_side_stream(cuda_lib):
    _check(cuda_lib, [(384, 512, 1024, 16), (640, 1024, 512, 32)], seed=7, stream=torch.cuda.Stream())


def test_group_65b_layer(cuda_lib):
    wl = workloads.LAYER_65B
    specs = [(wl.M[0], n_in, n_out, wl.r) for _, n_in, n_out in wl.projections]
    _check(cuda_lib, specs, alpha=wl.alpha, seed=1000)
