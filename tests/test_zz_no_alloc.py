"""The no-allocation quantizer entry point, qlora_quantize_nf4_noalloc.

It serves callers that cannot obtain device memory at the moment they
quantize (a host that forbids cudaMalloc after start-up, or a plugin without
access to its host framework's allocator): its scratch is a fixed device
array inside the library instead of a caller workspace.  Its results must be
bit-identical to qlora_quantize_nf4, including on a second call in a row that
finds the previous call's data still in the shared scratch.
"""

import ctypes

import numpy as np
import pytest
import torch

import bit_nf4_quantized_11_b200 as q
from bit_nf4_quantized_11_b200 import synth
from oracle import nf4

pytestmark = pytest.mark.gpu

ERR_SCRATCH_LIMIT = -6
MAX_BLOCKS = 1 << 22


def _noalloc_fn():
    f = q.load().qlora_quantize_nf4_noalloc
    P, I64 = ctypes.c_void_p, ctypes.c_int64
    f.restype = ctypes.c_int
    f.argtypes = [P, I64, I64, P, P, P, P, P]
    return f


def _bits(t):
    return t.detach().cpu().numpy().view(np.uint8)


def test_noalloc_quantizer_matches_workspace_quantizer(cuda_lib):
    f = _noalloc_fn()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    # two calls in a row: a larger tensor, then a smaller one that finds the
    # first call's values left in the shared scratch
    for i, (rows, cols) in enumerate([(1024, 4096), (300, 640)]):
        W = synth.weight(rows, cols, 0.02, seed=40 + i).cuda()
        ref = q.quantize_nf4(W)
        out = q.alloc_nf4(rows, cols, W.device)
        for t in (out.codes, out.q8, out.step2, out.mean):
            t.fill_(0x5A if t.dtype in (torch.uint8, torch.int8) else 7.0)
        st = f(W.data_ptr(), rows, cols, out.codes.data_ptr(), out.q8.data_ptr(),
               out.step2.data_ptr(), out.mean.data_ptr(), stream)
        assert st == 0, q.status_string(st)
        torch.cuda.synchronize()
        assert q.last_device_status() == 0
        for a, b in ((out.codes, ref.codes), (out.q8, ref.q8), (out.step2, ref.step2), (out.mean, ref.mean)):
            assert np.array_equal(_bits(a), _bits(b))
        if i == 1:
            # the second call also against the CPU oracle directly
            o = nf4.quantize(W.cpu().numpy())
            assert np.array_equal(out.codes.cpu().numpy(), o["packed"])
            assert np.array_equal(out.q8.cpu().numpy(), o["q8"])
            assert np.array_equal(_bits(out.step2), nf4.f32_bits(o["step2"]).view(np.uint8))
            assert np.array_equal(_bits(out.mean), nf4.f32_bits([o["mean"]]).view(np.uint8))


def test_noalloc_quantizer_rejects_sizes_beyond_its_scratch(cuda_lib):
    f = _noalloc_fn()
    W = torch.zeros(64, 64, dtype=torch.float32, device="cuda")
    out = q.alloc_nf4(64, 64, W.device)
    rows, cols = 4097, 65536                     # 4097 * 1024 blocks > 2**22
    assert rows * cols // 64 > MAX_BLOCKS
    st = f(W.data_ptr(), rows, cols, out.codes.data_ptr(), out.q8.data_ptr(),
           out.step2.data_ptr(), out.mean.data_ptr(), None)
    assert st == ERR_SCRATCH_LIMIT
    assert "scratch" in q.status_string(st)
