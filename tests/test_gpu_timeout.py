"""Bounded device waits: a kernel that waits on a pipeline barrier that
nothing completes gives up after the configured limit, sets the device
error flag and returns; the host reads QLORA_ERR_TIMEOUT, and the context
stays usable for the next call.  No trap, fault or hang is involved."""

import pytest
import torch

from bit_nf4_quantized_11_b200 import synth

pytestmark = pytest.mark.gpu


def test_wait_times_out_and_context_survives(cuda_lib):
    q = cuda_lib
    prev = q.set_wait_timeout_ns(2_000_000)          # 2 ms
    try:
        assert q.selftest_wait_timeout() == -5       # QLORA_ERR_TIMEOUT
        assert q.last_device_status() == 0           # flag was cleared
    finally:
        q.set_wait_timeout_ns(prev)
    W = synth.weight(128, 256, seed=1).cuda()
    w = q.quantize_nf4(W)
    d = q.dequantize_nf4(w)
    assert q.last_device_status() == 0
    assert torch.isfinite(d.float()).all()
