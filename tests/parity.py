"""Comparison helpers shared by the GPU parity tests (no method arithmetic)."""

import numpy as np

# Float tolerance for h, dx, dA, dB (the layer's outputs are bf16 or fp32
# computed from bf16-rounded intermediates): relative Frobenius error and
# max-abs error relative to the reference RMS.
REL_FRO = 2e-2
MAX_ABS_RMS = 5e-2


def to_np(t):
    import torch
    t = t.detach().cpu()
    if t.dtype == torch.bfloat16:
        return t.float().numpy().astype(np.float64)
    return t.numpy()


def bf16_bits(t):
    import torch
    return t.detach().cpu().view(torch.int16).numpy().view(np.uint16)


def f32_bits(t):
    return t.detach().cpu().numpy().view(np.uint32)


def assert_close(got, ref, name, rel_fro=REL_FRO, max_abs_rms=MAX_ABS_RMS):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (name, got.shape, ref.shape)
    assert np.all(np.isfinite(got)), f"{name}: non-finite values"
    diff = got - ref
    nref = np.linalg.norm(ref)
    rms = nref / np.sqrt(max(ref.size, 1))
    rel = np.linalg.norm(diff) / max(nref, 1e-300)
    mx = np.abs(diff).max() if diff.size else 0.0
    assert rel <= rel_fro, f"{name}: rel Frobenius error {rel:.3e} > {rel_fro}"
    assert mx <= max_abs_rms * rms, f"{name}: max abs error {mx:.3e} > {max_abs_rms} x RMS {rms:.3e}"
    return rel, mx / max(rms, 1e-300)
