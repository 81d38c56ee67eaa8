"""QLoRA linear layer forward and backward in fp64 (oracle -- test
infrastructure only).

Shapes follow the PyTorch Linear convention: x [M, in], W0 [out, in],
A [r, in], B [out, r], h [M, out]; s = alpha / r.

Forward ("QLoRA", llm-compass, 方法与公式, the displayed formula):
    h = dequant(W0) x + (alpha/r) B A x
written for row-major token batches as
    h = x W^T + s (x A^T) B^T,            W = dequant(W0)

Backward: the base is frozen and only the adapters are trained, while the
gradient still flows through the quantized base to the layer input
("QLoRA", aigrafen.se, opening paragraph; llm-compass, 方法与公式, the
sentence after the formula).  With dh = dL/dh:
    dx = dh W + s (dh B) A
    dB = s dh^T (x A^T)
    dA = s (dh B)^T x
dequant(W0) is treated as a constant: there is no gradient for the codes.

Everything is computed in fp64 on the bf16 inputs' exact values and on the
oracle's own dequantized weight; no intermediate rounding is applied.
"""

from __future__ import annotations

import numpy as np


def _f64(a):
    return np.asarray(a, dtype=np.float64)


def linear_fwd(x, W, A, B, alpha: float):
    """h = x W^T + s (x A^T) B^T in fp64; also returns u = x A^T (pre-scale)."""
    x, W, A, B = _f64(x), _f64(W), _f64(A), _f64(B)
    r = A.shape[0]
    s = float(alpha) / float(r)
    u = x @ A.T                       # [M, r]
    h = x @ W.T + s * (u @ B.T)       # [M, out]
    return h, u


def linear_bwd(dh, x, W, A, B, alpha: float):
    """(dx, dA, dB) of L = sum(dh * h) for the forward above, in fp64."""
    dh, x, W, A, B = _f64(dh), _f64(x), _f64(W), _f64(A), _f64(B)
    r = A.shape[0]
    s = float(alpha) / float(r)
    g = dh @ B                        # [M, r]
    u = x @ A.T                       # [M, r]
    dx = dh @ W + s * (g @ A)         # [M, in]
    dB = s * (dh.T @ u)               # [out, r]
    dA = s * (g.T @ x)                # [r, in]
    return dx, dA, dB


def linear_fwd_rows(x, W, A, B, alpha: float, rows):
    """Forward restricted to the token rows ``rows`` (for sampled checks of
    full-size outputs); identical arithmetic to :func:`linear_fwd`."""
    rows = np.asarray(rows)
    h, _ = linear_fwd(_f64(x)[rows], W, A, B, alpha)
    return h


def linear_dx_rows(dh, W, A, B, alpha: float, rows):
    """dx restricted to the token rows ``rows``; same arithmetic as
    :func:`linear_bwd`."""
    dh, W, A, B = _f64(dh)[np.asarray(rows)], _f64(W), _f64(A), _f64(B)
    s = float(alpha) / float(A.shape[0])
    return dh @ W + s * ((dh @ B) @ A)


def lora_grads(dh, x, A, B, alpha: float):
    """(dA, dB) alone, with the same arithmetic as :func:`linear_bwd`."""
    dh, x, A, B = _f64(dh), _f64(x), _f64(A), _f64(B)
    s = float(alpha) / float(A.shape[0])
    g = dh @ B
    u = x @ A.T
    return s * (g.T @ x), s * (dh.T @ u)


# --------------------------------------------------------------------------
# LoRA dropout
# --------------------------------------------------------------------------
# The configurations on every page set lora_dropout = 0.05 ("QLoRA",
# aigrafen.se, the LoraConfig of the code example; llm-compass, 实现要点;
# skillbyai, Quantized base plus LoRA; learn-interview-questions, section 3).
# Reading D1 (the pages give no formula): dropout acts on the input of the
# LoRA branch only, with inverted scaling, and the keep mask is an input of
# the layer (the caller draws it), so that
#     h  = x W^T + s ((x * k) / (1 - p)) A^T B^T
# and the backward is the exact gradient of that expression for the same k:
#     dx = dh W + s ((dh B) A) * k / (1 - p)
#     dB = s dh^T (((x * k) / (1 - p)) A^T)
#     dA = s / (1 - p) (dh B)^T (x * k)
# with k in {0, 1} per element of x and 0 <= p < 1.  The mask is stored as
# bits: bit (i mod 8) of byte i // 8 of a row is the keep flag of column i.


def unpack_keep(keep_bits, cols: int) -> np.ndarray:
    """0/1 keep mask [M, cols] of bit-packed rows [M, cols/8] (bit i%8 of
    byte i//8, least significant bit first)."""
    kb = np.asarray(keep_bits, dtype=np.uint8)
    out = np.zeros((kb.shape[0], cols), dtype=np.float64)
    for i in range(cols):
        out[:, i] = (kb[:, i // 8] >> (i % 8)) & 1
    return out


def linear_fwd_dropout(x, W, A, B, alpha: float, keep, p: float):
    """h of reading D1 in fp64; also returns u = ((x * k) / (1 - p)) A^T."""
    x, W, A, B, keep = _f64(x), _f64(W), _f64(A), _f64(B), _f64(keep)
    s = float(alpha) / float(A.shape[0])
    xd = x * keep / (1.0 - p)
    u = xd @ A.T
    return x @ W.T + s * (u @ B.T), u


def linear_bwd_dropout(dh, x, W, A, B, alpha: float, keep, p: float):
    """(dx, dA, dB) of L = sum(dh * h) for the forward of reading D1."""
    dh, x, W, A, B, keep = _f64(dh), _f64(x), _f64(W), _f64(A), _f64(B), _f64(keep)
    s = float(alpha) / float(A.shape[0])
    g = dh @ B
    xd = x * keep / (1.0 - p)
    dx = dh @ W + s * (g @ A) * keep / (1.0 - p)
    dB = s * (dh.T @ (xd @ A.T))
    dA = s * (g.T @ xd)
    return dx, dA, dB
