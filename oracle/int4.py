"""Uniform INT4 (absmax) comparison code (fp64 NumPy oracle -- test
infrastructure only).

What the pages fix
------------------
* Standard INT4 spreads its levels uniformly over the range, whereas NF4
  places them at normal quantiles; on normally distributed weights uniform
  levels waste resolution (the pages say in the tails) and NF4 gives a lower
  quantization error at the same bit width.  ("QLoRA", llm-compass, 方法与公式
  item 1; learn-interview-questions QLoRA page, section 2 "4-bit NormalFloat
  (NF4) vs. Standard INT4"; aigrafen.se, the BitsAndBytesConfig comment.)

Reading I1 (the pages give no INT4 construction): the symmetric uniform code
of the same blockwise absmax scheme -- levels fl32(k/7) for k = -7..7 at codes
0..14 (zero at code 7, as in NF4), code 15 a second copy of +1 so that all 16
codes stay valid -- with everything else (64-weight blocks, reciprocal
normalisation, nearest level with ties to the lower index through exact
midpoints, nibble packing, double quantization of the scales, dequantization)
exactly as for NF4 (readings R2-R6 of the nf4 module).
"""

from __future__ import annotations

import numpy as np

from .nf4 import (BLOCK, ZERO_INDEX, bf16_bits_from_f32, block_absmax, dequant_scales, double_quantize, fl32,
                  normalise, pack)


def levels() -> np.ndarray:
    """The 16 fp32 levels of reading I1 (fp64 values)."""
    lv = fl32(np.arange(-7, 8, dtype=np.float64) / 7.0)
    return np.concatenate([lv, [1.0]])


def midpoints() -> np.ndarray:
    """Exact fp64 midpoints of consecutive levels (the last one is 1.0)."""
    lv = levels()
    return (lv[:-1] + lv[1:]) / 2.0


def nearest_level(v: np.ndarray) -> np.ndarray:
    """Number of midpoints strictly below v: the nearest level, ties to the
    lower index."""
    return np.searchsorted(midpoints(), np.asarray(v, dtype=np.float64), side="left").astype(np.uint8)


def encode(W: np.ndarray, c: np.ndarray) -> np.ndarray:
    """4-bit INT4 code of every weight, reading I1 with the normalisation of R3."""
    W = np.asarray(W, dtype=np.float64)
    rows, cols = W.shape
    blocks = W.reshape(-1, BLOCK)
    codes = np.full(blocks.shape, ZERO_INDEX, dtype=np.uint8)
    nz = c > 0
    codes[nz] = nearest_level(normalise(blocks[nz], c[nz]))
    return codes.reshape(rows, cols)


def quantize(W: np.ndarray) -> dict:
    """INT4 blockwise quantization with the NF4 module's double quantization."""
    W = np.asarray(W, dtype=np.float32).astype(np.float64)
    c = block_absmax(W)
    codes = encode(W, c)
    q8, step2, mean = double_quantize(c)
    return dict(codes=codes, packed=pack(codes), absmax=c, q8=q8, step2=step2, mean=mean)


def dequantize_bits(codes: np.ndarray, q8, step2, mean) -> np.ndarray:
    """bf16 bit patterns of bf16_rne(fl32(level[code] * c_hat))."""
    codes = np.asarray(codes, dtype=np.uint8)
    rows, cols = codes.shape
    c_hat = dequant_scales(q8, step2, mean)
    prod = fl32(levels()[codes.reshape(-1, BLOCK)] * c_hat[:, None])
    return bf16_bits_from_f32(prod).reshape(rows, cols)
