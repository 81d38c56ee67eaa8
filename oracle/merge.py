"""Adapter merge into a 16-bit copy of the base (fp64 NumPy oracle -- test
infrastructure only).

What the pages fix
------------------
* After training the adapter can be kept separate or merged into the model
  for serving; merging needs the base dequantized first, and merging straight
  back into the 4-bit base is lossy (the merged weight carries quantization
  error), so the merge goes into a higher-precision copy of the base.
  ("QLoRA", llm-compass, sections 与 baseline 对比 (deployment row of the
  comparison table) and 调参与实践经验 (the note on merging); "QLoRA:
  Fine-Tuning on One Consumer GPU", skillbyai, sections "Quantized base plus
  LoRA" and "Merging the adapter for serving"; auryth glossary QLoRA,
  Veelgestelde vragen, the question on inference.)
* The layer being merged is ``h = dequant(W0) x + (alpha/r) B A x``
  (llm-compass, 方法与公式), so the merged weight is W0_hat + (alpha/r) B A.

Reading M1 (the pages give no arithmetic for the merge): the merged weight
is bf16, W0_hat is the bf16 dequantized base of reading R6, and per element

    acc = fp32 sum over j = 0 .. r-1, in that order, of B[o, j] * A[j, i]
          (each product of two bf16 numbers is exact in fp32),
    W'[o, i] = bf16_rne(fl32(W0_hat[o, i] + fl32(s * acc))),  s = fl32(alpha / r).

Reading M2: re-quantizing W' to NF4 (the lossy "merge back into 4 bit") is
the quantizer of reading R7 applied to W'.
"""

from __future__ import annotations

import numpy as np

from .nf4 import bf16_bits_from_f32, bf16_to_f64, fl32


def lora_product_f32(A_bits: np.ndarray, B_bits: np.ndarray) -> np.ndarray:
    """acc[o, i]: fp32 running sum over j in order of B[o, j] * A[j, i]
    (products exact in fp32, one rounding per addition)."""
    A = bf16_to_f64(A_bits)            # [r, in]
    B = bf16_to_f64(B_bits)            # [out, r]
    acc = np.zeros((B.shape[0], A.shape[1]), dtype=np.float64)
    for j in range(A.shape[0]):
        acc = fl32(acc + np.outer(B[:, j], A[j, :]))
    return acc


def merge_adapter_bits(w_hat_bits: np.ndarray, A_bits: np.ndarray, B_bits: np.ndarray,
                       alpha: float) -> np.ndarray:
    """bf16 bit patterns of W' = W0_hat + (alpha/r) B A (reading M1)."""
    r = np.asarray(A_bits).shape[0]
    s = float(fl32(float(np.float32(alpha)) / float(r)))
    acc = lora_product_f32(A_bits, B_bits)
    u = fl32(bf16_to_f64(w_hat_bits) + fl32(s * acc))
    return bf16_bits_from_f32(u)
