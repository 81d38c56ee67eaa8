"""CPU oracle for the QLoRA NF4 linear layer -- TEST INFRASTRUCTURE ONLY.

This package is a plain, slow, fp64 NumPy statement of what the GPU library
computes.  Only the test-suite, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import it.
The product path (the CUDA library and its Python binding) never imports,
links or executes anything in here, and this package never imports the
product package: the two share no code, no tables and no constants.

Sources (the pages that describe the method, cited by page title and section):

* "QLoRA" -- llm-compass (brenchcc.github.io/llm-compass/lora/qlora),
  section 方法与公式 (method and formula): the forward formula
  ``h = dequant(W0_NF4) x + (alpha/r) B A x``; NF4 as a quantile code with
  equal expected mass per bin, blocks of 64 weights with one scale each;
  double quantization of the block constants to 8 bit (0.5 -> ~0.13 bit/param).
* "QLoRA (Quantized Low-Rank Adaptation): 4-bit NormalFloat (NF4) & Paged
  Optimizers" -- learn-interview-questions, section 2 (NF4 vs. standard
  INT4): 16 bins with equal expected mass; section 1: double quantization
  saves 0.37 bit/param.
* "QLoRA" -- aigrafen.se, opening paragraph: gradients are back-propagated
  through the quantized base, only the adapters are updated.
* "QLoRA" -- auryth.ai glossary, section "Hoe het werkt" (architecture
  diagram): dequantize on the fly per layer; 8-bit quantization scales;
  LoRA A, B in 16-bit.

Where the pages leave a step open, the module docstrings state the reading
taken.  Every fp32 operation is evaluated in fp64 and rounded once to fp32;
for a single +, -, *, / this equals the correctly rounded fp32 result
(53 >= 2*24 + 2, Figueroa 1995), so the oracle reproduces fp32 semantics
exactly without relying on any fp32 hardware path.

Modules:
  nf4       codebook, thresholds, blockwise quantize, double quantization,
            dequantize, nibble packing
  linear    QLoRA linear forward / backward in fp64, with and without LoRA dropout
  overhead  storage arithmetic of the quantization constants
  merge     adapter merge into a bf16 copy of the dequantized base
  int4      the uniform INT4 absmax code the pages compare NF4 with
"""

from . import nf4, linear, overhead, merge, int4  # noqa: F401
