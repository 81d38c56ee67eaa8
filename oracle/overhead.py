"""Storage arithmetic of NF4 with double quantization (oracle -- test
infrastructure only).

The pages state the overhead of the quantization constants: fp32 block
constants cost about 0.5 bit/param for small blocks, and quantizing them to
8 bit brings this to about 0.13 bit/param ("QLoRA", llm-compass, 方法与公式
item 2), a saving of 0.37 bit/param ("QLoRA ... NF4 & Paged Optimizers",
learn-interview-questions, section 1).  The functions below count the bits
of each stored array per weight for a given layout.
"""

from __future__ import annotations


def scale_bits_per_param(block: int = 64, scale_bits: int = 32) -> float:
    """Overhead of one fp32 absmax per block of ``block`` weights."""
    return scale_bits / block


def dq_bits_per_param(block: int = 64, group: int = 256, code_bits: int = 8,
                      step_bits: int = 32, mean_bits: int = 32,
                      n_params: int | None = None) -> float:
    """Overhead with double quantization: one ``code_bits`` code per block,
    one fp32 step per ``group`` blocks, and (when ``n_params`` is given) one
    fp32 mean per tensor."""
    bits = code_bits / block + step_bits / (block * group)
    if n_params:
        bits += mean_bits / n_params
    return bits


def bits_per_param(block: int = 64, group: int = 256, n_params: int | None = None) -> float:
    """Total storage per weight: the 4-bit code plus the double-quantized constants."""
    return 4.0 + dq_bits_per_param(block, group, n_params=n_params)


def stored_bytes(rows: int, cols: int, block: int = 64, group: int = 256) -> int:
    """Bytes of codes + int8 scale codes + fp32 steps + fp32 mean for one matrix."""
    n = rows * cols
    n_blocks = n // block
    n_groups = -(-n_blocks // group)
    return n // 2 + n_blocks + 4 * n_groups + 4
