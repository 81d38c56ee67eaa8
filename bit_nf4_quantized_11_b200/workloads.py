"""Workload shapes (no arithmetic): the linear layers the measurements use.

Each workload lists (name, in_features, out_features) projections with the
token count M, LoRA rank r, alpha and the frozen-weight distribution.
Shapes are those of Llama-style 7B / 65B / 70B models, the model sizes the
pages discuss (7B in ~6 GB, 65B on one 48 GB card).
"""

from __future__ import annotations

from dataclasses import dataclass, field


@dataclass(frozen=True)
class Workload:
    name: str
    projections: tuple          # ((label, in_features, out_features), ...)
    M: tuple                    # token counts (several for the GEMV regime)
    r: int
    alpha: float
    w_std: float
    w_dist: str = "normal"
    backward: bool = True
    notes: str = field(default="", compare=False)


SMALL_512 = Workload(
    name="single-linear-512x512-M64-r8",
    projections=(("linear", 512, 512),), M=(64,), r=8, alpha=16.0, w_std=0.02,
    notes="small parity case")

ATTN_7B = Workload(
    name="llama7b-attn-proj-4096x4096-M4096-r16",
    projections=(("q_proj", 4096, 4096),), M=(4096,), r=16, alpha=32.0, w_std=0.02,
    notes="batch 4 x seq 1024 tokens through one 4096x4096 projection")

MLP_7B = Workload(
    name="llama7b-mlp-4096x11008-M8192-r16-t5",
    projections=(("gate_proj", 4096, 11008), ("up_proj", 4096, 11008), ("down_proj", 11008, 4096)),
    M=(8192,), r=16, alpha=32.0, w_std=0.02, w_dist="student_t5",
    notes="heavy-tailed weights stress the absmax blocks")

GEMV_70B = Workload(
    name="llama70b-mlp-8192x28672-M1-4-16-r16-gemv",
    projections=(("up_proj", 8192, 28672), ("down_proj", 28672, 8192)), M=(1, 4, 16),
    r=16, alpha=32.0, w_std=0.015, backward=False,
    notes="few-token decode regime, forward only")

LAYER_65B = Workload(
    name="llama65b-decoder-layer-8192-22016-M2048-r64",
    projections=(("q_proj", 8192, 8192), ("k_proj", 8192, 8192), ("v_proj", 8192, 8192),
                 ("o_proj", 8192, 8192), ("gate_proj", 8192, 22016), ("up_proj", 8192, 22016),
                 ("down_proj", 22016, 8192)),
    M=(2048,), r=64, alpha=16.0, w_std=0.01,
    notes="all seven linears of one decoder layer, each with its own input")

ALL = (SMALL_512, ATTN_7B, MLP_7B, GEMV_70B, LAYER_65B)


def fwd_bwd_flops(M: int, in_f: int, out_f: int, r: int) -> float:
    """Algorithmic FLOPs of one forward + backward (no dW0; dequant not counted):
    forward 2*M*in*out + 2*M*r*(in+out); backward dx 2*M*in*out + 2*M*r*in,
    du 2*M*out*r, dB 2*M*out*r, dA 2*M*r*in."""
    return 4.0 * M * in_f * out_f + 6.0 * M * r * (in_f + out_f)


def quant_bytes(rows: int, cols: int) -> float:
    """Algorithmic HBM bytes of quantizing an fp32 [rows, cols] weight: read
    4 B/weight, write 0.5 B codes + 1/64 B scale codes + 4/16384 B steps."""
    n = rows * cols
    return 4.0 * n + n / 2 + n / 64 + 4.0 * (-(-(n // 64) // 256)) + 4


def gemv_weight_bytes(rows: int, cols: int) -> float:
    """Packed-weight bytes streamed by the few-token forward (codes + scale
    codes + steps + mean)."""
    n = rows * cols
    return n / 2 + n / 64 + 4.0 * (-(-(n // 64) // 256)) + 4
