"""NF4 codebook, blockwise quantization, double quantization and dequantization
(fp64 NumPy oracle -- test infrastructure only).

What the pages fix
------------------
* NF4 is a 4-bit quantile code for zero-mean normal data: 16 levels placed at
  standard-normal quantiles so that every bin holds the same expected mass,
  normalised to [-1, 1].  ("QLoRA", llm-compass, 方法与公式 item 1;
  "QLoRA ... NF4 & Paged Optimizers", learn-interview-questions, section 2.)
* Quantization is blockwise: blocks of 64 weights, one absmax scale per block.
  (llm-compass, 方法与公式 item 1.)
* The fp32 block constants are themselves quantized to 8 bit ("double
  quantization"), taking their overhead from ~0.5 to ~0.13 bit/param.
  (llm-compass, 方法与公式 item 2; auryth glossary "Hoe het werkt" diagram,
  item 2: 8-bit scale per weight block.)

Readings where the pages are silent (each one is a stated choice)
------------------------------------------------------------------
R1 Codebook construction.  16 levels cannot be symmetric quantiles and also
   contain an exact zero, so the code is split 8 positive / 7 negative / one
   exact 0.  With ``delta = 1 - (1/32 + 1/30)/2`` the positive side takes the
   normal quantiles at ``p_i = delta - i*(delta-1/2)/8`` (i = 0..7), the negative
   side the mirrored quantiles at ``p_i = delta - i*(delta-1/2)/7`` (i = 0..6);
   all are divided by ``Phi^-1(delta)`` so that the extremes are exactly -1, +1,
   then rounded to fp32.  On each side the normal mass between consecutive
   levels is constant, which is the "equal mass per bin" property in the form
   that admits an exact zero.
R2 Nearest level, ties to the lower index; implemented as a comparison with the
   exact fp64 midpoints of consecutive fp32 levels.
R3 Normalisation ``v = fl32(w * fl32(1/c))`` (reciprocal then multiply) rather
   than a division; an all-zero block (c = 0) encodes every weight as the zero
   level (index 7).  When 1/c overflows fp32 (c below ~2.9e-39, a subnormal
   absmax), the reciprocal is unusable and ``v = fl32(w / c)`` (one correctly
   rounded division) is taken instead, so such a block still gets the nearest
   level of every weight and a zero weight the zero level.
R4 Packing: element 2i of a row goes to the low nibble of byte i, 2i+1 to the
   high nibble; blocks are 64 consecutive weights in row-major order.
R5 Double quantization: one fp32 mean per tensor (pairwise fp64 sum of all
   block scales, zero-padded to a power of two, divided by the block count,
   rounded to fp32); per group of 256 consecutive blocks a linear symmetric
   int8 code with ``step2 = fl32(max|c - mean| / 127)`` and round-half-even of
   ``fl32(d * fl32(1/step2))``, or of ``fl32(d / step2)`` when that reciprocal
   overflows (as in R3); a zero step gives code 0.  The first-level codes
   always use the exact block absmax.
R6 Dequantization: ``c_hat = fl32(fl32(q8 * step2) + mean)`` and
   ``w_hat = bf16_rne(fl32(level[code] * c_hat))``.
R7 16-bit input: weights loaded in bf16 (as a 16-bit checkpoint is loaded
   before quantization; "QLoRA: Fine-Tuning on One Consumer GPU", skillbyai,
   section "Merging the adapter for serving", which loads the base in
   bfloat16) are quantized by the same steps applied to the exact fp32 value
   of each bf16 number; bf16 -> fp32 widening is exact, so nothing else
   changes.
"""

from __future__ import annotations

import math
import statistics

import numpy as np

BLOCK = 64          # weights per first-level block (llm-compass, 方法与公式 item 1)
DQ_GROUP = 256      # first-level scales per second-level group
N_LEVELS = 16
ZERO_INDEX = 7      # index of the exact-zero level (7 negative levels below it)


# --------------------------------------------------------------------------
# rounding helpers (fp64 -> fp32 -> bf16), written out from their definitions
# --------------------------------------------------------------------------

def fl32(x):
    """Round fp64 value(s) to the nearest fp32 (ties to even), returned as fp64."""
    return np.asarray(x, dtype=np.float64).astype(np.float32).astype(np.float64)


def f32_bits(x) -> np.ndarray:
    """IEEE-754 binary32 bit patterns of fp32-representable value(s)."""
    return np.asarray(x, dtype=np.float64).astype(np.float32).view(np.uint32)


def bf16_bits_from_f32(x) -> np.ndarray:
    """bfloat16 bit patterns of fp32 value(s), round to nearest even.

    bf16 keeps the top 16 bits of the fp32 pattern; the dropped 16 bits are
    rounded to nearest with ties to even, which on the unsigned pattern is
    ``(u + 0x7FFF + lsb) >> 16`` with ``lsb`` the lowest kept bit.  Inputs are
    finite here, so NaN handling is not needed.
    """
    u = f32_bits(x).astype(np.uint64)
    lsb = (u >> np.uint64(16)) & np.uint64(1)
    return ((u + np.uint64(0x7FFF) + lsb) >> np.uint64(16)).astype(np.uint16)


def bf16_to_f64(bits) -> np.ndarray:
    """Value(s) of bfloat16 bit patterns as fp64."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return b.view(np.float32).astype(np.float64)


# --------------------------------------------------------------------------
# R1/R2 codebook and thresholds
# --------------------------------------------------------------------------

def codebook_delta() -> float:
    """Outermost quantile probability of reading R1: the mean of the
    bin-centre probabilities 1 - 1/(2n) for n = 16 and n = 15 bins."""
    return 1.0 - 0.5 * (1.0 / 32.0 + 1.0 / 30.0)


def codebook_f64() -> np.ndarray:
    """The 16 NF4 levels in fp64, ascending, before fp32 rounding (reading R1)."""
    nd = statistics.NormalDist()
    delta = codebook_delta()
    positive = [nd.inv_cdf(delta - i * (delta - 0.5) / 8.0) for i in range(8)]
    negative = [-nd.inv_cdf(delta - i * (delta - 0.5) / 7.0) for i in range(7)]
    norm = nd.inv_cdf(delta)
    levels = sorted(positive + negative + [0.0])
    return np.array([v / norm for v in levels], dtype=np.float64)


def codebook() -> np.ndarray:
    """The 16 NF4 levels rounded to fp32 (returned as fp64 values)."""
    return fl32(codebook_f64())


def midpoints() -> np.ndarray:
    """Exact midpoints of consecutive fp32 levels (exact in fp64)."""
    q = codebook()
    return (q[:-1] + q[1:]) / 2.0


def thresholds() -> np.ndarray:
    """The 15 decision thresholds: each exact midpoint rounded toward -inf to
    fp32, so that for every fp32 v, ``v > thr_j`` iff ``v > midpoint_j``."""
    mids = midpoints()
    out = np.empty_like(mids)
    for j, m in enumerate(mids):
        t = float(np.float32(m))
        if t > m:                       # rounded up: step one fp32 ulp down
            t = float(np.nextafter(np.float32(t), np.float32(-np.inf)))
        out[j] = t
    return out


# --------------------------------------------------------------------------
# R2-R4 first-level quantization
# --------------------------------------------------------------------------

def block_absmax(W: np.ndarray) -> np.ndarray:
    """Absmax of every 64-weight block, blocks in row-major order (exact)."""
    W = np.asarray(W, dtype=np.float64)
    rows, cols = W.shape
    assert cols % BLOCK == 0, "cols must be a multiple of the block size"
    return np.abs(W.reshape(rows * cols // BLOCK, BLOCK)).max(axis=1)


def nearest_level(v: np.ndarray) -> np.ndarray:
    """Index of the nearest fp32 level to each fp32 value v, ties to the lower
    index: the number of exact midpoints strictly below v (reading R2)."""
    return np.searchsorted(midpoints(), np.asarray(v, dtype=np.float64),
                           side="left").astype(np.uint8)


def normalise(blocks: np.ndarray, c: np.ndarray) -> np.ndarray:
    """Normalised values v of the weights of blocks with a nonzero absmax c
    (one row of ``blocks`` per block, reading R3): ``fl32(w * fl32(1/c))``,
    or ``fl32(w / c)`` for a block whose fp32 reciprocal overflows."""
    c = np.asarray(c, dtype=np.float64)
    with np.errstate(over="ignore"):
        recip = fl32(1.0 / c)                       # fl32(1 / c_b), inf for tiny c_b
    v = fl32(blocks * recip[:, None])               # fl32(w * r_b)
    over = ~np.isfinite(recip)
    if over.any():
        v[over] = fl32(blocks[over] / c[over, None])   # fl32(w / c_b)
    return v


def encode(W: np.ndarray, c: np.ndarray) -> np.ndarray:
    """4-bit code of every weight (unpacked, shape of W), given the exact block
    absmax c (reading R3)."""
    W = np.asarray(W, dtype=np.float64)
    rows, cols = W.shape
    blocks = W.reshape(-1, BLOCK)
    codes = np.full(blocks.shape, ZERO_INDEX, dtype=np.uint8)
    nz = c > 0
    codes[nz] = nearest_level(normalise(blocks[nz], c[nz]))
    return codes.reshape(rows, cols)


def pack(codes: np.ndarray) -> np.ndarray:
    """Two codes per byte, even element in the low nibble (reading R4)."""
    codes = np.asarray(codes, dtype=np.uint8)
    return (codes[:, 0::2] | (codes[:, 1::2] << 4)).astype(np.uint8)


def unpack(packed: np.ndarray) -> np.ndarray:
    """Inverse of :func:`pack`."""
    packed = np.asarray(packed, dtype=np.uint8)
    out = np.empty((packed.shape[0], packed.shape[1] * 2), dtype=np.uint8)
    out[:, 0::2] = packed & 0x0F
    out[:, 1::2] = packed >> 4
    return out


# --------------------------------------------------------------------------
# R5 double quantization of the block scales
# --------------------------------------------------------------------------

def pairwise_sum(values: np.ndarray) -> float:
    """fp64 sum in a fixed binary tree: zero-pad to a power of two, then add
    adjacent pairs level by level until one value is left."""
    a = np.asarray(values, dtype=np.float64).ravel()
    n = 1
    while n < a.size:
        n *= 2
    buf = np.zeros(n, dtype=np.float64)
    buf[:a.size] = a
    while buf.size > 1:
        buf = buf[0::2] + buf[1::2]
    return float(buf[0])


def scale_mean(c: np.ndarray) -> float:
    """mean = fl32(pairwise_sum(c) / n_blocks), the division in fp64."""
    return float(fl32(pairwise_sum(c) / float(len(c))))


def double_quantize(c: np.ndarray):
    """Second-level quantization of the block scales c (reading R5).

    Returns (q8 int8[n_blocks], step2 fp64[n_groups] (fp32 values), mean).
    """
    c = np.asarray(c, dtype=np.float64)
    mean = scale_mean(c)
    q8, step2 = second_level(c, mean)
    return q8, step2, mean


def second_level(c: np.ndarray, mean: float):
    """q8 and step2 of the block scales c against a given per-tensor mean
    (the part of reading R5 after the mean): per group of 256 blocks,
    d = fl32(c - mean), step2 = fl32(max|d| / 127),
    q8 = clip(rint(fl32(d * fl32(1/step2))), -127, 127), with fl32(d / step2)
    in place of the product when fl32(1/step2) overflows, and 0 where
    step2 = 0.  Returns (q8 int8[n], step2 fp64[n_groups])."""
    c = np.asarray(c, dtype=np.float64)
    n = c.size
    d = fl32(c - mean)                                   # fl32(c_b - mean)
    n_groups = (n + DQ_GROUP - 1) // DQ_GROUP
    q8 = np.zeros(n, dtype=np.int8)
    step2 = np.zeros(n_groups, dtype=np.float64)
    for g in range(n_groups):
        sl = slice(g * DQ_GROUP, min(n, (g + 1) * DQ_GROUP))
        S = float(np.abs(d[sl]).max())
        st = float(fl32(S / 127.0))
        step2[g] = st
        if st == 0.0:
            continue                                     # all codes 0
        with np.errstate(over="ignore"):
            inv = float(fl32(1.0 / st))                  # fl32(1 / step2)
        q = fl32(d[sl] * inv) if np.isfinite(inv) else fl32(d[sl] / st)
        q8[sl] = np.clip(np.rint(q), -127, 127).astype(np.int8)
    return q8, step2


# --------------------------------------------------------------------------
# full quantizer and dequantizer
# --------------------------------------------------------------------------

def quantize(W: np.ndarray) -> dict:
    """Quantize an fp32 weight [rows, cols] to NF4 with double quantization.

    Returns a dict with
      codes   uint8 [rows, cols]     unpacked 4-bit codes
      packed  uint8 [rows, cols/2]   two codes per byte (R4)
      absmax  fp64  [n_blocks]       exact first-level scales c_b
      q8      int8  [n_blocks]       second-level codes
      step2   fp64  [n_groups]       fp32 values of the per-group steps
      mean    float                  fp32 value of the per-tensor mean
    """
    W = np.asarray(W, dtype=np.float32).astype(np.float64)
    c = block_absmax(W)
    codes = encode(W, c)
    q8, step2, mean = double_quantize(c)
    return dict(codes=codes, packed=pack(codes), absmax=c, q8=q8,
                step2=step2, mean=mean)


def quantize_bf16(bits: np.ndarray) -> dict:
    """Quantize a weight given as bf16 bit patterns [rows, cols] (reading R7):
    :func:`quantize` of the exact values of the bf16 numbers."""
    return quantize(bf16_to_f64(bits))


def dequant_scales(q8: np.ndarray, step2: np.ndarray, mean: float) -> np.ndarray:
    """c_hat_b = fl32(fl32(q8_b * step2_g) + mean) for every block (R6)."""
    q8 = np.asarray(q8, dtype=np.float64)
    g = np.arange(q8.size) // DQ_GROUP
    return fl32(fl32(q8 * np.asarray(step2, dtype=np.float64)[g]) + mean)


def dequantize_bits(codes: np.ndarray, q8, step2, mean, blocks=None) -> np.ndarray:
    """bf16 bit patterns of the dequantized weight [rows, cols] (R6).

    ``blocks`` optionally gives the global block index of every 64-code block
    of ``codes`` (row-major), for dequantizing a subset of a tensor's rows."""
    codes = np.asarray(codes, dtype=np.uint8)
    rows, cols = codes.shape
    c_hat = dequant_scales(q8, step2, mean)
    if blocks is not None:
        c_hat = c_hat[np.asarray(blocks)]
    levels = codebook()
    lv = levels[codes.reshape(-1, BLOCK)]                 # level[code]
    prod = fl32(lv * c_hat[:, None])                      # fl32(level * c_hat)
    return bf16_bits_from_f32(prod).reshape(rows, cols)


def dequantize(codes: np.ndarray, q8, step2, mean, blocks=None) -> np.ndarray:
    """Dequantized weight [rows, cols] as fp64 values of bf16 numbers
    (``blocks`` as in :func:`dequantize_bits`)."""
    return bf16_to_f64(dequantize_bits(codes, q8, step2, mean, blocks))


def quantize_rows(W: np.ndarray, rows) -> dict:
    """First-level codes of the selected rows of W, with the second-level
    statistics (q8, step2, mean) of the WHOLE tensor, since the mean and the
    256-block groups span rows.  Identical to the corresponding rows of
    :func:`quantize`; used to check large tensors on sampled rows."""
    W = np.asarray(W, dtype=np.float32)
    rows = np.asarray(rows)
    c = block_absmax(W)
    q8, step2, mean = double_quantize(c)
    nbr = W.shape[1] // BLOCK
    blocks = (rows[:, None] * nbr + np.arange(nbr)[None, :]).ravel()
    codes = encode(W[rows].astype(np.float64), c[blocks])
    return dict(codes=codes, packed=pack(codes), absmax=c, q8=q8, step2=step2,
                mean=mean, blocks=blocks)
