"""QLoRA NF4 linear layer for NVIDIA B200 (sm_100a).

Thin Python binding over the C ABI of ``libqlora_nf4.so`` (declared in
``include/qlora_nf4.h``).  This module only marshals arguments: it checks
dtypes and devices, allocates the caller-owned outputs and workspaces with
PyTorch, and passes raw pointers plus the current CUDA stream to the library.
Every step of the computation runs in the library's CUDA kernels; there is no
fallback path.  If the shared library is missing, :func:`load` raises.

Entry points (same names as the C ABI, without the ``qlora_`` prefix):
  codebook()                      -> (levels[16], thresholds[15])
  quantize_nf4(W)                 -> NF4Weight
  dequantize_nf4(w)               -> bf16 [rows, cols]
  linear_fwd(x, w, A, B, alpha)   -> (h, us)
  linear_bwd(dh, x, us, w, A, B, alpha) -> (dx, dA, dB)
  linear_fwd_group(problems), linear_bwd_group(problems)   (n projections issued together)
  workspace_size(op, M, in_features, out_features, r)
  last_device_status(), set_wait_timeout_ns(ns), selftest_wait_timeout()
"""

from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import torch

__all__ = [
    "load", "library_path", "codebook", "NF4Weight", "quantize_nf4", "quantize_nf4_noalloc",
    "dequantize_nf4", "alloc_nf4",
    "linear_fwd", "linear_bwd", "workspace_size", "last_device_status",
    "LinearProblem", "linear_fwd_group", "linear_bwd_group", "linear_group_workspace_size",
    "set_wait_timeout_ns", "selftest_wait_timeout", "QLoRAError", "status_string",
    "timing_enable", "timing_reset", "timing_collect", "KERNEL_NAMES", "merge_adapter",
    "quantize_codebook", "dequantize_codebook", "CODEBOOK_NF4", "CODEBOOK_INT4",
    "linear_fwd_dropout", "linear_bwd_dropout", "pack_keep_mask", "OP_LINEAR_FWD_DROPOUT", "OP_LINEAR_BWD_DROPOUT",
    "OP_QUANTIZE", "OP_DEQUANTIZE", "OP_LINEAR_FWD", "OP_LINEAR_BWD",
    "quantize_shard_plan", "quantize_shard_workspace_size", "quantize_nf4_shard_local", "quantize_nf4_shard_finish",
]

OP_QUANTIZE, OP_DEQUANTIZE, OP_LINEAR_FWD, OP_LINEAR_BWD = 0, 1, 2, 3
STATUS = {0: "QLORA_OK", -1: "QLORA_ERR_INVALID_ARG", -2: "QLORA_ERR_UNSUPPORTED_SHAPE",
          -3: "QLORA_ERR_WORKSPACE", -4: "QLORA_ERR_CUDA", -5: "QLORA_ERR_TIMEOUT",
          -6: "QLORA_ERR_SCRATCH_LIMIT"}

_PKG_DIR = os.path.dirname(os.path.abspath(__file__))
_LIB = None


def library_path() -> str:
    return os.path.join(_PKG_DIR, "libqlora_nf4.so")


class QLoRAError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what}: {STATUS.get(status, status)} ({status_string(status)})")
        self.status = status


class _Weight(ctypes.Structure):
    _fields_ = [("codes", ctypes.c_void_p), ("q8", ctypes.c_void_p), ("step2", ctypes.c_void_p),
                ("mean", ctypes.c_void_p), ("rows", ctypes.c_int64), ("cols", ctypes.c_int64)]


class _Problem(ctypes.Structure):
    _fields_ = [("x", ctypes.c_void_p), ("w", ctypes.POINTER(_Weight)), ("A", ctypes.c_void_p),
                ("B", ctypes.c_void_p), ("M", ctypes.c_int64), ("r", ctypes.c_int), ("alpha", ctypes.c_float),
                ("h", ctypes.c_void_p), ("us", ctypes.c_void_p), ("dh", ctypes.c_void_p), ("dx", ctypes.c_void_p),
                ("dA", ctypes.c_void_p), ("dB", ctypes.c_void_p)]


def load():
    """Load libqlora_nf4.so (built in-tree); raises if it is missing."""
    global _LIB
    if _LIB is not None:
        return _LIB
    path = library_path()
    if not os.path.exists(path):
        raise RuntimeError(
            f"{path} is missing: build it with `python -m bit_nf4_quantized_11_b200.build` "
            "(there is no fallback implementation)")
    lib = ctypes.CDLL(path)
    P, I64, I, F, SZ = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
    W = ctypes.POINTER(_Weight)
    sig = {
        "qlora_nf4_codebook": (I, [ctypes.POINTER(ctypes.c_float), ctypes.POINTER(ctypes.c_float)]),
        "qlora_workspace_size": (SZ, [I, I64, I64, I64, I]),
        "qlora_quantize_nf4": (I, [P, I64, I64, P, P, P, P, P, SZ, P]),
        "qlora_dequantize_nf4": (I, [W, P, P]),
        "qlora_linear_fwd": (I, [P, I64, W, P, P, I, F, P, P, P, SZ, P]),
        "qlora_linear_bwd": (I, [P, P, P, I64, W, P, P, I, F, P, P, P, P, SZ, P]),
        "qlora_last_device_status": (I, [P]),
        "qlora_linear_group_workspace_size": (SZ, [I, I, ctypes.POINTER(_Problem)]),
        "qlora_linear_fwd_group": (I, [I, ctypes.POINTER(_Problem), P, SZ, P]),
        "qlora_linear_bwd_group": (I, [I, ctypes.POINTER(_Problem), P, SZ, P]),
        "qlora_set_wait_timeout_ns": (ctypes.c_uint64, [ctypes.c_uint64]),
        "qlora_selftest_wait_timeout": (I, [P]),
        "qlora_status_string": (ctypes.c_char_p, [I]),
        "qlora_quantize_nf4_noalloc": (I, [P, I64, I64, P, P, P, P, P]),
        "qlora_quantize_nf4_bf16": (I, [P, I64, I64, P, P, P, P, P, SZ, P]),
        "qlora_merge_adapter": (I, [W, P, P, I, F, P, P]),
        "qlora_codebook": (I, [I, ctypes.POINTER(ctypes.c_float), ctypes.POINTER(ctypes.c_float)]),
        "qlora_quantize_codebook": (I, [I, P, I64, I64, P, P, P, P, P, SZ, P]),
        "qlora_dequantize_codebook": (I, [I, W, P, P]),
        "qlora_linear_fwd_dropout": (I, [P, I64, W, P, P, I, F, P, F, P, P, P, SZ, P]),
        "qlora_linear_bwd_dropout": (I, [P, P, P, I64, W, P, P, I, F, P, F, P, P, P, P, SZ, P]),
        "qlora_quantize_shard_plan": (I, [I64, I, I, ctypes.POINTER(ctypes.c_int64), ctypes.POINTER(ctypes.c_int64),
                                          ctypes.POINTER(ctypes.c_int64)]),
        "qlora_quantize_shard_workspace_size": (SZ, [I64, I64]),
        "qlora_quantize_nf4_shard_local": (I, [P, I64, P, P, I64, P, SZ, P]),
        "qlora_quantize_nf4_shard_finish": (I, [P, I64, I64, I64, P, P, P, P, SZ, P]),
        "qlora_timing_enable": (I, [I]),
        "qlora_timing_reset": (None, []),
        "qlora_timing_collect": (I, [ctypes.c_char_p, ctypes.POINTER(ctypes.c_double),
                                     ctypes.POINTER(ctypes.c_int64)]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype, fn.argtypes = res, args
    _LIB = lib
    return lib


def status_string(status: int) -> str:
    return load().qlora_status_string(int(status)).decode()


def _check(status: int, what: str):
    if status != 0:
        raise QLoRAError(status, what)


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else ctypes.c_void_p(0)


def _need(t, dtype, name, shape=None):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")


@dataclass
class NF4Weight:
    """A quantized weight W0 [rows=out, cols=in] in the library's storage format."""
    codes: torch.Tensor   # uint8 [rows, cols/2]
    q8: torch.Tensor      # int8  [rows*cols/64]
    step2: torch.Tensor   # fp32  [ceil(n_blocks/256)]
    mean: torch.Tensor    # fp32  [1]
    rows: int
    cols: int

    def _c(self) -> _Weight:
        return _Weight(self.codes.data_ptr(), self.q8.data_ptr(), self.step2.data_ptr(),
                       self.mean.data_ptr(), self.rows, self.cols)

    def nbytes(self) -> int:
        return sum(t.numel() * t.element_size() for t in (self.codes, self.q8, self.step2, self.mean))


CODEBOOK_NF4, CODEBOOK_INT4 = 0, 1


def codebook(kind: int = CODEBOOK_NF4):
    """The 16 levels and 15 thresholds of a codebook computed by the library
    (host): NF4 (default) or the uniform INT4 comparison code."""
    lib = load()
    lv = (ctypes.c_float * 16)()
    th = (ctypes.c_float * 15)()
    if kind == CODEBOOK_NF4:
        _check(lib.qlora_nf4_codebook(lv, th), "qlora_nf4_codebook")
    else:
        _check(lib.qlora_codebook(int(kind), lv, th), "qlora_codebook")
    return list(lv), list(th)


def quantize_codebook(W: torch.Tensor, kind: int, out: NF4Weight | None = None, workspace=None) -> NF4Weight:
    """Blockwise 4-bit quantization of an fp32 weight with the levels of
    codebook `kind` (CODEBOOK_NF4 or CODEBOOK_INT4), double-quantized scales."""
    _need(W, torch.float32, "W")
    rows, cols = W.shape
    w = out if out is not None else alloc_nf4(rows, cols, W.device)
    ws = _workspace(workspace_size(OP_QUANTIZE, 0, cols, rows, 0), W.device, workspace)
    _check(load().qlora_quantize_codebook(int(kind), _ptr(W), rows, cols, _ptr(w.codes), _ptr(w.q8), _ptr(w.step2),
                                          _ptr(w.mean), _ptr(ws), ws.numel() if ws is not None else 0, _stream()),
           "qlora_quantize_codebook")
    return w


def dequantize_codebook(w: NF4Weight, kind: int, out: torch.Tensor | None = None) -> torch.Tensor:
    """bf16 [rows, cols] of a weight quantized with codebook `kind`."""
    o = out if out is not None else torch.empty((w.rows, w.cols), dtype=torch.bfloat16, device=w.codes.device)
    _need(o, torch.bfloat16, "out", (w.rows, w.cols))
    cw = w._c()
    _check(load().qlora_dequantize_codebook(int(kind), ctypes.byref(cw), _ptr(o), _stream()),
           "qlora_dequantize_codebook")
    return o


def workspace_size(op: int, M: int, in_features: int, out_features: int, r: int) -> int:
    n = load().qlora_workspace_size(int(op), int(M), int(in_features), int(out_features), int(r))
    if n == ctypes.c_size_t(-1).value:
        raise ValueError("invalid workspace query")
    return int(n)


def _workspace(nbytes: int, device, ws=None):
    if nbytes == 0:
        return None
    if ws is not None and ws.numel() >= nbytes:
        return ws
    return torch.empty(nbytes, dtype=torch.uint8, device=device)


def alloc_nf4(rows: int, cols: int, device) -> NF4Weight:
    n_blocks = rows * cols // 64
    n_groups = -(-n_blocks // 256)
    return NF4Weight(
        codes=torch.empty((rows, cols // 2), dtype=torch.uint8, device=device),
        q8=torch.empty(n_blocks, dtype=torch.int8, device=device),
        step2=torch.empty(n_groups, dtype=torch.float32, device=device),
        mean=torch.empty(1, dtype=torch.float32, device=device),
        rows=rows, cols=cols)


def quantize_nf4(W: torch.Tensor, out: NF4Weight | None = None, workspace=None) -> NF4Weight:
    """NF4 + double quantization of an fp32 or bf16 weight [rows, cols]
    (cols % 64 == 0); a bf16 weight is quantized as its exact fp32 values."""
    if not (isinstance(W, torch.Tensor) and W.dtype == torch.bfloat16):
        _need(W, torch.float32, "W")
    else:
        _need(W, torch.bfloat16, "W")
    rows, cols = W.shape
    w = out if out is not None else alloc_nf4(rows, cols, W.device)
    ws = _workspace(workspace_size(OP_QUANTIZE, 0, cols, rows, 0), W.device, workspace)
    fn, name = ((load().qlora_quantize_nf4_bf16, "qlora_quantize_nf4_bf16") if W.dtype == torch.bfloat16
                else (load().qlora_quantize_nf4, "qlora_quantize_nf4"))
    _check(fn(_ptr(W), rows, cols, _ptr(w.codes), _ptr(w.q8), _ptr(w.step2), _ptr(w.mean), _ptr(ws),
              ws.numel() if ws is not None else 0, _stream()), name)
    return w


def quantize_shard_plan(n_blocks_total: int, world: int, rank: int) -> tuple[int, int, int]:
    """(block_begin, block_end, roots_per_rank) of `rank`'s slice of a weight
    of n_blocks_total 64-weight blocks split over `world` ranks."""
    b0, b1, cpr = ctypes.c_int64(0), ctypes.c_int64(0), ctypes.c_int64(0)
    _check(load().qlora_quantize_shard_plan(int(n_blocks_total), int(world), int(rank), ctypes.byref(b0),
                                            ctypes.byref(b1), ctypes.byref(cpr)), "qlora_quantize_shard_plan")
    return b0.value, b1.value, cpr.value


def quantize_shard_workspace_size(n_blocks_shard: int, n_roots_total: int) -> int:
    n = load().qlora_quantize_shard_workspace_size(int(n_blocks_shard), int(n_roots_total))
    if n == ctypes.c_size_t(-1).value:
        raise QLoRAError(-1, "qlora_quantize_shard_workspace_size")
    return int(n)


def quantize_nf4_shard_local(W_shard: torch.Tensor, roots_per_rank: int, n_roots_total: int):
    """First half of a sharded quantization: (codes uint8 [n_blocks_shard*32],
    roots fp64 [roots_per_rank], workspace) for a shard given as fp32 weights
    (any shape, numel % 64 == 0).  Keep the workspace for the finishing call."""
    _need(W_shard, torch.float32, "W_shard")
    if W_shard.numel() % 64:
        raise ValueError("a shard holds whole 64-weight blocks")
    nb = W_shard.numel() // 64
    dev = W_shard.device
    codes = torch.empty(nb * 32, dtype=torch.uint8, device=dev)
    roots = torch.empty(roots_per_rank, dtype=torch.float64, device=dev)
    ws = torch.empty(quantize_shard_workspace_size(nb, n_roots_total), dtype=torch.uint8, device=dev)
    _check(load().qlora_quantize_nf4_shard_local(_ptr(W_shard) if nb else None, nb, _ptr(codes) if nb else None,
                                                 _ptr(roots), int(roots_per_rank), _ptr(ws), ws.numel(), _stream()),
           "qlora_quantize_nf4_shard_local")
    return codes, roots, ws


def quantize_nf4_shard_finish(roots_all: torch.Tensor, n_blocks_total: int, n_blocks_shard: int,
                              workspace: torch.Tensor):
    """Second half: (q8 int8 [n_blocks_shard], step2 fp32 [ceil(n_blocks_shard/256)],
    mean fp32 [1]) from the all-gathered roots (fp64, rank order)."""
    _need(roots_all, torch.float64, "roots_all")
    dev = roots_all.device
    q8 = torch.empty(n_blocks_shard, dtype=torch.int8, device=dev)
    step2 = torch.empty((n_blocks_shard + 255) // 256, dtype=torch.float32, device=dev)
    mean = torch.empty(1, dtype=torch.float32, device=dev)
    _check(load().qlora_quantize_nf4_shard_finish(_ptr(roots_all), roots_all.numel(), int(n_blocks_total),
                                                  int(n_blocks_shard), _ptr(q8), _ptr(step2), _ptr(mean),
                                                  _ptr(workspace), workspace.numel(), _stream()),
           "qlora_quantize_nf4_shard_finish")
    return q8, step2, mean


def merge_adapter(w: NF4Weight, A: torch.Tensor, B: torch.Tensor, alpha: float,
                  out: torch.Tensor | None = None) -> torch.Tensor:
    """bf16 [out, in] = dequant(W0) + (alpha/r) B A, the adapter merged into a
    bf16 copy of the base (A bf16 [r, in], B bf16 [out, r])."""
    r = A.shape[0]
    _need(A, torch.bfloat16, "A", (r, w.cols))
    _need(B, torch.bfloat16, "B", (w.rows, r))
    o = out if out is not None else torch.empty((w.rows, w.cols), dtype=torch.bfloat16, device=A.device)
    _need(o, torch.bfloat16, "out", (w.rows, w.cols))
    cw = w._c()
    _check(load().qlora_merge_adapter(ctypes.byref(cw), _ptr(A), _ptr(B), r, float(alpha), _ptr(o), _stream()),
           "qlora_merge_adapter")
    return o


def quantize_nf4_noalloc(W: torch.Tensor, out: NF4Weight | None = None) -> NF4Weight:
    """As quantize_nf4, but the library uses its own fixed device scratch
    (at most 2**22 blocks of 64 weights) instead of a caller workspace."""
    _need(W, torch.float32, "W")
    rows, cols = W.shape
    w = out if out is not None else alloc_nf4(rows, cols, W.device)
    _check(load().qlora_quantize_nf4_noalloc(_ptr(W), rows, cols, _ptr(w.codes), _ptr(w.q8),
                                             _ptr(w.step2), _ptr(w.mean), _stream()),
           "qlora_quantize_nf4_noalloc")
    return w


def dequantize_nf4(w: NF4Weight, out: torch.Tensor | None = None) -> torch.Tensor:
    """bf16 [rows, cols] dequantized weight."""
    o = out if out is not None else torch.empty((w.rows, w.cols), dtype=torch.bfloat16, device=w.codes.device)
    _need(o, torch.bfloat16, "out", (w.rows, w.cols))
    cw = w._c()
    _check(load().qlora_dequantize_nf4(ctypes.byref(cw), _ptr(o), _stream()), "qlora_dequantize_nf4")
    return o


def linear_fwd(x, w: NF4Weight, A, B, alpha: float, h=None, us=None, workspace=None):
    """h = x dequant(W0)^T + us B^T with us = bf16((alpha/r) x A^T); returns (h, us)."""
    M = x.shape[0]
    r = A.shape[0]
    _need(x, torch.bfloat16, "x", (M, w.cols))
    _need(A, torch.bfloat16, "A", (r, w.cols))
    _need(B, torch.bfloat16, "B", (w.rows, r))
    h = h if h is not None else torch.empty((M, w.rows), dtype=torch.bfloat16, device=x.device)
    us = us if us is not None else torch.empty((M, r), dtype=torch.bfloat16, device=x.device)
    _need(h, torch.bfloat16, "h", (M, w.rows))
    _need(us, torch.bfloat16, "us", (M, r))
    ws = _workspace(workspace_size(OP_LINEAR_FWD, M, w.cols, w.rows, r), x.device, workspace)
    cw = w._c()
    _check(load().qlora_linear_fwd(_ptr(x), M, ctypes.byref(cw), _ptr(A), _ptr(B), r, float(alpha),
                                   _ptr(h), _ptr(us), _ptr(ws), ws.numel() if ws is not None else 0,
                                   _stream()), "qlora_linear_fwd")
    return h, us


def linear_bwd(dh, x, us, w: NF4Weight, A, B, alpha: float, dx=None, dA=None, dB=None, workspace=None):
    """Backward with W0 frozen; returns (dx bf16 [M, in], dA fp32 [r, in], dB fp32 [out, r])."""
    M = x.shape[0]
    r = A.shape[0]
    _need(dh, torch.bfloat16, "dh", (M, w.rows))
    _need(x, torch.bfloat16, "x", (M, w.cols))
    _need(us, torch.bfloat16, "us", (M, r))
    _need(A, torch.bfloat16, "A", (r, w.cols))
    _need(B, torch.bfloat16, "B", (w.rows, r))
    dev = x.device
    dx = dx if dx is not None else torch.empty((M, w.cols), dtype=torch.bfloat16, device=dev)
    dA = dA if dA is not None else torch.empty((r, w.cols), dtype=torch.float32, device=dev)
    dB = dB if dB is not None else torch.empty((w.rows, r), dtype=torch.float32, device=dev)
    ws = _workspace(workspace_size(OP_LINEAR_BWD, M, w.cols, w.rows, r), dev, workspace)
    cw = w._c()
    _check(load().qlora_linear_bwd(_ptr(dh), _ptr(x), _ptr(us), M, ctypes.byref(cw), _ptr(A), _ptr(B), r,
                                   float(alpha), _ptr(dx), _ptr(dA), _ptr(dB), _ptr(ws),
                                   ws.numel() if ws is not None else 0, _stream()), "qlora_linear_bwd")
    return dx, dA, dB


@dataclass
class LinearProblem:
    """One projection of a grouped call: inputs x, w, A, B, alpha; forward
    outputs h, us; backward input dh and outputs dx, dA, dB (allocated by the
    grouped calls when None)."""
    x: torch.Tensor
    w: "NF4Weight"
    A: torch.Tensor
    B: torch.Tensor
    alpha: float
    h: torch.Tensor | None = None
    us: torch.Tensor | None = None
    dh: torch.Tensor | None = None
    dx: torch.Tensor | None = None
    dA: torch.Tensor | None = None
    dB: torch.Tensor | None = None


def _group_array(problems, backward: bool):
    arr = (_Problem * len(problems))()
    keep = []                                      # ctypes weight structs must outlive the call
    for i, p in enumerate(problems):
        M, r, w = p.x.shape[0], p.A.shape[0], p.w
        _need(p.x, torch.bfloat16, "x", (M, w.cols))
        _need(p.A, torch.bfloat16, "A", (r, w.cols))
        _need(p.B, torch.bfloat16, "B", (w.rows, r))
        dev = p.x.device
        if not backward:
            p.h = p.h if p.h is not None else torch.empty((M, w.rows), dtype=torch.bfloat16, device=dev)
            p.us = p.us if p.us is not None else torch.empty((M, r), dtype=torch.bfloat16, device=dev)
            _need(p.h, torch.bfloat16, "h", (M, w.rows))
        else:
            _need(p.dh, torch.bfloat16, "dh", (M, w.rows))
            p.dx = p.dx if p.dx is not None else torch.empty((M, w.cols), dtype=torch.bfloat16, device=dev)
            p.dA = p.dA if p.dA is not None else torch.empty((r, w.cols), dtype=torch.float32, device=dev)
            p.dB = p.dB if p.dB is not None else torch.empty((w.rows, r), dtype=torch.float32, device=dev)
            _need(p.dx, torch.bfloat16, "dx", (M, w.cols))
            _need(p.dA, torch.float32, "dA", (r, w.cols))
            _need(p.dB, torch.float32, "dB", (w.rows, r))
        _need(p.us, torch.bfloat16, "us", (M, r))
        cw = w._c()
        keep.append(cw)
        arr[i] = _Problem(_ptr(p.x).value, ctypes.pointer(cw), _ptr(p.A).value, _ptr(p.B).value, M, r,
                          float(p.alpha), _ptr(p.h).value, _ptr(p.us).value, _ptr(p.dh).value, _ptr(p.dx).value,
                          _ptr(p.dA).value, _ptr(p.dB).value)
    return arr, keep


def linear_group_workspace_size(backward: bool, problems) -> int:
    arr, _keep = _group_array(problems, backward)
    n = load().qlora_linear_group_workspace_size(int(bool(backward)), len(problems), arr)
    if n == ctypes.c_size_t(-1).value:
        raise ValueError("invalid grouped workspace query")
    return n


def linear_fwd_group(problems, workspace=None):
    """Forward of independent projections (LinearProblem list), the same
    results as linear_fwd on each; rank-r products overlap the GEMMs.  Fills
    and returns the problems' h and us."""
    if not problems:
        return problems
    arr, _keep = _group_array(problems, False)
    n = load().qlora_linear_group_workspace_size(0, len(problems), arr)
    ws = _workspace(n, problems[0].x.device, workspace)
    _check(load().qlora_linear_fwd_group(len(problems), arr, _ptr(ws), ws.numel() if ws is not None else 0,
                                         _stream()), "qlora_linear_fwd_group")
    return problems


def linear_bwd_group(problems, workspace=None):
    """Backward of independent projections, the same results as linear_bwd on
    each; fills and returns the problems' dx, dA and dB."""
    if not problems:
        return problems
    arr, _keep = _group_array(problems, True)
    n = load().qlora_linear_group_workspace_size(1, len(problems), arr)
    ws = _workspace(n, problems[0].x.device, workspace)
    _check(load().qlora_linear_bwd_group(len(problems), arr, _ptr(ws), ws.numel() if ws is not None else 0,
                                         _stream()), "qlora_linear_bwd_group")
    return problems


OP_LINEAR_FWD_DROPOUT, OP_LINEAR_BWD_DROPOUT = 4, 5


def pack_keep_mask(keep: torch.Tensor) -> torch.Tensor:
    """bool [M, n] keep mask -> the uint8 [M, n/8] bit layout of the dropout
    calls (bit i % 8 of byte i // 8 keeps column i)."""
    M, n = keep.shape
    w = (1 << torch.arange(8, device=keep.device, dtype=torch.int32))
    return (keep.reshape(M, n // 8, 8).to(torch.int32) * w).sum(-1).to(torch.uint8).contiguous()


def linear_fwd_dropout(x, w: NF4Weight, A, B, alpha: float, keep_bits, p: float, h=None, us=None, workspace=None):
    """Forward with LoRA dropout on the adapter input: h = x W0^T + us B^T,
    us = bf16((alpha/r)/(1-p) (x * k) A^T); keep_bits uint8 [M, in/8]."""
    M = x.shape[0]
    r = A.shape[0]
    _need(x, torch.bfloat16, "x", (M, w.cols))
    _need(A, torch.bfloat16, "A", (r, w.cols))
    _need(B, torch.bfloat16, "B", (w.rows, r))
    _need(keep_bits, torch.uint8, "keep_bits", (M, w.cols // 8))
    h = h if h is not None else torch.empty((M, w.rows), dtype=torch.bfloat16, device=x.device)
    us = us if us is not None else torch.empty((M, r), dtype=torch.bfloat16, device=x.device)
    _need(h, torch.bfloat16, "h", (M, w.rows))
    _need(us, torch.bfloat16, "us", (M, r))
    ws = _workspace(workspace_size(OP_LINEAR_FWD_DROPOUT, M, w.cols, w.rows, r), x.device, workspace)
    cw = w._c()
    _check(load().qlora_linear_fwd_dropout(_ptr(x), M, ctypes.byref(cw), _ptr(A), _ptr(B), r, float(alpha),
                                           _ptr(keep_bits), float(p), _ptr(h), _ptr(us), _ptr(ws),
                                           ws.numel() if ws is not None else 0, _stream()),
           "qlora_linear_fwd_dropout")
    return h, us


def linear_bwd_dropout(dh, x, us, w: NF4Weight, A, B, alpha: float, keep_bits, p: float, dx=None, dA=None, dB=None,
                       workspace=None):
    """Backward of :func:`linear_fwd_dropout` (same keep_bits and p)."""
    M = x.shape[0]
    r = A.shape[0]
    _need(dh, torch.bfloat16, "dh", (M, w.rows))
    _need(x, torch.bfloat16, "x", (M, w.cols))
    _need(us, torch.bfloat16, "us", (M, r))
    _need(A, torch.bfloat16, "A", (r, w.cols))
    _need(B, torch.bfloat16, "B", (w.rows, r))
    _need(keep_bits, torch.uint8, "keep_bits", (M, w.cols // 8))
    dev = x.device
    dx = dx if dx is not None else torch.empty((M, w.cols), dtype=torch.bfloat16, device=dev)
    dA = dA if dA is not None else torch.empty((r, w.cols), dtype=torch.float32, device=dev)
    dB = dB if dB is not None else torch.empty((w.rows, r), dtype=torch.float32, device=dev)
    ws = _workspace(workspace_size(OP_LINEAR_BWD_DROPOUT, M, w.cols, w.rows, r), dev, workspace)
    cw = w._c()
    _check(load().qlora_linear_bwd_dropout(_ptr(dh), _ptr(x), _ptr(us), M, ctypes.byref(cw), _ptr(A), _ptr(B), r,
                                           float(alpha), _ptr(keep_bits), float(p), _ptr(dx), _ptr(dA), _ptr(dB),
                                           _ptr(ws), ws.numel() if ws is not None else 0, _stream()),
           "qlora_linear_bwd_dropout")
    return dx, dA, dB


def last_device_status() -> int:
    """Synchronize the current stream, read and clear the device error flag."""
    return int(load().qlora_last_device_status(_stream()))


def set_wait_timeout_ns(ns: int) -> int:
    return int(load().qlora_set_wait_timeout_ns(int(ns)))


def selftest_wait_timeout() -> int:
    return int(load().qlora_selftest_wait_timeout(_stream()))


KERNEL_NAMES = ("quantize_blocks", "scale_mean_tree", "dq_scales", "dequantize", "gemm_fwd", "gemm_dx",
                "gemv", "gemv_finalize", "lora_rowwise", "lora_rowwise_du", "lora_colwise",
                "merge_adapter", "dropout_dx", "lora_fewtok", "lora_pad")


def timing_enable(on: bool = True) -> bool:
    """Bracket every library kernel launch with CUDA events on its stream."""
    return bool(load().qlora_timing_enable(1 if on else 0))


def timing_reset() -> None:
    load().qlora_timing_reset()


def timing_collect(kernel: str):
    """(total device ms, launches) of one kernel since the last reset."""
    ms = ctypes.c_double(0.0)
    n = ctypes.c_int64(0)
    _check(load().qlora_timing_collect(kernel.encode(), ctypes.byref(ms), ctypes.byref(n)),
           "qlora_timing_collect")
    return ms.value, n.value

