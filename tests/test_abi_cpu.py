"""C-ABI checks that need no GPU: the shared library loads, exports every
function declared in include/qlora_nf4.h, computes the same NF4 codebook as
the oracle bit for bit (a host-only call), sizes workspaces consistently, and
rejects bad arguments with the documented status before launching anything.

Only calls that return before any CUDA work are made here; the pointers
passed are aligned dummies that are never dereferenced.
"""

import ctypes
import os
import re

import numpy as np
import pytest

import bit_nf4_quantized_11_b200 as q
from oracle import int4, nf4

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "qlora_nf4.h")

OK, EINVAL, ESHAPE, EWS, ECUDA, ETIMEOUT = 0, -1, -2, -3, -4, -5
FAKE = 1 << 20          # 16- and 256-byte aligned, never dereferenced


@pytest.fixture(scope="module")
def lib():
    from bit_nf4_quantized_11_b200 import build
    build.build()
    return q.load()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(qlora_[a-z0-9_]+)\s*\(", text)))


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert len(names) >= 10
    for n in names:
        assert hasattr(lib, n), n


def test_library_codebook_equals_oracle_bit_for_bit(lib):
    lv, th = q.codebook()
    assert np.array_equal(np.array(lv, dtype=np.float32).view(np.uint32), nf4.f32_bits(nf4.codebook()))
    assert np.array_equal(np.array(th, dtype=np.float32).view(np.uint32), nf4.f32_bits(nf4.thresholds()))


def test_codebook_null_levels_rejected(lib):
    assert lib.qlora_nf4_codebook(None, None) == EINVAL


def test_int4_codebook_equals_oracle_bit_for_bit(lib):
    lv, th = q.codebook(q.CODEBOOK_INT4)
    assert np.array_equal(np.array(lv, dtype=np.float32).view(np.uint32), nf4.f32_bits(int4.levels()))
    mid = int4.midpoints()
    th32 = np.array(th, dtype=np.float32).astype(np.float64)
    assert np.all(th32 <= mid) and np.all(np.nextafter(th32.astype(np.float32), np.float32(2)) > mid)
    lv2, _ = q.codebook(q.CODEBOOK_NF4)
    assert lv2 == q.codebook()[0]


def test_codebook_kind_rejected(lib):
    lv = (ctypes.c_float * 16)()
    assert lib.qlora_codebook(2, lv, None) == EINVAL
    assert lib.qlora_codebook(-1, lv, None) == EINVAL
    assert lib.qlora_quantize_codebook(7, FAKE, 64, 64, FAKE, FAKE, FAKE, FAKE, FAKE, 1 << 20, None) == EINVAL


def test_status_strings(lib):
    for s in (OK, EINVAL, ESHAPE, EWS, ECUDA, ETIMEOUT):
        assert len(q.status_string(s)) >= 2
    assert q.status_string(12345) == "unknown status"


def test_workspace_sizes(lib):
    # quantize: absmax fp32 per block + fp64 tree partials
    n = q.workspace_size(q.OP_QUANTIZE, 0, 4096, 4096, 0)
    assert n >= 4096 * 4096 // 64 * 4
    assert q.workspace_size(q.OP_DEQUANTIZE, 0, 512, 512, 0) == 0
    # forward: at most the split-K partials of the rank-r down-projection
    assert q.workspace_size(q.OP_LINEAR_FWD, 4096, 4096, 4096, 16) <= 4096 * 16 * 4 * 64
    assert q.workspace_size(q.OP_LINEAR_FWD, 64, 128, 128, 8) == 0           # one K range
    assert q.workspace_size(q.OP_LINEAR_FWD, 4, 8192, 28672, 16) > 0        # split-K GEMV partials
    nb = q.workspace_size(q.OP_LINEAR_BWD, 4096, 4096, 4096, 16)
    assert nb >= 4096 * 16 * 2
    assert lib.qlora_workspace_size(99, 1, 64, 64, 8) == ctypes.c_size_t(-1).value
    assert lib.qlora_workspace_size(q.OP_LINEAR_FWD, -1, 64, 64, 8) == ctypes.c_size_t(-1).value


def _weight(rows=64, cols=64, codes=FAKE):
    return q._Weight(codes, FAKE, FAKE, FAKE, rows, cols)


def test_quantize_argument_errors(lib):
    ws = q.workspace_size(q.OP_QUANTIZE, 0, 128, 64, 0)
    f = lib.qlora_quantize_nf4
    assert f(None, 64, 128, FAKE, FAKE, FAKE, FAKE, FAKE, ws, None) == EINVAL
    assert f(FAKE + 4, 64, 128, FAKE, FAKE, FAKE, FAKE, FAKE, ws, None) == EINVAL      # misaligned W
    assert f(FAKE, 64, 100, FAKE, FAKE, FAKE, FAKE, FAKE, ws, None) == ESHAPE         # cols % 64
    assert f(FAKE, 0, 128, FAKE, FAKE, FAKE, FAKE, FAKE, ws, None) == ESHAPE          # rows < 1
    assert f(FAKE, 64, 128, FAKE, FAKE, FAKE, FAKE, None, ws, None) == EWS            # no workspace
    assert f(FAKE, 64, 128, FAKE, FAKE, FAKE, FAKE, FAKE, ws - 1, None) == EWS        # too small
    assert f(FAKE, 64, 128, FAKE, FAKE, FAKE, FAKE, FAKE + 16, ws, None) == EWS       # misaligned ws


def test_shard_quantize_argument_errors(lib):
    loc, fin = lib.qlora_quantize_nf4_shard_local, lib.qlora_quantize_nf4_shard_finish
    ws = q.quantize_shard_workspace_size(4096, 2)
    assert lib.qlora_quantize_shard_workspace_size(-1, 2) == ctypes.c_size_t(-1).value
    assert lib.qlora_quantize_shard_workspace_size(10, 0) == ctypes.c_size_t(-1).value
    assert loc(FAKE, 4096, FAKE, None, 1, FAKE, ws, None) == EINVAL              # no roots
    assert loc(FAKE, 4097, FAKE, FAKE, 1, FAKE, ws, None) == EINVAL              # shard larger than its chunks
    assert loc(FAKE + 4, 4096, FAKE, FAKE, 1, FAKE, ws, None) == EINVAL          # misaligned W
    assert loc(FAKE, 4096, FAKE, FAKE, 1, None, ws, None) == EWS                 # no workspace
    assert loc(FAKE, 4096, FAKE, FAKE, 1, FAKE, 1024, None) == EWS               # absmaxes do not fit
    assert fin(FAKE, 2, 8193, 4096, FAKE, FAKE, FAKE, FAKE, ws, None) == EINVAL  # more blocks than the roots cover
    assert fin(FAKE, 2, 4096, 4097, FAKE, FAKE, FAKE, FAKE, ws, None) == EINVAL  # shard larger than the weight
    assert fin(FAKE, 2, 8192, 4096, FAKE, FAKE, None, FAKE, ws, None) == EINVAL  # no mean
    assert fin(FAKE, 2, 8192, 4096, FAKE, FAKE, FAKE, FAKE, ws - 1, None) == EWS


def test_dequantize_argument_errors(lib):
    f = lib.qlora_dequantize_nf4
    assert f(None, FAKE, None) == EINVAL
    w = _weight(codes=0)
    assert f(ctypes.byref(w), FAKE, None) == EINVAL
    w = _weight(cols=96)
    assert f(ctypes.byref(w), FAKE, None) == ESHAPE
    w = _weight()
    assert f(ctypes.byref(w), FAKE + 2, None) == EINVAL


def test_linear_argument_errors(lib):
    fwd, bwd = lib.qlora_linear_fwd, lib.qlora_linear_bwd
    w = _weight(128, 128)
    wb = ctypes.byref(w)
    # null / misaligned pointers
    assert fwd(None, 64, wb, FAKE, FAKE, 8, 16.0, FAKE, FAKE, None, 0, None) == EINVAL
    assert fwd(FAKE, 64, wb, FAKE, FAKE, 8, 16.0, FAKE, FAKE + 8, None, 0, None) == EINVAL
    assert fwd(FAKE, 64, wb, FAKE, FAKE, 8, float("nan"), FAKE, FAKE, None, 0, None) == EINVAL
    # shape rules: 1 <= r <= 256, M >= 1, in/out multiples of 64
    for r in (0, -3, 257, 264):
        assert fwd(FAKE, 64, wb, FAKE, FAKE, r, 16.0, FAKE, FAKE, None, 0, None) == ESHAPE
    # a rank that is not a multiple of 8 runs on padded copies in the workspace
    for r in (1, 4, 12):
        assert fwd(FAKE, 64, wb, FAKE, FAKE, r, 16.0, FAKE, FAKE, None, 0, None) == EWS
        assert lib.qlora_workspace_size(2, 64, 128, 128, r) > 0
    assert fwd(FAKE, 0, wb, FAKE, FAKE, 8, 16.0, FAKE, FAKE, None, 0, None) == ESHAPE
    w2 = _weight(96, 128)
    assert fwd(FAKE, 64, ctypes.byref(w2), FAKE, FAKE, 8, 16.0, FAKE, FAKE, None, 0, None) == ESHAPE
    # the GEMV path needs a workspace when K spans several groups of slices
    w3 = _weight(128, 8192)
    assert fwd(FAKE, 4, ctypes.byref(w3), FAKE, FAKE, 8, 16.0, FAKE, FAKE, None, 0, None) == EWS
    # backward always needs one
    assert bwd(FAKE, FAKE, FAKE, 64, wb, FAKE, FAKE, 8, 16.0, FAKE, FAKE, FAKE, None, 0, None) == EWS
    assert bwd(FAKE, FAKE, None, 64, wb, FAKE, FAKE, 8, 16.0, FAKE, FAKE, FAKE, FAKE, 1 << 30, None) == EINVAL
    assert bwd(FAKE, FAKE, FAKE, 64, wb, FAKE, FAKE, 257, 16.0, FAKE, FAKE, FAKE, FAKE, 1 << 30, None) == ESHAPE


def test_group_argument_errors(lib):
    fwd, bwd, wsz = lib.qlora_linear_fwd_group, lib.qlora_linear_bwd_group, lib.qlora_linear_group_workspace_size
    w1, w2 = _weight(128, 128), _weight(256, 192)
    keep = (w1, w2)

    def prob(w, M=64, r=8, x=FAKE):
        return q._Problem(x, ctypes.pointer(w), FAKE, FAKE, M, r, 16.0, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE)

    arr = (q._Problem * 2)(prob(w1), prob(w2, M=300, r=12))
    # each projection's single-call workspace, rounded to 256 bytes, one after another
    for backward, op in ((0, q.OP_LINEAR_FWD), (1, q.OP_LINEAR_BWD)):
        each = [q.workspace_size(op, 64, 128, 128, 8), q.workspace_size(op, 300, 192, 256, 12)]
        assert wsz(backward, 2, arr) == sum(-(-n // 256) * 256 for n in each)
    assert wsz(0, 2, arr) > 0                       # r = 12 runs on padded copies
    size_max = ctypes.c_size_t(-1).value
    assert wsz(0, -1, arr) == size_max and wsz(0, 1, None) == size_max
    assert wsz(0, 0, None) == 0
    assert fwd(-1, arr, None, 0, None) == EINVAL and bwd(-1, arr, None, 0, None) == EINVAL
    assert fwd(1, None, None, 0, None) == EINVAL
    assert fwd(0, None, None, 0, None) == OK and bwd(0, None, None, 0, None) == OK
    # the first failing projection's status, before anything is issued
    bad = (q._Problem * 3)(prob(w1), prob(w2, r=0), prob(w1, x=FAKE + 8))
    assert fwd(3, bad, FAKE, 1 << 30, None) == ESHAPE
    assert bwd(3, bad, FAKE, 1 << 30, None) == ESHAPE
    bad[1] = prob(w2)
    assert fwd(3, bad, FAKE, 1 << 30, None) == EINVAL
    # a missing or short workspace
    assert fwd(2, arr, None, 0, None) == EWS
    assert bwd(2, arr, FAKE, wsz(1, 2, arr) - 256, None) == EWS
    assert bwd(2, arr, FAKE + 16, 1 << 30, None) == EWS            # not 256-byte aligned
    del keep


def test_dropout_argument_errors(lib):
    fwd, bwd = lib.qlora_linear_fwd_dropout, lib.qlora_linear_bwd_dropout
    w = _weight(128, 128)
    wb = ctypes.byref(w)
    # keep mask: null or not 4-byte aligned, p outside [0, 1)
    assert fwd(FAKE, 64, wb, FAKE, FAKE, 8, 16.0, None, 0.05, FAKE, FAKE, None, 0, None) == EINVAL
    assert fwd(FAKE, 64, wb, FAKE, FAKE, 8, 16.0, FAKE + 2, 0.05, FAKE, FAKE, None, 0, None) == EINVAL
    assert fwd(FAKE, 64, wb, FAKE, FAKE, 8, 16.0, FAKE, 1.0, FAKE, FAKE, None, 0, None) == EINVAL
    assert fwd(FAKE, 64, wb, FAKE, FAKE, 8, 16.0, FAKE, -0.1, FAKE, FAKE, None, 0, None) == EINVAL
    # the few-token forward needs a workspace when K spans several slice groups;
    # the large-M one none (the mask is applied in place of a copy)
    w3 = _weight(128, 8192)
    assert fwd(FAKE, 4, ctypes.byref(w3), FAKE, FAKE, 8, 16.0, FAKE, 0.05, FAKE, FAKE, None, 0, None) == EWS
    assert q.workspace_size(q.OP_LINEAR_FWD_DROPOUT, 64, 128, 128, 8) == 0
    assert q.workspace_size(q.OP_LINEAR_BWD_DROPOUT, 64, 128, 128, 8) == q.workspace_size(q.OP_LINEAR_BWD, 64, 128,
                                                                                           128, 8)
    assert bwd(FAKE, FAKE, FAKE, 64, wb, FAKE, FAKE, 8, 16.0, FAKE + 1, 0.05, FAKE, FAKE, FAKE, FAKE, 1 << 30,
               None) == EINVAL
    assert bwd(FAKE, FAKE, FAKE, 64, wb, FAKE, FAKE, 8, 16.0, FAKE, 0.05, FAKE, FAKE, FAKE, None, 0, None) == EWS


def test_merge_argument_errors(lib):
    f = lib.qlora_merge_adapter
    w = _weight(128, 128)
    wb = ctypes.byref(w)
    assert f(None, FAKE, FAKE, 8, 16.0, FAKE, None) == EINVAL
    assert f(wb, None, FAKE, 8, 16.0, FAKE, None) == EINVAL
    assert f(wb, FAKE, FAKE, 8, 16.0, FAKE + 8, None) == EINVAL          # misaligned output
    assert f(wb, FAKE, FAKE, 8, float("inf"), FAKE, None) == EINVAL
    for r in (0, 257):
        assert f(wb, FAKE, FAKE, r, 16.0, FAKE, None) == ESHAPE
    w2 = _weight(96, 128)
    assert f(ctypes.byref(w2), FAKE, FAKE, 8, 16.0, FAKE, None) == ESHAPE


def test_timeout_setter_roundtrip(lib):
    prev = q.set_wait_timeout_ns(5_000_000)
    assert q.set_wait_timeout_ns(prev) == 5_000_000
    assert q.set_wait_timeout_ns(10) >= 1000      # previous value returned
    assert q.set_wait_timeout_ns(prev) == 1000     # clamped to the 1 us minimum


def test_binding_fails_loudly_without_library(tmp_path, monkeypatch):
    import importlib
    monkeypatch.setattr(q, "_LIB", None)
    monkeypatch.setattr(q, "library_path", lambda: str(tmp_path / "missing.so"))
    with pytest.raises(RuntimeError, match="no fallback"):
        q.load()
    importlib.reload(q)


def test_header_compiles_as_c_and_links(lib, tmp_path):
    # the boundary is plain C: the header compiles as C99 with warnings as
    # errors, and a C program links against the library and calls a host-only
    # entry point through it
    import shutil
    import subprocess
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    src = tmp_path / "abi.c"
    src.write_text(
        '#include "qlora_nf4.h"\n'
        "#include <stdio.h>\n"
        "int main(void) {\n"
        "  float levels[16], thr[15];\n"
        "  qlora_linear_problem p = {0};\n"
        "  (void)p;\n"
        "  if (qlora_nf4_codebook(levels, thr) != QLORA_OK) return 1;\n"
        "  if (qlora_linear_group_workspace_size(0, 0, NULL) != 0) return 2;\n"
        '  printf("%.9g %.9g\\n", levels[0], levels[15]);\n'
        "  return levels[7] == 0.0f ? 0 : 3;\n"
        "}\n")
    exe = tmp_path / "abi"
    libdir = os.path.dirname(q.library_path())
    res = subprocess.run([cc, "-std=c99", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(root, "include"),
                          str(src), "-o", str(exe), "-L", libdir, "-lqlora_nf4", f"-Wl,-rpath,{libdir}"],
                         capture_output=True, text=True)
    assert res.returncode == 0, res.stderr
    run = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert run.returncode == 0, run.stdout + run.stderr
    assert run.stdout.split()[0] == "-1" and run.stdout.split()[1] == "1"
