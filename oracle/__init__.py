"""CPU oracle for the LLM.int8() mixed-precision linear (test infrastructure).

Only the tests, the package's smoke check and the benchmark's CPU-baseline
leg import this module. It is independent of the CUDA library: it neither
imports nor links anything from the package, and the package never imports
it. The arithmetic lives in ``llmint8_oracle.c`` (plain single-threaded C);
this file only widens fp16 inputs to fp32 (exact) and moves arrays in and
out through ctypes.

Pipeline, in the order of the source page's three steps (page "Hugging Face
将 LLM.int8() 8-bit 量化集成进 transformers 与 accelerate", section
"LLM.int8() 的简要总结", a gentle summary of LLM.int8()):

1. ``outlier_cols``        - hidden columns holding any |x| >= threshold
2. ``quantize_rowwise``    - absmax row quantization of the non-outlier part
3. ``int8_matmul``         - exact int8 x int8 -> int32 product
4. ``outlier_weight``      - W's outlier columns (fp16 W or CB * SCB / 127)
5. ``mixed_output``        - outer-product dequant plus the fp16 outlier product
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "llmint8_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lib = None

CFLAGS = ["-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off", "-fno-fast-math"]


def build(force: bool = False) -> str:
    """Compile the C oracle into ``oracle/liboracle.so`` (gcc, a few seconds)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        subprocess.check_call(["gcc", *CFLAGS, "-o", _LIB_PATH, _SRC, "-lm"])
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB_PATH)
        P = ctypes.c_void_p
        I64 = ctypes.c_int64
        lib.oracle_outlier_cols.argtypes = [P, I64, I64, ctypes.c_float, P]
        lib.oracle_outlier_cols.restype = I64
        lib.oracle_quantize_rows.argtypes = [P, I64, I64, P, P, P]
        lib.oracle_quantize_rows.restype = I64
        lib.oracle_int8_matmul.argtypes = [P, I64, P, I64, I64, P]
        lib.oracle_int8_matmul.restype = I64
        lib.oracle_outlier_weight.argtypes = [P, P, P, I64, I64, P, I64, P]
        lib.oracle_outlier_weight.restype = None
        lib.oracle_mixed_output.argtypes = [P, P, P, I64, I64, P, I64, P, I64, P, P]
        lib.oracle_bias_act.restype = None
        lib.oracle_bias_act.argtypes = [P, I64, I64, P, ctypes.c_int]
        lib.oracle_mixed_output.restype = None
        lib.oracle_quantize_rows_asym.argtypes = [P, I64, I64, P, P, P, P]
        lib.oracle_quantize_rows_asym.restype = I64
        lib.oracle_code_row_sums.argtypes = [P, I64, I64, P]
        lib.oracle_code_row_sums.restype = None
        lib.oracle_mixed_output_asym.argtypes = [P, P, P, P, P, I64, I64, P, I64, P, I64, P, P]
        lib.oracle_mixed_output_asym.restype = None
        _lib = lib
    return _lib


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p) if a is not None else None


def _f32(x) -> np.ndarray:
    """Exact widening of fp16 (or fp32) data to a C-contiguous fp32 array."""
    x = np.asarray(x)
    if x.dtype not in (np.float16, np.float32):
        raise TypeError(f"oracle inputs are fp16 or fp32, got {x.dtype}")
    return np.ascontiguousarray(x, dtype=np.float32)


def outlier_mask(X, threshold: float) -> np.ndarray:
    """uint8 [K]: 1 where some row holds |x| >= threshold (threshold <= 0: none)."""
    x = _f32(X)
    rows, cols = x.shape
    mask = np.zeros(cols, dtype=np.uint8)
    _load().oracle_outlier_cols(_ptr(x), rows, cols, np.float32(threshold), _ptr(mask))
    return mask


def outlier_cols(X, threshold: float) -> np.ndarray:
    """Ascending int64 indices of the outlier columns."""
    return np.flatnonzero(outlier_mask(X, threshold)).astype(np.int64)


def quantize_rowwise(X, outlier: np.ndarray | None = None):
    """(codes int8 [M x K], absmax fp32 [M]) over the non-outlier columns.

    ``outlier`` is a uint8 mask [K] or an index array, or None for no outliers."""
    x = _f32(X)
    rows, cols = x.shape
    mask = None
    if outlier is not None:
        outlier = np.asarray(outlier)
        if outlier.dtype == np.uint8 and outlier.shape == (cols,):
            mask = np.ascontiguousarray(outlier)
        else:
            mask = np.zeros(cols, dtype=np.uint8)
            mask[outlier.astype(np.int64)] = 1
    codes = np.empty((rows, cols), dtype=np.int8)
    absmax = np.empty(rows, dtype=np.float32)
    bad = _load().oracle_quantize_rows(_ptr(x), rows, cols, _ptr(mask), _ptr(codes), _ptr(absmax))
    if bad:
        raise AssertionError(f"oracle produced {bad} codes outside [-127, 127]")
    return codes, absmax


def int8_matmul(A: np.ndarray, B: np.ndarray) -> np.ndarray:
    """Exact int32 [M x N] = A[M x K] . B[N x K]^T (int64 sums, checked)."""
    A = np.ascontiguousarray(A, dtype=np.int8)
    B = np.ascontiguousarray(B, dtype=np.int8)
    (M, K), (N, K2) = A.shape, B.shape
    assert K == K2
    acc = np.empty((M, N), dtype=np.int32)
    over = _load().oracle_int8_matmul(_ptr(A), M, _ptr(B), N, K, _ptr(acc))
    if over:
        raise OverflowError(f"{over} int8 sums do not fit in int32")
    return acc


def outlier_weight(cols: np.ndarray, N: int, K: int, W=None, CB=None, SB=None) -> np.ndarray:
    """fp32 [N x |O|]: W[:, cols] if the fp16 weight is given, else CB*SB/127 per row."""
    cols = np.ascontiguousarray(cols, dtype=np.int64)
    Wt = np.empty((N, cols.size), dtype=np.float32)
    w = _f32(W) if W is not None else None
    cb = np.ascontiguousarray(CB, dtype=np.int8) if CB is not None else None
    sb = np.ascontiguousarray(SB, dtype=np.float32) if SB is not None else None
    if w is None and (cb is None or sb is None):
        raise ValueError("need W, or CB and SB")
    _load().oracle_outlier_weight(_ptr(w), _ptr(cb), _ptr(sb), N, K, _ptr(cols), cols.size, _ptr(Wt))
    return Wt


def mixed_output(acc, SX, SB, X, cols, Wt) -> np.ndarray:
    """fp64 [M x N] = acc*SX*SB/127^2 + X[:, cols] . Wt^T."""
    acc = np.ascontiguousarray(acc, dtype=np.int32)
    M, N = acc.shape
    x = _f32(X)
    K = x.shape[1]
    cols = np.ascontiguousarray(cols, dtype=np.int64)
    Wt = np.ascontiguousarray(Wt, dtype=np.float32)
    sx = np.ascontiguousarray(SX, dtype=np.float32)
    sb = np.ascontiguousarray(SB, dtype=np.float32)
    Y = np.empty((M, N), dtype=np.float64)
    _load().oracle_mixed_output(_ptr(acc), _ptr(sx), _ptr(sb), M, N, _ptr(x), K, _ptr(cols),
                                cols.size, _ptr(Wt), _ptr(Y))
    return Y


ACTIVATIONS = {None: 0, "none": 0, "gelu_tanh": 1}


def bias_act(Y, bias=None, activation=None) -> np.ndarray:
    """fp64 act(Y + bias): bias fp16/fp32 [N] or None, activation None or
    "gelu_tanh" (BLOOM's tanh-form GELU)."""
    Y = np.array(Y, dtype=np.float64, order="C")
    M, N = Y.shape
    b = None if bias is None else np.ascontiguousarray(np.asarray(bias).astype(np.float32))
    _load().oracle_bias_act(_ptr(Y), M, N, None if b is None else _ptr(b), ACTIVATIONS[activation])
    return Y


def quantize_weight(W):
    """Offline weight preparation: row-wise absmax over the full row (no outliers)."""
    return quantize_rowwise(W, None)


def matmul_mixed(X, threshold: float, W=None, CB=None, SB=None, use_fp16_weight_cols: bool = True, bias=None,
                 activation=None):
    """The whole LLM.int8() linear on the host.

    X fp16 [M x K]. The weight is given as fp16 W [N x K] (then CB/SB are made
    from it), or as CB/SB only. ``use_fp16_weight_cols`` picks the source of
    W's outlier columns when W is given (False: recover them from CB*SB/127).
    ``bias`` (fp16 [N]) and ``activation`` follow the linear (bias_act).
    Returns a dict with O (ascending columns), CX, SX, CB, SB, acc, Wt,
    Y_lin (the linear alone) and Y (after bias and activation), both fp64."""
    x = _f32(X)
    if CB is None:
        CB, SB = quantize_weight(W)
    N, K = CB.shape
    O = outlier_cols(x, threshold)
    CX, SX = quantize_rowwise(x, O)
    acc = int8_matmul(CX, CB)
    Wt = outlier_weight(O, N, K, W=W if (W is not None and use_fp16_weight_cols) else None, CB=CB, SB=SB)
    Y_lin = mixed_output(acc, SX, SB, x, O, Wt)
    Y = Y_lin if (bias is None and not ACTIVATIONS[activation]) else bias_act(Y_lin, bias, activation)
    return dict(O=O, CX=CX, SX=SX, CB=CB, SB=SB, acc=acc, Wt=Wt, Y_lin=Y_lin, Y=Y)


# ---- the zero-point (unsigned int8) variant: section "模型量化简介" ----------------

def _mask(outlier, cols):
    if outlier is None:
        return None
    outlier = np.asarray(outlier)
    if outlier.dtype == np.uint8 and outlier.shape == (cols,):
        return np.ascontiguousarray(outlier)
    mask = np.zeros(cols, dtype=np.uint8)
    mask[outlier.astype(np.int64)] = 1
    return mask


def quantize_rowwise_asym(X, outlier: np.ndarray | None = None, return_clamped: bool = False):
    """(codes int8 [M x K] = q - 128, scale fp32 [M], zero int32 [M]) of the
    zero-point quantization over the non-outlier columns: range
    [min(0, min x), max(0, max x)], s = 255 / range, z = rint(-lo * s),
    q = clamp(rint(x * s) + z, 0, 255); outlier columns get q = z. With
    ``return_clamped`` a fourth item: how many codes the clamp moved."""
    x = _f32(X)
    rows, cols = x.shape
    mask = _mask(outlier, cols)
    codes = np.empty((rows, cols), dtype=np.int8)
    scale = np.empty(rows, dtype=np.float32)
    zero = np.empty(rows, dtype=np.int32)
    # The clamp is part of the reading: rint(x s) and rint(-lo s) round
    # separately, so the row's extreme values can land one step past [0, 255].
    clamped = _load().oracle_quantize_rows_asym(_ptr(x), rows, cols, _ptr(mask), _ptr(codes), _ptr(scale),
                                                _ptr(zero))
    if return_clamped:
        return codes, scale, zero, int(clamped)
    return codes, scale, zero


def code_row_sums(CB) -> np.ndarray:
    """int64 [N]: sum over K of each row of the int8 weight codes."""
    cb = np.ascontiguousarray(CB, dtype=np.int8)
    N, K = cb.shape
    R = np.empty(N, dtype=np.int64)
    _load().oracle_code_row_sums(_ptr(cb), N, K, _ptr(R))
    return R


def mixed_output_asym(acc, scale, zero, R, SB, X, cols, Wt) -> np.ndarray:
    """fp64 [M x N] = (acc + (128 - z_i) R_j) SB_j / (127 s_i) + X[:, cols] . Wt^T."""
    acc = np.ascontiguousarray(acc, dtype=np.int32)
    M, N = acc.shape
    x = _f32(X)
    K = x.shape[1]
    cols = np.ascontiguousarray(cols, dtype=np.int64)
    Wt = np.ascontiguousarray(Wt, dtype=np.float32)
    sc = np.ascontiguousarray(scale, dtype=np.float32)
    z = np.ascontiguousarray(zero, dtype=np.int32)
    r = np.ascontiguousarray(R, dtype=np.int64)
    sb = np.ascontiguousarray(SB, dtype=np.float32)
    Y = np.empty((M, N), dtype=np.float64)
    _load().oracle_mixed_output_asym(_ptr(acc), _ptr(sc), _ptr(z), _ptr(r), _ptr(sb), M, N, _ptr(x), K,
                                     _ptr(cols), cols.size, _ptr(Wt), _ptr(Y))
    return Y


def matmul_mixed_asym(X, threshold: float, W=None, CB=None, SB=None, use_fp16_weight_cols: bool = True):
    """The LLM.int8() linear with zero-point codes for X (the weight keeps its
    absmax codes). Returns a dict with O, CX, SXs (scales), ZX (zero points),
    CB, SB, R (code row sums), acc (int8 product of the stored codes), Wt and
    Y (fp64)."""
    x = _f32(X)
    if CB is None:
        CB, SB = quantize_weight(W)
    N, K = CB.shape
    O = outlier_cols(x, threshold)
    CX, SXs, ZX = quantize_rowwise_asym(x, O)
    acc = int8_matmul(CX, CB)
    R = code_row_sums(CB)
    Wt = outlier_weight(O, N, K, W=W if (W is not None and use_fp16_weight_cols) else None, CB=CB, SB=SB)
    Y = mixed_output_asym(acc, SXs, ZX, R, SB, x, O, Wt)
    return dict(O=O, CX=CX, SXs=SXs, ZX=ZX, CB=CB, SB=SB, R=R, acc=acc, Wt=Wt, Y=Y)
