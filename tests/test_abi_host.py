"""Host-side checks of the C-ABI library: it loads without a GPU, exports
every entry point the header declares, sizes its workspace, and rejects bad
arguments before queuing any GPU work. Fake (never dereferenced) pointer
values stand in for device memory; every call here returns before any CUDA
call is made."""
import ctypes
import os
import re

import pytest

from conftest import ROOT

HEADER = os.path.join(ROOT, "include", "llmint8.h")


@pytest.fixture(scope="module")
def lib():
    from int8_mixed_precision_rowwise_b200 import build as b
    b.build()
    import int8_mixed_precision_rowwise_b200 as m
    return m


def declared_functions():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"LLMINT8_API\s+[\w\s\*]+?\b(llmint8_\w+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for need in ("llmint8_quantize_rowwise", "llmint8_find_outlier_cols", "llmint8_matmul_mixed"):
        assert need in names


def test_library_exports_every_declared_symbol(lib):
    cdll = ctypes.CDLL(lib.LIB_PATH)
    for name in declared_functions():
        assert hasattr(cdll, name), name
    assert set(lib.EXPORTED) == set(declared_functions())


def test_status_strings(lib):
    assert lib.status_string(0) == "LLMINT8_OK"
    for s in range(1, 7):
        assert lib.status_string(s).startswith("LLMINT8_ERR_")
    assert lib.status_string(99) == "LLMINT8_ERR_UNKNOWN"


def test_workspace_sizes(lib):
    M, N, K = 2048, 16384, 4096
    need = lib.workspace_size(M, N, K)
    # at least CX + SX + col_idx + bitmap
    assert need >= M * K + 4 * M + 4 * K + K // 8
    assert need % 256 == 0
    # the prefill path keeps per-call copies of W's outlier columns: 32 columns x N, and SB
    grow = lib.workspace_size(M, 2 * N, K) - lib.workspace_size(M, N, K)
    assert 33 * 4 * N <= grow <= 33 * 4 * N + 1024
    assert lib.workspace_size(32, 2 * N, K) == lib.workspace_size(32, N, K)  # decode shapes have no such copies
    # from M = 256 (CTA-pair GEMM) the stream-K slots: 80 pairs x 256 KB of int32 partials, and their flags
    assert lib.workspace_size(256, N, K) - lib.workspace_size(255, N, K) >= 80 * 262144
    assert lib.quantize_workspace_size(M, K) < need
    assert lib.workspace_size(-1, N, K) == 0


A = 0x10000  # aligned fake device address
P = ctypes.c_void_p


def _mm(lib, X=A, M=64, K=128, CB=A, SCB=A, W=None, N=64, t=6.0, Y=A, ws=A, wsb=None):
    wsb = lib.workspace_size(M, N, K) if wsb is None else wsb
    return lib._matmul_mixed(X, M, K, CB, SCB, W, N, t, Y, ws, wsb, None, None)


def test_workspace_holds_the_fixed_regions(lib):
    """Every workspace, whatever its shape, has the header and the resident
    quantizer's two outlier bitmaps (sized for the widest X) at the front, so
    that calls of any shapes can share it."""
    fixed = 256 + 2 * 4 * ((133143 + 31) // 32)
    for rows, cols in [(1, 16), (8, 64), (4096, 4096), (2048, 57344)]:
        assert lib.quantize_workspace_size(rows, cols) >= fixed + (cols + 31) // 32 * 4 + cols * 4
    for M, N, K in [(1, 16, 16), (32, 14336, 14336), (2048, 16384, 4096)]:
        assert lib.workspace_size(M, N, K) >= fixed + M * K + 4 * M


def test_matmul_argument_errors(lib):
    assert _mm(lib, K=100) == lib.ERR_UNSUPPORTED_SHAPE     # K % 16
    assert _mm(lib, K=0) == lib.ERR_UNSUPPORTED_SHAPE
    assert _mm(lib, K=133152) == lib.ERR_UNSUPPORTED_SHAPE  # > LLMINT8_MAX_K
    assert _mm(lib, M=-1) == lib.ERR_INVALID_ARG
    assert _mm(lib, X=None) == lib.ERR_INVALID_ARG
    assert _mm(lib, CB=None) == lib.ERR_INVALID_ARG
    assert _mm(lib, SCB=None) == lib.ERR_INVALID_ARG
    assert _mm(lib, Y=None) == lib.ERR_INVALID_ARG
    assert _mm(lib, ws=None) == lib.ERR_INVALID_ARG
    assert _mm(lib, X=A + 8) == lib.ERR_ALIGNMENT
    assert _mm(lib, W=A + 2) == lib.ERR_ALIGNMENT
    assert _mm(lib, Y=A + 4) == lib.ERR_ALIGNMENT
    assert _mm(lib, wsb=1024) == lib.ERR_WORKSPACE
    assert _mm(lib, M=0) == lib.OK   # empty: no-op, nothing queued
    assert _mm(lib, N=0) == lib.OK


def test_matmul_ex_argument_errors(lib):
    """The bias/activation entry point checks its two extra arguments before
    anything is queued; the others are checked as for llmint8_matmul_mixed."""
    f = lib._matmul_mixed_ex
    M, N, K = 64, 64, 128
    ws = lib.workspace_size(M, N, K)

    def call(bias=None, act=0, X=A, wsb=ws):
        return f(X, M, K, A, A, None, N, 6.0, bias, act, A, A, wsb, None, None)

    assert call(act=2) == lib.ERR_INVALID_ARG
    assert call(act=-1) == lib.ERR_INVALID_ARG
    assert call(bias=A + 2) == lib.ERR_ALIGNMENT
    assert call(X=None, act=1) == lib.ERR_INVALID_ARG
    assert call(wsb=1024, bias=A, act=1) == lib.ERR_WORKSPACE


def test_matmul_fp16w_argument_errors(lib):
    f = lib._matmul_mixed_fp16w
    M, N, K = 64, 64, 128
    ws = lib.workspace_size_fp16w(M, N, K)
    assert ws >= lib.workspace_size(M, N, K) + N * K + 4 * N

    def call(W=A, wsb=ws, K=K, act=0):
        return f(A, M, K, W, N, 6.0, None, act, A, A, wsb, None, None)

    assert call(W=None) == lib.ERR_INVALID_ARG
    assert call(W=A + 8) == lib.ERR_ALIGNMENT
    assert call(wsb=lib.workspace_size(M, N, K)) == lib.ERR_WORKSPACE
    assert call(K=100) == lib.ERR_UNSUPPORTED_SHAPE
    assert call(act=3) == lib.ERR_INVALID_ARG


def test_asym_argument_errors(lib):
    """The zero-point entry points check their arguments before queuing work;
    K is limited to LLMINT8_MAX_K_ASYM (int32 sums of codes up to 128 in size)."""
    q = lib._quantize_rowwise_asym
    ws = lib.quantize_workspace_size(32, 64)
    assert q(A, 32, 64, 6.0, A, A, A, None, A, ws, None) == lib.ERR_INVALID_ARG      # bitmap needed when t > 0
    assert q(A, 32, 64, 0.0, A, A, None, None, A, ws, None) == lib.ERR_INVALID_ARG   # zero points
    assert q(A, 32, 60, 0.0, A, A, A, None, A, ws, None) == lib.ERR_UNSUPPORTED_SHAPE
    assert q(A, 32, lib.MAX_K_ASYM + 16, 0.0, A, A, A, None, A, 1 << 30, None) == lib.ERR_UNSUPPORTED_SHAPE
    assert q(A, 32, 64, 0.0, A, A + 4, A, None, A, ws, None) == lib.ERR_ALIGNMENT
    assert q(A, 32, 64, 0.0, A, A, A, None, A, 16, None) == lib.ERR_WORKSPACE
    assert q(A, 0, 64, 0.0, A, A, A, None, A, ws, None) == lib.OK
    r = lib._code_row_sums
    assert r(A, 8, 64, None, None) == lib.ERR_INVALID_ARG
    assert r(A, 8, 60, A, None) == lib.ERR_UNSUPPORTED_SHAPE
    assert r(A + 8, 8, 64, A, None) == lib.ERR_ALIGNMENT
    assert r(A, 0, 64, A, None) == lib.OK
    m = lib._matmul_mixed_asym
    M, N, K = 64, 64, 128
    wsa = lib.workspace_size_asym(M, N, K)
    assert wsa >= lib.workspace_size(M, 1, K) + 4 * M

    def call(R=A, wsb=wsa, K=K, X=A):
        return m(X, M, K, A, A, R, None, N, 6.0, A, A, wsb, None, None)

    assert call(R=None) == lib.ERR_INVALID_ARG
    assert call(R=A + 2) == lib.ERR_ALIGNMENT
    assert call(X=A + 8) == lib.ERR_ALIGNMENT
    assert call(wsb=wsa - 256) == lib.ERR_WORKSPACE
    assert call(K=lib.MAX_K_ASYM + 16) == lib.ERR_UNSUPPORTED_SHAPE


def test_quantize_argument_errors(lib):
    q = lib._quantize_rowwise
    ws = lib.quantize_workspace_size(32, 64)
    assert q(A, 32, 60, 6.0, A, A, A, A, ws, None) == lib.ERR_UNSUPPORTED_SHAPE
    assert q(A, 32, 64, 6.0, A, A, None, A, ws, None) == lib.ERR_INVALID_ARG     # bitmap needed when t > 0
    assert q(A, 32, 64, 6.0, A, A + 1, A, A, ws, None) == lib.ERR_ALIGNMENT
    assert q(A, 32, 64, 6.0, A, A, A, A, 16, None) == lib.ERR_WORKSPACE
    assert q(A, 0, 64, 0.0, A, A, None, A, ws, None) == lib.OK                   # no rows, no bitmap: nothing queued
    # (no rows with a bitmap queues one memset of it: a GPU test covers that)


def test_find_outlier_cols_argument_errors(lib):
    f = lib._find_outlier_cols
    assert f(None, 64, A, A, None, None) == lib.ERR_INVALID_ARG
    assert f(A, 0, A, A, None, None) == lib.ERR_UNSUPPORTED_SHAPE
    assert f(A + 4, 64, A, A, None, None) == lib.ERR_ALIGNMENT


def test_gemm_argument_errors(lib):
    g = lib._gemm_s8s8s32
    ws = lib.workspace_size(64, 64, 128)
    assert g(A, 64, A, 64, 120, A, A, ws, None) == lib.ERR_UNSUPPORTED_SHAPE
    assert g(A, 64, None, 64, 128, A, A, ws, None) == lib.ERR_INVALID_ARG
    assert g(A, 64, A, 64, 128, A + 8, A, ws, None) == lib.ERR_ALIGNMENT
    assert g(A, 64, A, 64, 128, A, A, 8, None) == lib.ERR_WORKSPACE
    assert g(A, 0, A, 64, 128, A, A, ws, None) == lib.OK


def test_no_cpu_fallback(lib):
    """Tensors on the CPU are refused: the library has no host compute path."""
    import torch
    X = torch.zeros((4, 16), dtype=torch.float16)
    with pytest.raises(TypeError):
        lib.quantize_rowwise(X, 6.0)
    with pytest.raises(TypeError):
        lib.matmul_mixed(X, torch.zeros((4, 16), dtype=torch.int8), torch.zeros(4))


def test_tensor_parallel_argument_errors(lib):
    """The tensor-parallel pieces check their arguments before queuing work."""
    qg = lib._quantize_rowwise_given
    assert qg(A, 32, 64, A, 1, None, A, None, None, None) == lib.ERR_INVALID_ARG   # no absmax in or out
    assert qg(A, 32, 64, None, 2, None, A, A, None, None) == lib.ERR_INVALID_ARG   # bitmaps missing
    assert qg(A, 32, 60, None, 0, None, A, A, None, None) == lib.ERR_UNSUPPORTED_SHAPE
    assert qg(A, 32, 64, A + 4, 1, None, A, A, None, None) == lib.ERR_ALIGNMENT
    assert qg(A, 0, 64, None, 0, None, A, A, None, None) == lib.OK                 # no rows, no bitmap_out
    mc = lib._matmul_codes

    def call(out=lib.OUT_F16, wsb=256, K=128, Y=A, cnt=A, act=0):
        return mc(A, A, A, 64, K, A, A, None, 64, A, cnt, None, act, out, Y, A, wsb, None)

    assert call(out=2) == lib.ERR_INVALID_ARG
    assert call(act=5) == lib.ERR_INVALID_ARG
    assert call(cnt=None) == lib.ERR_INVALID_ARG
    assert call(cnt=A + 2) == lib.ERR_ALIGNMENT
    assert call(Y=A + 8) == lib.ERR_ALIGNMENT
    assert call(wsb=64) == lib.ERR_WORKSPACE
    assert call(K=100) == lib.ERR_UNSUPPORTED_SHAPE
    ba = lib._bias_act_to_f16
    assert ba(A, 8, 10, None, 0, A, None) == lib.ERR_UNSUPPORTED_SHAPE              # N % 4
    assert ba(A, 8, 16, None, 2, A, None) == lib.ERR_INVALID_ARG
    assert ba(A + 4, 8, 16, None, 0, A, None) == lib.ERR_ALIGNMENT
    assert ba(A, 0, 16, None, 0, A, None) == lib.OK
    gc = lib._gather_column_blocks
    assert gc(A, 2, 8, 12, A, None) == lib.ERR_UNSUPPORTED_SHAPE                   # Nr % 8
    assert gc(None, 2, 8, 16, A, None) == lib.ERR_INVALID_ARG
    assert gc(A, 0, 8, 16, A, None) == lib.OK
