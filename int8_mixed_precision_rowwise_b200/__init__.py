"""Python binding of ``libllmint8.so``, the B200 LLM.int8() linear layer.

The functions below carry the C entry points' names (without the
``llmint8_`` prefix) and only marshal arguments: torch supplies device
memory and the current CUDA stream, every step of the computation runs in
the library's CUDA kernels. There is no CPU path: if the library is missing
or no CUDA device is present, calls fail loudly.

Method: the LLM.int8() mixed-precision decomposition described on the page
"Hugging Face 将 LLM.int8() 8-bit 量化集成进 transformers 与 accelerate"
(sections "模型量化简介", "LLM.int8() 的简要总结", "MatMul 内部", "用法").
"""
from __future__ import annotations

import ctypes
import os

__all__ = [
    "LIB_PATH", "LLMInt8Error", "status_string", "quantize_workspace_size", "workspace_size",
    "workspace_init", "read_status", "quantize_rowwise", "find_outlier_cols", "matmul_mixed",
    "gemm_s8s8s32", "Int8MixedLinear", "DEFAULT_THRESHOLD", "quantize_rowwise_noalloc", "noalloc_read_status",
    "matmul_mixed_fp16w",
    "workspace_size_fp16w", "ACTIVATIONS", "quantize_rowwise_asym", "code_row_sums", "workspace_size_asym",
    "matmul_mixed_asym", "MAX_K_ASYM", "quantize_rowwise_given", "matmul_codes", "bias_act_to_f16",
    "gather_column_blocks", "OUT_F16", "OUT_F32", "outlier_bitmap",
]

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libllmint8.so")
DEFAULT_THRESHOLD = 6.0
MAX_K_ASYM = 132104  # LLMINT8_MAX_K_ASYM

OK, ERR_INVALID_ARG, ERR_ALIGNMENT, ERR_UNSUPPORTED_SHAPE, ERR_WORKSPACE, ERR_CUDA, ERR_DEVICE = range(7)
OUT_F16, OUT_F32 = 0, 1  # LLMINT8_OUT_*

class _Debug(ctypes.Structure):
    _fields_ = [("codes", ctypes.c_void_p), ("row_absmax", ctypes.c_void_p), ("col_idx", ctypes.c_void_p),
                ("count", ctypes.c_void_p), ("acc", ctypes.c_void_p), ("gemm_begin", ctypes.c_void_p),
                ("gemm_end", ctypes.c_void_p)]


_P = ctypes.c_void_p
_I64 = ctypes.c_int64
_ST = ctypes.c_int
# ctypes signatures of the C entry points (name -> (restype, argtypes)).
_SIGNATURES = {
    "llmint8_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "llmint8_quantize_workspace_size": (ctypes.c_size_t, [_I64, _I64]),
    "llmint8_workspace_size": (ctypes.c_size_t, [_I64, _I64, _I64]),
    "llmint8_workspace_init": (_ST, [_P, ctypes.c_size_t, _P]),
    "llmint8_read_status": (_ST, [_P, ctypes.c_size_t, ctypes.c_int, ctypes.POINTER(ctypes.c_uint32)]),
    "llmint8_quantize_rowwise": (_ST, [_P, _I64, _I64, ctypes.c_float, _P, _P, _P, _P, ctypes.c_size_t, _P]),
    "llmint8_find_outlier_cols": (_ST, [_P, _I64, _P, _P, _P, _P]),
    "llmint8_matmul_mixed": (_ST, [_P, _I64, _I64, _P, _P, _P, _I64, ctypes.c_float, _P, _P, ctypes.c_size_t,
                                   ctypes.POINTER(_Debug), _P]),
    "llmint8_matmul_mixed_ex": (_ST, [_P, _I64, _I64, _P, _P, _P, _I64, ctypes.c_float, _P, ctypes.c_int, _P, _P,
                                      ctypes.c_size_t, ctypes.POINTER(_Debug), _P]),
    "llmint8_workspace_size_fp16w": (ctypes.c_size_t, [_I64, _I64, _I64]),
    "llmint8_matmul_mixed_fp16w": (_ST, [_P, _I64, _I64, _P, _I64, ctypes.c_float, _P, ctypes.c_int, _P, _P,
                                         ctypes.c_size_t, ctypes.POINTER(_Debug), _P]),
    "llmint8_gemm_s8s8s32": (_ST, [_P, _I64, _P, _I64, _I64, _P, _P, ctypes.c_size_t, _P]),
    "llmint8_quantize_rowwise_noalloc": (_ST, [_P, _I64, _I64, ctypes.c_float, _P, _P, _P, _P]),
    "llmint8_noalloc_read_status": (_ST, [ctypes.c_int, ctypes.POINTER(ctypes.c_uint32)]),
    "llmint8_quantize_rowwise_given": (_ST, [_P, _I64, _I64, _P, ctypes.c_int, _P, _P, _P, _P, _P]),
    "llmint8_matmul_codes": (_ST, [_P, _P, _P, _I64, _I64, _P, _P, _P, _I64, _P, _P, _P, ctypes.c_int, ctypes.c_int,
                                   _P, _P, ctypes.c_size_t, _P]),
    "llmint8_bias_act_to_f16": (_ST, [_P, _I64, _I64, _P, ctypes.c_int, _P, _P]),
    "llmint8_gather_column_blocks": (_ST, [_P, _I64, _I64, _I64, _P, _P]),
    "llmint8_quantize_rowwise_asym": (_ST, [_P, _I64, _I64, ctypes.c_float, _P, _P, _P, _P, _P, ctypes.c_size_t,
                                            _P]),
    "llmint8_code_row_sums": (_ST, [_P, _I64, _I64, _P, _P]),
    "llmint8_workspace_size_asym": (ctypes.c_size_t, [_I64, _I64, _I64]),
    "llmint8_matmul_mixed_asym": (_ST, [_P, _I64, _I64, _P, _P, _P, _P, _I64, ctypes.c_float, _P, _P,
                                        ctypes.c_size_t, ctypes.POINTER(_Debug), _P]),
}
EXPORTED = tuple(_SIGNATURES)
NOALLOC_MAX_ROWS = NOALLOC_MAX_COLS = 65536
_fns: dict = {}


def load():
    """Load libllmint8.so (once) and bind its entry points. Raises ImportError
    when the library has not been built: there is no CPU fallback."""
    if not _fns:
        if not os.path.exists(LIB_PATH):
            raise ImportError(
                f"{LIB_PATH} is missing: build it with `python -m int8_mixed_precision_rowwise_b200.build` "
                "(nvcc, sm_100a). There is no CPU fallback.")
        cdll = ctypes.CDLL(LIB_PATH)
        fns = {}
        for name, (res, args) in _SIGNATURES.items():
            f = getattr(cdll, name)
            f.restype, f.argtypes = res, args
            fns["_" + name[len("llmint8_"):]] = f
        _fns.update(fns)
    return _fns


def __getattr__(name):
    # _matmul_mixed, _quantize_rowwise, ...: the raw ctypes entry points.
    if name.startswith("_") and "llmint8" + name in _SIGNATURES:
        return load()[name]
    raise AttributeError(name)


class LLMInt8Error(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)}")


def status_string(status: int) -> str:
    return load()["_status_string"](int(status)).decode()


def _check(status: int, where: str):
    if status != OK:
        raise LLMInt8Error(status, where)


def quantize_workspace_size(rows: int, cols: int) -> int:
    return int(load()["_quantize_workspace_size"](rows, cols))


def workspace_size(M: int, N: int, K: int) -> int:
    return int(load()["_workspace_size"](M, N, K))


# --------------------------------------------------------------------- torch glue

def _torch():
    import torch
    return torch


def _stream_ptr(device):
    torch = _torch()
    return torch.cuda.current_stream(device).cuda_stream


def _ptr(t):
    return None if t is None else t.data_ptr()


def _event(ev):
    """Raw cudaEvent_t of a torch.cuda.Event (created on its first record)."""
    if ev is None:
        return None
    if not ev.cuda_event:
        ev.record()
    return ev.cuda_event


def _need_cuda(t, name, dtype=None):
    torch = _torch()
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor (the library has no CPU path)")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")


# Cached workspaces, one per (device index, raw stream handle): calls that
# share a workspace must be ordered, which calls queued on one stream are, so
# two streams never share one.
_workspaces: dict = {}


def get_workspace(nbytes: int, device):
    """A zeroed, cached workspace of at least nbytes for `device` and its
    current stream (grown on demand)."""
    torch = _torch()
    d = torch.device(device)
    index = d.index if d.index is not None else torch.cuda.current_device()
    key = (index, _stream_ptr(torch.device("cuda", index)))
    ws = _workspaces.get(key)
    if ws is None or ws.numel() < nbytes:
        # The old buffer may still be in use by queued work on that stream:
        # torch's allocator keeps it alive until the stream reaches this point.
        ws = torch.zeros(max(nbytes, 4096), dtype=torch.uint8, device=d)
        _workspaces[key] = ws
    return ws


def workspaces(device=None) -> list:
    """The cached workspaces (of one device index, or all)."""
    return [ws for (idx, _), ws in _workspaces.items() if device is None or idx == device]


def workspace_init(ws) -> None:
    _check(load()["_workspace_init"](ws.data_ptr(), ws.numel(), _stream_ptr(ws.device)), "llmint8_workspace_init")


def read_status(ws, clear: bool = True) -> int:
    """The workspace's device status word (0: no kernel gave up on a wait)."""
    out = ctypes.c_uint32(0)
    st = load()["_read_status"](ws.data_ptr(), ws.numel(), int(clear), ctypes.byref(out))
    if st != ERR_DEVICE:
        _check(st, "llmint8_read_status")
    return int(out.value)


def noalloc_read_status(clear: bool = True) -> int:
    """The status word of the allocation-free quantizer's fixed array on the
    current device (0: none of its calls since the last clear gave up on a
    wait)."""
    out = ctypes.c_uint32(0)
    st = load()["_noalloc_read_status"](int(clear), ctypes.byref(out))
    if st != ERR_DEVICE:
        _check(st, "llmint8_noalloc_read_status")
    return int(out.value)


def quantize_rowwise(X, threshold: float = 0.0, codes=None, row_absmax=None, outlier_bitmap=None,
                     workspace=None):
    """(codes int8, row_absmax fp32, outlier_bitmap int32 words or None) of fp16 X [rows x cols]."""
    torch = _torch()
    _need_cuda(X, "X", torch.float16)
    rows, cols = X.shape
    dev = X.device
    if codes is None:
        codes = torch.empty((rows, cols), dtype=torch.int8, device=dev)
    if row_absmax is None:
        row_absmax = torch.empty(rows, dtype=torch.float32, device=dev)
    if outlier_bitmap is None and threshold > 0:
        outlier_bitmap = torch.empty((cols + 31) // 32, dtype=torch.int32, device=dev)
    ws = workspace if workspace is not None else get_workspace(quantize_workspace_size(rows, cols), dev)
    _check(load()["_quantize_rowwise"](X.data_ptr(), rows, cols, float(threshold), codes.data_ptr(),
                             row_absmax.data_ptr(), _ptr(outlier_bitmap), ws.data_ptr(), ws.numel(),
                             _stream_ptr(dev)), "llmint8_quantize_rowwise")
    return codes, row_absmax, outlier_bitmap


def quantize_rowwise_noalloc(X, threshold: float = 0.0, codes=None, row_absmax=None, outlier_bitmap=None):
    """quantize_rowwise without a workspace, for callers that cannot allocate
    device memory: the library's fixed scratch array (rows and cols up to
    65536) replaces it. Pass preallocated outputs to allocate nothing here
    either. Calls that overlap on the GPU share that scratch and race."""
    torch = _torch()
    _need_cuda(X, "X", torch.float16)
    rows, cols = X.shape
    dev = X.device
    if codes is None:
        codes = torch.empty((rows, cols), dtype=torch.int8, device=dev)
    if row_absmax is None:
        row_absmax = torch.empty(rows, dtype=torch.float32, device=dev)
    if outlier_bitmap is None and threshold > 0:
        outlier_bitmap = torch.empty((cols + 31) // 32, dtype=torch.int32, device=dev)
    _check(load()["_quantize_rowwise_noalloc"](X.data_ptr(), rows, cols, float(threshold), codes.data_ptr(),
                                     row_absmax.data_ptr(), _ptr(outlier_bitmap), _stream_ptr(dev)),
           "llmint8_quantize_rowwise_noalloc")
    return codes, row_absmax, outlier_bitmap


def outlier_bitmap(X, threshold: float, out=None):
    """int32 [ceil(cols/32)]: the outlier columns of fp16 X (all clear for
    threshold <= 0 or no rows). The quantizer computes it; its codes and row
    absmax are dropped."""
    torch = _torch()
    _need_cuda(X, "X", torch.float16)
    if out is None:
        out = torch.empty((X.shape[1] + 31) // 32, dtype=torch.int32, device=X.device)
    return quantize_rowwise(X, threshold, outlier_bitmap=out)[2]


def find_outlier_cols(outlier_bitmap, cols: int, col_idx=None, d_count=None, sync_count: bool = True):
    """(col_idx int32 [cols], d_count int32 [1], host count or None)."""
    torch = _torch()
    dev = outlier_bitmap.device
    if col_idx is None:
        col_idx = torch.empty(cols, dtype=torch.int32, device=dev)
    if d_count is None:
        d_count = torch.empty(1, dtype=torch.int32, device=dev)
    h = ctypes.c_int32(-1)
    _check(load()["_find_outlier_cols"](outlier_bitmap.data_ptr(), cols, col_idx.data_ptr(), d_count.data_ptr(),
                              ctypes.byref(h) if sync_count else None, _stream_ptr(dev)),
           "llmint8_find_outlier_cols")
    return col_idx, d_count, (int(h.value) if sync_count else None)


ACTIVATIONS = {None: 0, "none": 0, "gelu_tanh": 1}


def matmul_mixed(X, CB, SCB, W_f16=None, threshold: float = DEFAULT_THRESHOLD, Y=None, workspace=None,
                 debug: dict | None = None, bias=None, activation=None):
    """Y fp16 [M x N] = LLM.int8()(X fp16 [M x K], W given as CB int8 [N x K] + SCB fp32 [N]).

    ``bias`` (fp16 [N]) and ``activation`` (None or "gelu_tanh") are applied
    in the epilogue before the fp16 rounding (llmint8_matmul_mixed_ex).
    ``debug`` may map any of codes/row_absmax/col_idx/count/acc to CUDA tensors
    the call fills (parity checks), and gemm_begin/gemm_end to recorded
    torch.cuda.Event objects the library re-records around the GEMM launch."""
    torch = _torch()
    _need_cuda(X, "X", torch.float16)
    _need_cuda(CB, "CB", torch.int8)
    _need_cuda(SCB, "SCB", torch.float32)
    if W_f16 is not None:
        _need_cuda(W_f16, "W_f16", torch.float16)
    if bias is not None:
        _need_cuda(bias, "bias", torch.float16)
    if activation not in ACTIVATIONS:
        raise ValueError(f"activation must be one of {sorted(k for k in ACTIVATIONS if k)} or None")
    M, K = X.shape
    N = CB.shape[0]
    dev = X.device
    if Y is None:
        Y = torch.empty((M, N), dtype=torch.float16, device=dev)
    ws = workspace if workspace is not None else get_workspace(workspace_size(M, N, K), dev)
    dbg = None
    if debug:
        dbg = _Debug(*(_ptr(debug.get(k)) for k in ("codes", "row_absmax", "col_idx", "count", "acc")),
                     *(_event(debug.get(k)) for k in ("gemm_begin", "gemm_end")))
    if bias is None and not ACTIVATIONS[activation]:
        _check(load()["_matmul_mixed"](X.data_ptr(), M, K, CB.data_ptr(), SCB.data_ptr(), _ptr(W_f16), N,
                                       float(threshold), Y.data_ptr(), ws.data_ptr(), ws.numel(),
                                       ctypes.byref(dbg) if dbg else None, _stream_ptr(dev)), "llmint8_matmul_mixed")
    else:
        _check(load()["_matmul_mixed_ex"](X.data_ptr(), M, K, CB.data_ptr(), SCB.data_ptr(), _ptr(W_f16), N,
                                          float(threshold), _ptr(bias), ACTIVATIONS[activation], Y.data_ptr(),
                                          ws.data_ptr(), ws.numel(), ctypes.byref(dbg) if dbg else None,
                                          _stream_ptr(dev)), "llmint8_matmul_mixed_ex")
    return Y


def workspace_size_fp16w(M: int, N: int, K: int) -> int:
    return int(load()["_workspace_size_fp16w"](M, N, K))


def matmul_mixed_fp16w(X, W_f16, threshold: float = DEFAULT_THRESHOLD, Y=None, workspace=None,
                       debug: dict | None = None, bias=None, activation=None):
    """The linear with W kept in fp16 and quantized per output row on every
    call ("has fp16 weights" mode): Y fp16 [M x N] from X fp16 [M x K] and
    W_f16 fp16 [N x K]; bias, activation and debug as for matmul_mixed."""
    torch = _torch()
    _need_cuda(X, "X", torch.float16)
    _need_cuda(W_f16, "W_f16", torch.float16)
    if bias is not None:
        _need_cuda(bias, "bias", torch.float16)
    if activation not in ACTIVATIONS:
        raise ValueError(f"activation must be one of {sorted(k for k in ACTIVATIONS if k)} or None")
    M, K = X.shape
    N = W_f16.shape[0]
    dev = X.device
    if Y is None:
        Y = torch.empty((M, N), dtype=torch.float16, device=dev)
    ws = workspace if workspace is not None else get_workspace(workspace_size_fp16w(M, N, K), dev)
    dbg = None
    if debug:
        dbg = _Debug(*(_ptr(debug.get(k)) for k in ("codes", "row_absmax", "col_idx", "count", "acc")),
                     *(_event(debug.get(k)) for k in ("gemm_begin", "gemm_end")))
    _check(load()["_matmul_mixed_fp16w"](X.data_ptr(), M, K, W_f16.data_ptr(), N, float(threshold), _ptr(bias),
                                         ACTIVATIONS[activation], Y.data_ptr(), ws.data_ptr(), ws.numel(),
                                         ctypes.byref(dbg) if dbg else None, _stream_ptr(dev)),
           "llmint8_matmul_mixed_fp16w")
    return Y


def gemm_s8s8s32(A, B, acc=None, workspace=None):
    """int32 [M x N] = A int8 [M x K] . B int8 [N x K]^T."""
    torch = _torch()
    _need_cuda(A, "A", torch.int8)
    _need_cuda(B, "B", torch.int8)
    M, K = A.shape
    N = B.shape[0]
    if acc is None:
        acc = torch.empty((M, N), dtype=torch.int32, device=A.device)
    ws = workspace if workspace is not None else get_workspace(workspace_size(M, N, K), A.device)
    _check(load()["_gemm_s8s8s32"](A.data_ptr(), M, B.data_ptr(), N, K, acc.data_ptr(), ws.data_ptr(), ws.numel(),
                         _stream_ptr(A.device)), "llmint8_gemm_s8s8s32")
    return acc


class Int8MixedLinear:
    """An LLM.int8() linear layer: holds CB/SCB (and optionally the fp16 weight
    for the outlier columns), an optional fp16 bias and an optional activation
    fused after it, and applies matmul_mixed."""

    def __init__(self, CB, SCB, W_f16=None, threshold: float = DEFAULT_THRESHOLD, bias=None, activation=None,
                 has_fp16_weights: bool = False):
        self.CB, self.SCB, self.W_f16, self.threshold = CB, SCB, W_f16, threshold
        self.bias, self.activation = bias, activation
        # True: only W_f16 is kept and quantized on every call (Linear8bitLt's
        # training mode); CB/SCB are then unused.
        self.has_fp16_weights = has_fp16_weights

    @classmethod
    def from_fp16(cls, W, threshold: float = DEFAULT_THRESHOLD, keep_fp16_weights: bool = True, bias=None,
                  activation=None, has_fp16_weights: bool = False):
        """Quantize W fp16 [N x K] per output row (offline weight preparation),
        or, with has_fp16_weights, keep W in fp16 and quantize it per call."""
        if has_fp16_weights:
            return cls(None, None, W, threshold, bias, activation, has_fp16_weights=True)
        CB, SCB, _ = quantize_rowwise(W, 0.0)
        return cls(CB, SCB, W if keep_fp16_weights else None, threshold, bias, activation)

    def __call__(self, X, Y=None):
        if self.has_fp16_weights:
            return matmul_mixed_fp16w(X, self.W_f16, self.threshold, Y=Y, bias=self.bias,
                                      activation=self.activation)
        return matmul_mixed(X, self.CB, self.SCB, self.W_f16, self.threshold, Y=Y, bias=self.bias,
                            activation=self.activation)


# ---- zero-point (unsigned int8) codes for X ------------------------------------------

def quantize_rowwise_asym(X, threshold: float = 0.0, codes=None, scale=None, zero=None, outlier_bitmap=None,
                          workspace=None):
    """(codes int8 = q - 128, scale fp32 [rows], zero int32 [rows], outlier_bitmap or None) of
    fp16 X [rows x cols]: zero-point quantization over the non-outlier columns
    (llmint8_quantize_rowwise_asym)."""
    torch = _torch()
    _need_cuda(X, "X", torch.float16)
    rows, cols = X.shape
    dev = X.device
    if codes is None:
        codes = torch.empty((rows, cols), dtype=torch.int8, device=dev)
    if scale is None:
        scale = torch.empty(rows, dtype=torch.float32, device=dev)
    if zero is None:
        zero = torch.empty(rows, dtype=torch.int32, device=dev)
    if outlier_bitmap is None and threshold > 0:
        outlier_bitmap = torch.empty((cols + 31) // 32, dtype=torch.int32, device=dev)
    ws = workspace if workspace is not None else get_workspace(quantize_workspace_size(rows, cols), dev)
    _check(load()["_quantize_rowwise_asym"](X.data_ptr(), rows, cols, float(threshold), codes.data_ptr(),
                                            scale.data_ptr(), zero.data_ptr(), _ptr(outlier_bitmap), ws.data_ptr(),
                                            ws.numel(), _stream_ptr(dev)), "llmint8_quantize_rowwise_asym")
    return codes, scale, zero, outlier_bitmap


def code_row_sums(CB, out=None):
    """int32 [N]: the sum of each row of the int8 weight codes CB [N x K]."""
    torch = _torch()
    _need_cuda(CB, "CB", torch.int8)
    N, K = CB.shape
    if out is None:
        out = torch.empty(N, dtype=torch.int32, device=CB.device)
    _check(load()["_code_row_sums"](CB.data_ptr(), N, K, out.data_ptr(), _stream_ptr(CB.device)),
           "llmint8_code_row_sums")
    return out


def workspace_size_asym(M: int, N: int, K: int) -> int:
    return int(load()["_workspace_size_asym"](M, N, K))


def matmul_mixed_asym(X, CB, SCB, CB_row_sums, W_f16=None, threshold: float = DEFAULT_THRESHOLD, Y=None,
                      workspace=None, debug: dict | None = None):
    """Y fp16 [M x N] = the LLM.int8() linear with zero-point codes for X
    (llmint8_matmul_mixed_asym). ``CB_row_sums`` from code_row_sums(CB).
    ``debug`` as for matmul_mixed (row_absmax receives the scales s)."""
    torch = _torch()
    _need_cuda(X, "X", torch.float16)
    _need_cuda(CB, "CB", torch.int8)
    _need_cuda(SCB, "SCB", torch.float32)
    _need_cuda(CB_row_sums, "CB_row_sums", torch.int32)
    if W_f16 is not None:
        _need_cuda(W_f16, "W_f16", torch.float16)
    M, K = X.shape
    N = CB.shape[0]
    dev = X.device
    if Y is None:
        Y = torch.empty((M, N), dtype=torch.float16, device=dev)
    ws = workspace if workspace is not None else get_workspace(workspace_size_asym(M, N, K), dev)
    dbg = None
    if debug:
        dbg = _Debug(*(_ptr(debug.get(k)) for k in ("codes", "row_absmax", "col_idx", "count", "acc")),
                     *(_event(debug.get(k)) for k in ("gemm_begin", "gemm_end")))
    _check(load()["_matmul_mixed_asym"](X.data_ptr(), M, K, CB.data_ptr(), SCB.data_ptr(), CB_row_sums.data_ptr(),
                                        _ptr(W_f16), N, float(threshold), Y.data_ptr(), ws.data_ptr(), ws.numel(),
                                        ctypes.byref(dbg) if dbg else None, _stream_ptr(dev)),
           "llmint8_matmul_mixed_asym")
    return Y


# ---- tensor-parallel pieces (page "优化故事：Bloom 推理", section "支持 TP") ----------

def quantize_rowwise_given(X, outlier_bitmaps=None, row_absmax=None, codes=None, row_absmax_out=None,
                           bitmap_out=None):
    """(codes int8 [rows x cols], row absmax fp32 [rows], union bitmap int32 words) of
    fp16 X against a given outlier set: the OR of the bitmaps in
    ``outlier_bitmaps`` (int32 [n, ceil(cols/32)] or [ceil(cols/32)], or None
    for none). With ``row_absmax`` given (fp32 [rows], e.g. all-reduced over a
    row split) the rows are coded with it and it is returned; otherwise the
    absmax over the non-outlier columns is computed
    (llmint8_quantize_rowwise_given)."""
    torch = _torch()
    _need_cuda(X, "X", torch.float16)
    rows, cols = X.shape
    dev = X.device
    nw = (cols + 31) // 32
    nbm = 0
    if outlier_bitmaps is not None:
        _need_cuda(outlier_bitmaps, "outlier_bitmaps", torch.int32)
        if outlier_bitmaps.numel() % nw:
            raise ValueError("outlier_bitmaps must hold whole bitmaps of ceil(cols/32) words")
        nbm = outlier_bitmaps.numel() // nw
    if row_absmax is not None:
        _need_cuda(row_absmax, "row_absmax", torch.float32)
    if codes is None:
        codes = torch.empty((rows, cols), dtype=torch.int8, device=dev)
    if row_absmax is None and row_absmax_out is None:
        row_absmax_out = torch.empty(rows, dtype=torch.float32, device=dev)
    if bitmap_out is None:
        bitmap_out = torch.empty(nw, dtype=torch.int32, device=dev)
    _check(load()["_quantize_rowwise_given"](X.data_ptr(), rows, cols, _ptr(outlier_bitmaps), nbm, _ptr(row_absmax),
                                             codes.data_ptr(), _ptr(row_absmax_out), bitmap_out.data_ptr(),
                                             _stream_ptr(dev)), "llmint8_quantize_rowwise_given")
    return codes, (row_absmax if row_absmax is not None else row_absmax_out), bitmap_out


def matmul_codes(CX, SX, X, CB, SCB, col_idx, d_count, W_f16=None, bias=None, activation=None, out_f32=False,
                 Y=None, workspace=None):
    """Y [M x N] (fp16, or fp32 with ``out_f32``) = the LLM.int8() GEMM and
    epilogue on codes quantized beforehand: CX int8 [M x K], SX fp32 [M], X
    fp16 [M x K] (outlier values), CB/SCB/W_f16 as matmul_mixed, the outlier
    columns in col_idx int32 [K] / d_count int32 [1] (llmint8_matmul_codes)."""
    torch = _torch()
    _need_cuda(CX, "CX", torch.int8)
    _need_cuda(SX, "SX", torch.float32)
    _need_cuda(X, "X", torch.float16)
    _need_cuda(CB, "CB", torch.int8)
    _need_cuda(SCB, "SCB", torch.float32)
    _need_cuda(col_idx, "col_idx", torch.int32)
    _need_cuda(d_count, "d_count", torch.int32)
    if W_f16 is not None:
        _need_cuda(W_f16, "W_f16", torch.float16)
    if bias is not None:
        _need_cuda(bias, "bias", torch.float16)
    if activation not in ACTIVATIONS:
        raise ValueError(f"activation must be one of {sorted(k for k in ACTIVATIONS if k)} or None")
    M, K = CX.shape
    N = CB.shape[0]
    dev = CX.device
    if Y is None:
        Y = torch.empty((M, N), dtype=torch.float32 if out_f32 else torch.float16, device=dev)
    ws = workspace if workspace is not None else get_workspace(4096, dev)
    _check(load()["_matmul_codes"](CX.data_ptr(), SX.data_ptr(), X.data_ptr(), M, K, CB.data_ptr(), SCB.data_ptr(),
                                   _ptr(W_f16), N, col_idx.data_ptr(), d_count.data_ptr(), _ptr(bias),
                                   ACTIVATIONS[activation], OUT_F32 if out_f32 else OUT_F16, Y.data_ptr(),
                                   ws.data_ptr(), ws.numel(), _stream_ptr(dev)), "llmint8_matmul_codes")
    return Y


def bias_act_to_f16(Y32, bias=None, activation=None, Y=None):
    """fp16 act(Y32 + bias) of an fp32 [M x N] sum (llmint8_bias_act_to_f16)."""
    torch = _torch()
    _need_cuda(Y32, "Y32", torch.float32)
    if bias is not None:
        _need_cuda(bias, "bias", torch.float16)
    M, N = Y32.shape
    if Y is None:
        Y = torch.empty((M, N), dtype=torch.float16, device=Y32.device)
    _check(load()["_bias_act_to_f16"](Y32.data_ptr(), M, N, _ptr(bias), ACTIVATIONS[activation], Y.data_ptr(),
                                      _stream_ptr(Y32.device)), "llmint8_bias_act_to_f16")
    return Y


def gather_column_blocks(blocks, out=None):
    """fp16 [M x P*Nr] from column blocks fp16 [P, M, Nr] (llmint8_gather_column_blocks)."""
    torch = _torch()
    _need_cuda(blocks, "blocks", torch.float16)
    P, M, Nr = blocks.shape
    if out is None:
        out = torch.empty((M, P * Nr), dtype=torch.float16, device=blocks.device)
    _check(load()["_gather_column_blocks"](blocks.data_ptr(), P, M, Nr, out.data_ptr(), _stream_ptr(blocks.device)),
           "llmint8_gather_column_blocks")
    return out
