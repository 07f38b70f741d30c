"""The allocation-free quantizer entry point, llmint8_quantize_rowwise_noalloc.

It serves callers that cannot allocate device memory (a server whose memory
pool owns the whole GPU, a plugin barred from allocating after start-up, a
loop that cannot afford an allocation's synchronisation): its scratch is a
fixed array inside the library instead of a caller workspace. These tests
call it through the C ABI and compare it with llmint8_quantize_rowwise, the
entry point that takes a workspace, and with the oracle, on several calls in a
row; codes, row absmax bits and outlier bitmap must match exactly, as
everywhere else in the tests. The array's status word, read through
llmint8_noalloc_read_status, must stay clear.
This file is collected last so that a run stopping at the first failure has
already run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

from synthetic import Linear, make_activations


def _noalloc_fn(lib_path):
    cdll = ctypes.CDLL(lib_path)
    f = cdll.llmint8_quantize_rowwise_noalloc
    f.restype = ctypes.c_int
    f.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64, ctypes.c_float, ctypes.c_void_p,
                  ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]
    return f


def _status_fn(lib_path):
    cdll = ctypes.CDLL(lib_path)
    f = cdll.llmint8_noalloc_read_status
    f.restype = ctypes.c_int
    f.argtypes = [ctypes.c_int, ctypes.POINTER(ctypes.c_uint32)]
    return f


def test_noalloc_rejects_sizes_beyond_its_scratch():
    """Sizes past the fixed array are refused before any GPU work (no GPU needed)."""
    import int8_mixed_precision_rowwise_b200 as L
    f = _noalloc_fn(L.LIB_PATH)
    A = 0x10000
    assert f(A, 65537, 1024, 6.0, A, A, A, None) == L.ERR_UNSUPPORTED_SHAPE
    assert f(A, 16, 65536 + 16, 6.0, A, A, A, None) == L.ERR_UNSUPPORTED_SHAPE
    assert f(A, 16, 1000, 6.0, A, A, A, None) == L.ERR_UNSUPPORTED_SHAPE   # cols % 16
    assert f(A, 16, 1024, 6.0, A, A, None, None) == L.ERR_INVALID_ARG      # bitmap needed for t > 0
    assert f(A, 0, 1024, 0.0, A, A, None, None) == L.OK                    # empty, no bitmap: nothing queued
    assert _status_fn(L.LIB_PATH)(0, None) == L.ERR_INVALID_ARG             # status reader needs `out`


def _bitmap_to_mask(words: np.ndarray, cols: int) -> np.ndarray:
    bits = np.unpackbits(words.astype("<u4").view(np.uint8), bitorder="little")
    return bits[:cols].astype(np.uint8)


@pytest.mark.gpu
def test_noalloc_matches_workspace_entry_point_and_oracle(oracle_mod):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import int8_mixed_precision_rowwise_b200 as L
    f = _noalloc_fn(L.LIB_PATH)
    dev = torch.device("cuda", 0)
    stream = torch.cuda.current_stream(dev).cuda_stream
    assert L.noalloc_read_status(clear=True) == 0
    # Calls in a row; each follows a different shape, so stale scratch from
    # the call before (outlier list, count, barrier words) would show up in
    # its result. 700 x 4096 and 333 x 1024 run the whole CTA on each row,
    # 4096 x 4096 one warp per row (rows >= 8 per SM); t = 0 passes no bitmap.
    cases = [(700, 4096, 8, 1, 6.0), (333, 1024, 5, 2, 6.0), (4096, 4096, 8, 3, 6.0), (512, 2048, 4, 4, 0.0)]
    for M, K, n_out, seed, t in cases:
        X16, _ = make_activations(Linear("q", M, 0, K, n_out, 40.0), seed=seed)
        X = torch.from_numpy(X16).to(dev)
        ref_codes, ref_absmax, ref_bm = L.quantize_rowwise(X, t)
        codes = torch.empty((M, K), dtype=torch.int8, device=dev)
        absmax = torch.empty(M, dtype=torch.float32, device=dev)
        bm = torch.full(((K + 31) // 32,), -1, dtype=torch.int32, device=dev) if t > 0 else None
        st = f(X.data_ptr(), M, K, t, codes.data_ptr(), absmax.data_ptr(), bm.data_ptr() if bm is not None else None,
               stream)
        assert st == L.OK, L.status_string(st)
        torch.cuda.synchronize()
        # the same results as the entry point that takes a workspace ...
        assert torch.equal(codes, ref_codes)
        assert np.array_equal(absmax.cpu().numpy().view(np.uint32), ref_absmax.cpu().numpy().view(np.uint32))
        # ... and as the oracle
        mask = oracle_mod.outlier_mask(X16, t)
        c_ref, a_ref = oracle_mod.quantize_rowwise(X16, mask if t > 0 else None)
        assert np.array_equal(codes.cpu().numpy(), c_ref)
        assert np.array_equal(absmax.cpu().numpy().view(np.uint32), a_ref.view(np.uint32))
        if t > 0:
            assert torch.equal(bm, ref_bm)
            assert np.array_equal(_bitmap_to_mask(bm.cpu().numpy(), K), mask)
            assert int(bm.ne(0).sum()) > 0  # the outlier columns were found
    # no call gave up on a bounded wait
    out = ctypes.c_uint32(7)
    assert _status_fn(L.LIB_PATH)(1, ctypes.byref(out)) == L.OK and out.value == 0
