"""GPU parity of the zero-point (unsigned int8) variant: codes, scales, zero
points, outlier bitmaps and int32 products bit-exact against the oracle; the
fp16 output within 1e-2 + 2e-3 |y|."""
import numpy as np
import pytest
import torch

from synthetic import Linear, make_activations, make_random, make_weight

pytestmark = pytest.mark.gpu

ATOL, RTOL = 1e-2, 2e-3


@pytest.fixture(scope="module")
def lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import int8_mixed_precision_rowwise_b200 as m
    return m


@pytest.fixture(scope="module")
def dev(lib):
    return torch.device("cuda", 0)


def to_dev(a, dev):
    return torch.from_numpy(np.ascontiguousarray(a)).to(dev)


def bitmap_to_mask(words: np.ndarray, cols: int) -> np.ndarray:
    bits = np.unpackbits(words.astype("<u4").view(np.uint8), bitorder="little")
    return bits[:cols].astype(np.uint8)


@pytest.mark.parametrize("M,K,nout,t", [(8, 64, 2, 6.0), (300, 1024, 5, 6.0), (300, 1024, 5, 0.0),
                                        (4096, 4096, 8, 6.0), (2048, 14336, 7, 6.0), (3, 16, 1, 6.0)])
def test_quantize_asym_matches_oracle(lib, dev, oracle_mod, M, K, nout, t):
    lin = Linear("a", M, 1, K, nout, 40.0)
    X16, _ = make_activations(lin, seed=M + K)
    X16[M // 2] += np.float16(0.75)  # a row whose range is not symmetric about 0
    if M > 3:
        X16[1] = 0                   # an all-zero row
    # A row on [-1, 1] reaching both ends: s = 127.5, z = 128 and the code of
    # 1.0 lands on 256 before the clamp (the oracle counts it below).
    # (Its values stay below t, so the outlier columns do not change; its two
    # ends go to columns outside them.)
    crow = M - 1
    X16[crow] = np.clip(X16[crow], -1, 1)
    mask = oracle_mod.outlier_mask(X16, t) if t > 0 else np.zeros(K, np.uint8)
    c_lo, c_hi = np.flatnonzero(mask == 0)[[0, -1]]
    X16[crow, c_lo], X16[crow, c_hi] = -1.0, 1.0
    codes, scale, zero, bm = lib.quantize_rowwise_asym(to_dev(X16, dev), t)
    c_ref, s_ref, z_ref, clamped = oracle_mod.quantize_rowwise_asym(X16, mask, return_clamped=True)
    assert clamped >= 1 and c_ref[crow, c_hi] == 127 and z_ref[crow] == 128
    if t > 0:
        assert np.array_equal(bitmap_to_mask(bm.cpu().numpy(), K), mask)
    assert np.array_equal(scale.cpu().numpy().view(np.uint32), s_ref.view(np.uint32))
    assert np.array_equal(zero.cpu().numpy(), z_ref)
    assert np.array_equal(codes.cpu().numpy(), c_ref)


@pytest.mark.parametrize("M,K,rows_hit", [(4096, 4096, [4095]), (1000, 2064, [0, 999]), (150, 4096, [149])])
def test_quantize_asym_resident_stale_rows(lib, dev, oracle_mod, M, K, rows_hit):
    """Shapes that fit the shared-memory quantizer (detection and zero-point
    codes in one kernel): two outlier columns that only a few rows cross,
    while other rows take their maximum (column 37) or their minimum (column
    38) in them. Rows coded before the columns were known are coded again
    against the complete set: codes, scales and zero points are still the
    definition's."""
    X = np.random.default_rng(13).standard_normal((M, K)).astype(np.float32)
    X[:, 37] *= 0.1
    X[:, 37] += 5.5 * (np.arange(M) % 3 == 0)
    X[:, 38] *= 0.1
    X[:, 38] -= 5.5 * (np.arange(M) % 5 == 0)
    for r in rows_hit:
        X[r, 37], X[r, 38] = 50.0, -50.0
    X16 = X.astype(np.float16)
    codes, scale, zero, bm = lib.quantize_rowwise_asym(to_dev(X16, dev), 6.0)
    mask = oracle_mod.outlier_mask(X16, 6.0)
    assert mask[37] and mask[38]
    c_ref, s_ref, z_ref = oracle_mod.quantize_rowwise_asym(X16, mask)
    assert np.array_equal(bitmap_to_mask(bm.cpu().numpy(), K), mask)
    assert np.array_equal(scale.cpu().numpy().view(np.uint32), s_ref.view(np.uint32))
    assert np.array_equal(zero.cpu().numpy(), z_ref)
    assert np.array_equal(codes.cpu().numpy(), c_ref)


def test_code_row_sums_exact(lib, dev, oracle_mod):
    rng = np.random.default_rng(2)
    CB = rng.integers(-127, 128, size=(1000, 4096), dtype=np.int8)
    CB[3] = 127
    CB[4] = -127
    R = lib.code_row_sums(to_dev(CB, dev)).cpu().numpy()
    assert np.array_equal(R.astype(np.int64), oracle_mod.code_row_sums(CB))


@pytest.mark.parametrize("M,N,K,nout,give_w16", [
    (333, 777, 1024, 5, True), (333, 777, 1024, 5, False), (100, 700, 1024, 8, False),
    (16, 640, 1024, 6, True), (32, 300, 512, 3, False), (1024, 8192, 256, 6, True), (200, 384, 80, 2, True),
    # 150 tiles of 256 x 256 on 74 CTA pairs: the last tiles run stream-K
    (300, 19000, 384, 5, True)])
def test_matmul_asym_matches_oracle(lib, dev, oracle_mod, M, N, K, nout, give_w16):
    lin = Linear("a", M, N, K, nout, 60.0)
    X16, _ = make_activations(lin, seed=M + N)
    X16[0] += np.float16(1.5)  # asymmetric range
    W16 = make_weight(lin, seed=K)
    X, W = to_dev(X16, dev), to_dev(W16, dev)
    CB, SCB, _ = lib.quantize_rowwise(W, 0.0)
    R = lib.code_row_sums(CB)
    dbg = dict(codes=torch.empty((M, K), dtype=torch.int8, device=dev),
               row_absmax=torch.empty(M, dtype=torch.float32, device=dev),
               col_idx=torch.empty(K, dtype=torch.int32, device=dev),
               count=torch.empty(1, dtype=torch.int32, device=dev),
               acc=torch.empty((M, N), dtype=torch.int32, device=dev))
    Y = lib.matmul_mixed_asym(X, CB, SCB, R, W if give_w16 else None, 6.0, debug=dbg)
    torch.cuda.synchronize()
    r = oracle_mod.matmul_mixed_asym(X16, 6.0, W=W16, use_fp16_weight_cols=give_w16)
    n = int(dbg["count"].item())
    assert np.array_equal(dbg["col_idx"][:n].cpu().numpy(), r["O"])
    assert np.array_equal(CB.cpu().numpy(), r["CB"])
    assert np.array_equal(dbg["codes"].cpu().numpy(), r["CX"])
    assert np.array_equal(dbg["row_absmax"].cpu().numpy().view(np.uint32), r["SXs"].view(np.uint32))
    assert np.array_equal(dbg["acc"].cpu().numpy(), r["acc"])
    y = Y.cpu().numpy().astype(np.float64)
    err = np.abs(y - r["Y"])
    assert np.all(err <= ATOL + RTOL * np.abs(r["Y"])), f"worst {err.max():.4g}"


def test_matmul_asym_without_threshold_and_zero_rows(lib, dev, oracle_mod):
    X16 = make_random((300, 512), seed=9)
    X16[7] = 0
    X16[8] = np.abs(X16[8])
    W16 = make_random((256, 512), seed=10, scale=0.02)
    X, W = to_dev(X16, dev), to_dev(W16, dev)
    CB, SCB, _ = lib.quantize_rowwise(W, 0.0)
    Y = lib.matmul_mixed_asym(X, CB, SCB, lib.code_row_sums(CB), None, 0.0)
    torch.cuda.synchronize()
    r = oracle_mod.matmul_mixed_asym(X16, 0.0, W=W16, use_fp16_weight_cols=False)
    y = Y.cpu().numpy().astype(np.float64)
    assert np.all(np.abs(y - r["Y"]) <= ATOL + RTOL * np.abs(r["Y"]))
    assert not y[7].any()
