"""GPU parity: the CUDA path through the C-ABI against the CPU oracle.

Bar (the pages' definition, see the oracle): int8 codes, row absmax (as fp32
bits), the outlier column set and the int32 accumulators are bit-exact; the
fp16 output satisfies |y - y_ref| <= 1e-2 + 2e-3 |y_ref| elementwise, with
y_ref the oracle's fp64 value.

Sizes here span several 128x256 output tiles with ragged edges in M, N and
K, so the oracle finishes in seconds. The full-size workloads (prefill,
decode and the four BLOOM block linears) are compared in full too: codes,
row absmax, outlier set and weight codes against the oracle, the int32
accumulators against the oracle's product (decode; prefill under the `slow`
mark) or cuBLAS's on the oracle's codes, and every fp16 output against the
oracle's output step on those accumulators.
"""
import numpy as np
import pytest
import torch

import synthetic
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


def assert_y_close(y_gpu: np.ndarray, y_ref: np.ndarray, what=""):
    y = y_gpu.astype(np.float64)
    err = np.abs(y - y_ref)
    tol = ATOL + RTOL * np.abs(y_ref)
    bad = err > tol
    assert not bad.any(), (f"{what}: {bad.sum()} of {bad.size} outside tolerance; worst err "
                           f"{err.max():.4g} at {np.unravel_index(np.argmax(err - tol), err.shape)}")


def gpu_mixed(lib, dev, X16, W16, t, give_w16=True, with_debug=True):
    X = to_dev(X16, dev)
    W = to_dev(W16, dev)
    CB, SCB, _ = lib.quantize_rowwise(W, 0.0)
    M, K = X16.shape
    N = W16.shape[0]
    dbg = None
    if with_debug:
        dbg = dict(codes=torch.empty((M, K), dtype=torch.int8, device=dev),
                   row_absmax=torch.empty(M, dtype=torch.float32, device=dev),
                   col_idx=torch.full((K,), -1, dtype=torch.int32, device=dev),
                   count=torch.empty(1, dtype=torch.int32, device=dev),
                   acc=torch.empty((M, N), dtype=torch.int32, device=dev))
    Y = lib.matmul_mixed(X, CB, SCB, W if give_w16 else None, t, debug=dbg)
    torch.cuda.synchronize()
    out = dict(Y=Y.cpu().numpy(), CB=CB.cpu().numpy(), SB=SCB.cpu().numpy())
    if dbg:
        n = int(dbg["count"].item())
        out.update(CX=dbg["codes"].cpu().numpy(), SX=dbg["row_absmax"].cpu().numpy(),
                   O=dbg["col_idx"][:n].cpu().numpy().astype(np.int64), acc=dbg["acc"].cpu().numpy())
    return out


def check_full(lib, dev, oracle_mod, X16, W16, t, give_w16=True):
    g = gpu_mixed(lib, dev, X16, W16, t, give_w16)
    r = oracle_mod.matmul_mixed(X16, t, W=W16, use_fp16_weight_cols=give_w16)
    assert np.array_equal(g["CB"], r["CB"]), "weight codes"
    assert np.array_equal(g["SB"].view(np.uint32), r["SB"].view(np.uint32)), "weight absmax bits"
    assert np.array_equal(g["O"], r["O"]), f"outlier columns {g['O']} vs {r['O']}"
    assert np.array_equal(g["SX"].view(np.uint32), r["SX"].view(np.uint32)), "row absmax bits"
    assert np.array_equal(g["CX"], r["CX"]), "activation codes"
    assert np.array_equal(g["acc"], r["acc"]), "int32 accumulators"
    assert_y_close(g["Y"], r["Y"], "Y")
    return g, r


# ------------------------------------------------------------------ quantizer

@pytest.mark.parametrize("M,K,nout,scale", [(8, 64, 2, 20.0), (300, 1024, 5, 40.0), (513, 4096, 8, 40.0),
                                            (64, 14336, 6, 60.0), (9, 57344, 29, 60.0), (3, 16, 1, 60.0),
                                            # too large for shared memory: the streaming quantizer
                                            (6000, 4096, 8, 40.0), (1500, 12288, 6, 40.0)])
def test_quantize_rowwise_matches_oracle(lib, dev, oracle_mod, M, K, nout, scale):
    X16, _ = make_activations(Linear("q", M, 0, K, nout, scale), seed=M + K)
    codes, absmax, bm = lib.quantize_rowwise(to_dev(X16, dev), 6.0)
    mask = oracle_mod.outlier_mask(X16, 6.0)
    c_ref, a_ref = oracle_mod.quantize_rowwise(X16, mask)
    assert np.array_equal(bitmap_to_mask(bm.cpu().numpy(), K), mask)
    assert np.array_equal(absmax.cpu().numpy().view(np.uint32), a_ref.view(np.uint32))
    assert np.array_equal(codes.cpu().numpy(), c_ref)


def test_quantizer_workload_full(lib, dev, oracle_mod):
    """The 4096 x 4096 quantizer workload (8 columns x40), compared in full."""
    lin = synthetic.QUANT_4096.linears[0]
    X16, cols = make_activations(lin, seed=0)
    codes, absmax, bm = lib.quantize_rowwise(to_dev(X16, dev), 6.0)
    mask = oracle_mod.outlier_mask(X16, 6.0)
    assert set(cols.tolist()) <= set(np.flatnonzero(mask).tolist())
    c_ref, a_ref = oracle_mod.quantize_rowwise(X16, mask)
    assert np.array_equal(bitmap_to_mask(bm.cpu().numpy(), lin.K), mask)
    assert np.array_equal(absmax.cpu().numpy().view(np.uint32), a_ref.view(np.uint32))
    assert np.array_equal(codes.cpu().numpy(), c_ref)


def test_quantize_threshold_off_is_plain_absmax(lib, dev, oracle_mod):
    W16 = make_random((777, 1024), seed=7, scale=0.02)
    codes, absmax, bm = lib.quantize_rowwise(to_dev(W16, dev), 0.0)
    c_ref, a_ref = oracle_mod.quantize_rowwise(W16, None)
    assert bm is None
    assert np.array_equal(absmax.cpu().numpy().view(np.uint32), a_ref.view(np.uint32))
    assert np.array_equal(codes.cpu().numpy(), c_ref)


def test_quantize_worked_example(lib, dev):
    """The pages' absmax example (padded to 16 columns with zeros)."""
    x = np.zeros((1, 16), dtype=np.float16)
    x[0, :8] = [1.2, -0.5, -4.3, 1.2, -3.1, 0.8, 2.4, 5.4]
    codes, absmax, _ = lib.quantize_rowwise(to_dev(x, dev), 0.0)
    assert codes.cpu().numpy()[0, :8].tolist() == [28, -12, -101, 28, -73, 19, 56, 127]


def test_quantize_edge_rows(lib, dev, oracle_mod):
    """Zero rows, exact-threshold values, .5 ties, values just below the
    threshold, and rows whose maximum sits in a column that is an outlier only
    because of another row (the fix-up path)."""
    rng = np.random.default_rng(5)
    X = rng.standard_normal((200, 256)).astype(np.float32)
    X[3] = 0.0
    X[5, 10] = 6.0                       # exactly the threshold: outlier column 10
    X[6] = 0.0
    X[6, :3] = [127.0, 2.5, 3.5]         # ties: s = 1
    X[:, 40] *= 0.1
    X[7, 40] = 50.0                      # column 40 outlier because of row 7 ...
    X[8:100, 40] = 5.5                   # ... and the maximum of rows 8..99 sits there
    X[150:, 77] = 5.9                    # column 77 never reaches 6: it stays in the int8 part
    X16 = X.astype(np.float16)
    codes, absmax, bm = lib.quantize_rowwise(to_dev(X16, dev), 6.0)
    mask = oracle_mod.outlier_mask(X16, 6.0)
    c_ref, a_ref = oracle_mod.quantize_rowwise(X16, mask)
    assert mask[10] and mask[40] and not mask[77]
    assert np.array_equal(bitmap_to_mask(bm.cpu().numpy(), 256), mask)
    assert np.array_equal(absmax.cpu().numpy().view(np.uint32), a_ref.view(np.uint32))
    assert np.array_equal(codes.cpu().numpy(), c_ref)


@pytest.mark.parametrize("M,K,late_row,from_row", [
    (8192, 4096, 8100, 7000),    # a warp per row
    (2048, 14336, 2000, 1500),   # the CTA per row, 7 vectors a thread (BLOOM's hidden width)
    (1024, 57344, 1000, 700),    # the CTA per row, 32 vectors a thread (BLOOM's fc2 input)
])
def test_quantize_late_outlier_column(lib, dev, oracle_mod, M, K, late_row, from_row):
    """Shapes too large for the shared-memory quantizer, so the streaming one
    with its seed runs: the seed reads each group's first row only, so a
    column that crosses the threshold only in row `late_row` is found late,
    while rows from `from_row` on already took their maximum (5.5) in it. The
    result must still be the definition's (every row re-quantized against the
    final set)."""
    X = np.random.default_rng(8).standard_normal((M, K)).astype(np.float32)
    X[:, 100] *= 0.1
    X[from_row:, 100] = 5.5
    X[late_row, 100] = 50.0
    X16 = X.astype(np.float16)
    codes, absmax, bm = lib.quantize_rowwise(to_dev(X16, dev), 6.0)
    mask = oracle_mod.outlier_mask(X16, 6.0)
    assert mask[100]
    c_ref, a_ref = oracle_mod.quantize_rowwise(X16, mask)
    assert np.array_equal(bitmap_to_mask(bm.cpu().numpy(), K), mask)
    assert np.array_equal(absmax.cpu().numpy().view(np.uint32), a_ref.view(np.uint32))
    assert np.array_equal(codes.cpu().numpy(), c_ref)


@pytest.mark.parametrize("M,K,rows_hit", [
    (4096, 4096, [4095]),        # only the last chunk of the last CTA sees it
    (4096, 4096, [7 * 28 + 5]),  # mid-block of one CTA: its earlier chunks and every other CTA are stale
    (1000, 2064, [0, 999]),      # ragged rows per CTA, a partial bitmap word
    (150, 4096, [149]),          # about one row per CTA
])
def test_quantize_resident_stale_chunks(lib, dev, oracle_mod, M, K, rows_hit):
    """Shapes that fit the shared-memory quantizer, with an outlier column
    that only a few rows cross (the other rows take their maximum, 5.5, in
    it). Chunks quantized before the column was known must be quantized again
    against the complete set: the result is still the definition's."""
    X = np.random.default_rng(11).standard_normal((M, K)).astype(np.float32)
    X[:, 37] *= 0.1
    X[:, 37] += 5.5 * (np.arange(M) % 3 == 0)
    for r in rows_hit:
        X[r, 37] = 40.0
    X[:, 1000 % K] *= 30.0  # a column every chunk sees
    X16 = X.astype(np.float16)
    codes, absmax, bm = lib.quantize_rowwise(to_dev(X16, dev), 6.0)
    mask = oracle_mod.outlier_mask(X16, 6.0)
    assert mask[37]
    c_ref, a_ref = oracle_mod.quantize_rowwise(X16, mask)
    assert np.array_equal(bitmap_to_mask(bm.cpu().numpy(), K), mask)
    assert np.array_equal(absmax.cpu().numpy().view(np.uint32), a_ref.view(np.uint32))
    assert np.array_equal(codes.cpu().numpy(), c_ref)


@pytest.mark.parametrize("M,K", [(5000, 16), (777, 32), (40, 48), (3, 57344), (148 * 13, 4112)])
def test_quantize_resident_odd_shapes(lib, dev, oracle_mod, M, K):
    """Narrow rows (a vector or two per row, many rows per chunk), a few very
    long rows, and a ragged width, with and without the threshold."""
    X16 = make_random((M, K), seed=M + K, scale=2.0)
    X16[M // 2, K - 1] = 9.0
    for t in (6.0, 0.0):
        codes, absmax, bm = lib.quantize_rowwise(to_dev(X16, dev), t)
        mask = oracle_mod.outlier_mask(X16, t) if t > 0 else np.zeros(K, np.uint8)
        c_ref, a_ref = oracle_mod.quantize_rowwise(X16, mask)
        if t > 0:
            assert np.array_equal(bitmap_to_mask(bm.cpu().numpy(), K), mask)
        assert np.array_equal(absmax.cpu().numpy().view(np.uint32), a_ref.view(np.uint32))
        assert np.array_equal(codes.cpu().numpy(), c_ref)


def test_workspace_shared_across_shapes(lib, dev, oracle_mod):
    """One workspace for calls of several shapes and entry points, in an order
    that leaves other regions' data (codes, column lists) where a later shape
    keeps its outlier bookkeeping: every result is still the definition's."""
    shapes = [(64, 4096), (300, 1040), (2000, 256), (64, 4096), (1000, 2064), (4096, 4096), (64, 4096)]
    nbytes = max(max(lib.workspace_size(M, 512, K), lib.quantize_workspace_size(M, K)) for M, K in shapes)
    ws = torch.empty(nbytes, dtype=torch.uint8, device=dev)
    lib.workspace_init(ws)
    for i, (M, K) in enumerate(shapes):
        lin = Linear("ws", M, 512, K, 3 + i % 3, 50.0)
        X16, _ = make_activations(lin, seed=100 + i)
        X = to_dev(X16, dev)
        mask = oracle_mod.outlier_mask(X16, 6.0)
        c_ref, a_ref = oracle_mod.quantize_rowwise(X16, mask)
        codes, absmax, bm = lib.quantize_rowwise(X, 6.0, workspace=ws)
        assert np.array_equal(bitmap_to_mask(bm.cpu().numpy(), K), mask), (M, K)
        assert np.array_equal(absmax.cpu().numpy().view(np.uint32), a_ref.view(np.uint32)), (M, K)
        assert np.array_equal(codes.cpu().numpy(), c_ref), (M, K)
        if M <= 2000:  # and a matmul on the same workspace, its codes checked through the debug outputs
            W16 = make_weight(lin, seed=i)
            W = to_dev(W16, dev)
            CB, SCB, _ = lib.quantize_rowwise(W, 0.0, workspace=ws)
            dbg = dict(codes=torch.empty((M, K), dtype=torch.int8, device=dev),
                       row_absmax=torch.empty(M, dtype=torch.float32, device=dev),
                       col_idx=torch.empty(K, dtype=torch.int32, device=dev),
                       count=torch.empty(1, dtype=torch.int32, device=dev))
            lib.matmul_mixed(X, CB, SCB, W, 6.0, workspace=ws, debug=dbg)
            n = int(dbg["count"].item())
            assert np.array_equal(dbg["col_idx"][:n].cpu().numpy(), np.flatnonzero(mask)), (M, K)
            assert np.array_equal(dbg["codes"].cpu().numpy(), c_ref), (M, K)


def test_quantize_row_of_outliers(lib, dev, oracle_mod):
    """One row >= t everywhere makes every column an outlier: all codes 0,
    every absmax 0 (the int8 part is empty)."""
    X16 = make_random((40, 64), seed=6)
    X16[2] = 7.0
    codes, absmax, bm = lib.quantize_rowwise(to_dev(X16, dev), 6.0)
    assert np.array_equal(bitmap_to_mask(bm.cpu().numpy(), 64), np.ones(64, np.uint8))
    assert not codes.cpu().numpy().any() and not absmax.cpu().numpy().any()


def test_find_outlier_cols(lib, dev):
    K = 14336
    rng = np.random.default_rng(9)
    for n in (0, 1, 29, 700):
        cols = np.sort(rng.choice(K, n, replace=False))
        mask = np.zeros(K, dtype=np.uint8)
        mask[cols] = 1
        words = np.packbits(mask, bitorder="little").view("<u4").astype(np.int32)
        col_idx, d_count, h = lib.find_outlier_cols(to_dev(words, dev), K)
        assert h == n and int(d_count.item()) == n
        assert np.array_equal(col_idx[:n].cpu().numpy(), cols)


# ------------------------------------------------------------------ int8 GEMM

@pytest.mark.parametrize("M,N,K", [(1, 300, 512), (8, 200, 256), (17, 129, 1040), (32, 136, 768),
                                   (33, 257, 1024), (300, 520, 1040), (128, 256, 128), (257, 513, 80),
                                   (64, 64, 16)])
def test_gemm_s8s8s32_exact(lib, dev, oracle_mod, M, N, K):
    rng = np.random.default_rng(M * 7 + N)
    A = rng.integers(-127, 128, size=(M, K), dtype=np.int8)
    B = rng.integers(-127, 128, size=(N, K), dtype=np.int8)
    acc = lib.gemm_s8s8s32(to_dev(A, dev), to_dev(B, dev))
    assert np.array_equal(acc.cpu().numpy(), oracle_mod.int8_matmul(A, B))


def test_gemm_int32_margin(lib, dev):
    """K = 57344 with every code at +-127: the sums reach 924,901,376 exactly."""
    K = 57344
    A = np.full((40, K), 127, dtype=np.int8)
    A[1::2] = -127
    B = np.full((24, K), 127, dtype=np.int8)
    B[::3] = -127
    acc = lib.gemm_s8s8s32(to_dev(A, dev), to_dev(B, dev)).cpu().numpy()
    ref = (np.where(np.arange(40) % 2, -1, 1)[:, None] * np.where(np.arange(24) % 3 == 0, -1, 1)[None, :]
           * K * 127 * 127)
    assert np.array_equal(acc.astype(np.int64), ref)


def test_gemm_matches_torch_int_mm(lib, dev):
    """An independent library check of the int32 product at a tile-spanning size."""
    rng = np.random.default_rng(1)
    A = torch.from_numpy(rng.integers(-127, 128, size=(512, 2048), dtype=np.int8)).to(dev)
    B = torch.from_numpy(rng.integers(-127, 128, size=(768, 2048), dtype=np.int8)).to(dev)
    acc = lib.gemm_s8s8s32(A, B)
    ref = torch._int_mm(A, B.t().contiguous())
    assert torch.equal(acc, ref)


# Stream-K: on a GPU with P = SMs / 2 CTA pairs, a prefill GEMM (M >= 256)
# whose 256 x 256 tiles number more than P and not a multiple of P, with at
# least two K stages (256 bytes of K) a tile, splits its last tiles over the
# pairs by K stages when that beats every whole-tile width (charging the
# split 2%). These shapes take that path on a 148-SM B200; the parked partial
# sums must add up to the same int32 products bit for bit.
def _takes_stream_k(M, N, K, sms):
    P = sms // 2
    m_blk = (M + 255) // 256
    best = None
    for bn, eff in ((256, 1000), (224, 946), (192, 920), (128, 950)):
        tiles = m_blk * ((N + bn - 1) // bn)
        pairs = min(tiles, P)
        cost = (tiles + pairs - 1) // pairs * bn * 1000000 // eff
        best = cost if best is None else min(best, cost)
    tiles = m_blk * ((N + 255) // 256)
    stages = ((K + 127) // 128 + 1) // 2
    return tiles > P and tiles % P != 0 and stages >= 2 and tiles * 256 * 1020 // P < best


STREAM_K_SHAPES = [(512, 10240, 4096), (300, 19000, 384), (256, 20480, 1152), (2048, 14336, 4224)]


@pytest.mark.parametrize("M,N,K", STREAM_K_SHAPES)
def test_gemm_stream_k_exact(lib, dev, M, N, K):
    """The int32 product on the stream-K path (ragged M, N and last K stage
    among the shapes) against torch._int_mm (cuBLAS), twice on one workspace
    (the stream-K flags must be back at zero after a call) and once more from
    a CUDA-graph replay."""
    if torch.cuda.get_device_properties(dev).multi_processor_count == 148:
        assert _takes_stream_k(M, N, K, 148)
    rng = np.random.default_rng(M + N + K)
    A = torch.from_numpy(rng.integers(-127, 128, size=(M, K), dtype=np.int8)).to(dev)
    B = torch.from_numpy(rng.integers(-127, 128, size=(N, K), dtype=np.int8)).to(dev)
    ref = torch._int_mm(A, B.t().contiguous())
    ws = lib.get_workspace(lib.workspace_size(M, N, K), dev)
    for _ in range(2):
        acc = lib.gemm_s8s8s32(A, B, workspace=ws)
        assert torch.equal(acc, ref)
    acc.zero_()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        lib.gemm_s8s8s32(A, B, acc=acc, workspace=ws)
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(acc, ref)
    del g
    assert lib.read_status(ws, clear=False) == 0


@pytest.mark.parametrize("M,N,K,nout", [(256, 20480, 1152, 5), (300, 19000, 384, 3)])
def test_matmul_mixed_stream_k(lib, dev, oracle_mod, M, N, K, nout):
    """The whole linear on the stream-K path against the oracle, every element."""
    if torch.cuda.get_device_properties(dev).multi_processor_count == 148:
        assert _takes_stream_k(M, N, K, 148)
    lin = Linear("sk", M, N, K, nout, 40.0)
    X16, _ = make_activations(lin, seed=5)
    W16 = make_weight(lin, seed=5)
    check_full(lib, dev, oracle_mod, X16, W16, 6.0)


# ------------------------------------------------------------------ full linear

def test_tiny_workload(lib, dev, oracle_mod):
    lin = synthetic.TINY.linears[0]
    X16, W16, _ = synthetic.make_problem(lin, seed=0)
    g, r = check_full(lib, dev, oracle_mod, X16, W16, 6.0)
    assert g["O"].tolist() == [5, 37]


@pytest.mark.parametrize("M,N,K,nout,give_w16", [
    (333, 777, 1024, 5, True), (333, 777, 1024, 5, False), (129, 300, 2048, 40, True),
    (1, 640, 1024, 6, False), (8, 640, 1024, 6, True), (16, 200, 512, 3, False), (17, 640, 1024, 6, True),
    (32, 640, 1024, 6, False), (256, 512, 256, 0, True), (200, 384, 80, 2, True),
    # the epilogue's pipelined staging: at its column limit, one past it, both W sources,
    # the single-CTA form, and more tiles than CTA pairs (each pair prefetches its next tile)
    (300, 1000, 1024, 8, True), (300, 1000, 1024, 8, False), (300, 1000, 1024, 9, False),
    (100, 700, 1024, 8, False), (1024, 8192, 256, 6, True), (1024, 8192, 256, 6, False),
    # more outlier columns than one staged chunk: chunks outermost, partial sums kept in TMEM
    (512, 700, 1024, 33, True), (512, 700, 1024, 70, False), (300, 1000, 2048, 64, True)])
def test_matmul_mixed_matches_oracle(lib, dev, oracle_mod, M, N, K, nout, give_w16):
    lin = Linear("t", M, N, K, nout, 60.0)
    X16, cols = make_activations(lin, seed=M + N)
    W16 = make_weight(lin, seed=K)
    g, r = check_full(lib, dev, oracle_mod, X16, W16, 6.0, give_w16)
    if M >= 16:  # with few tokens a planted x60 column can stay below 6 (|z| < 0.1)
        assert set(cols.tolist()) <= set(r["O"].tolist())


def test_threshold_off_and_no_outliers(lib, dev, oracle_mod):
    X16 = make_random((150, 512), seed=3)
    W16 = make_random((300, 512), seed=4, scale=0.02)
    check_full(lib, dev, oracle_mod, X16, W16, 0.0)
    g, _ = check_full(lib, dev, oracle_mod, X16, W16, 6.0)     # N(0,1): nothing reaches 6
    assert g["O"].size == 0


@pytest.mark.parametrize("M", [48, 7])
def test_all_columns_outliers(lib, dev, oracle_mod, M):
    """A tiny threshold sends every column to the fp16 side (more outlier
    columns than the epilogue stages at once)."""
    X16 = make_random((M, 96), seed=11)
    W16 = make_random((136, 96), seed=12, scale=0.02)
    g, r = check_full(lib, dev, oracle_mod, X16, W16, 1e-3)
    assert g["O"].size == 96 and not g["CX"].any()


# ------------------------------------------------------------------ fused decode kernel (M <= 32)

@pytest.mark.parametrize("M,N,K", [(1, 100, 16), (3, 129, 80), (16, 300, 1040), (21, 1000, 4096),
                                   (2, 4000, 1024), (32, 256, 57344)])
def test_decode_split_tiles(lib, dev, oracle_mod, M, N, K):
    """The decode kernel spreads (weight tile, 128-byte K slice) units over
    the SMs: from a single unit (one CTA) up to tiles split over dozens of
    CTAs. The split products are summed exactly: acc is compared bit for bit."""
    lin = Linear("d", M, N, K, 3, 60.0)
    X16, _ = make_activations(lin, seed=M * 7 + K)
    W16 = make_weight(lin, seed=N)
    check_full(lib, dev, oracle_mod, X16, W16, 6.0, give_w16=False)


@pytest.mark.parametrize("n_cols,give_w16", [(32, False), (33, True), (33, False), (1, True)])
def test_decode_outlier_count_at_staging_limit(lib, dev, oracle_mod, n_cols, give_w16):
    """Every CTA of the decode kernel keeps its own list of the first 32
    outlier columns; with one more it reads the whole list that CTA 0
    publishes, in chunks. Columns spread over the K range, some in the last
    8-column group."""
    M, N, K = 5, 700, 2048
    X16 = make_random((M, K), seed=31)
    cols = np.unique(np.concatenate([np.linspace(3, K - 2, n_cols - 1).astype(np.int64), [K - 1]]))
    assert cols.size == n_cols
    rng = np.random.default_rng(n_cols)
    X16[rng.integers(0, M, cols.size), cols] = (40.0 * rng.choice([-1.0, 1.0], cols.size)).astype(np.float16)
    W16 = make_random((N, K), seed=32, scale=0.02)
    g, r = check_full(lib, dev, oracle_mod, X16, W16, 6.0, give_w16=give_w16)
    assert np.array_equal(np.sort(r["O"]), cols)


def test_decode_threshold_off(lib, dev, oracle_mod):
    X16 = make_random((5, 2048), seed=21)
    W16 = make_random((700, 2048), seed=22, scale=0.02)
    g, _ = check_full(lib, dev, oracle_mod, X16, W16, 0.0)
    assert g["O"].size == 0


def test_decode_after_prefill_same_workspace(lib, dev, oracle_mod):
    """A prefill call leaves its bitmap and codes in the shared workspace; the
    decode call after it must not depend on them (and the reverse)."""
    lin = Linear("t", 300, 640, 1024, 6, 60.0)
    X16, _ = make_activations(lin, seed=5)
    W16 = make_weight(lin, seed=5)
    check_full(lib, dev, oracle_mod, X16, W16, 6.0)
    check_full(lib, dev, oracle_mod, X16[:9], W16, 6.0)
    check_full(lib, dev, oracle_mod, X16[100:], W16, 6.0)


def test_decode_repeat_and_graph(lib, dev):
    """Tile counters return to zero after each call: repeated calls and CUDA
    graph replays give identical results."""
    lin = Linear("t", 4, 3000, 2048, 4, 60.0)
    X16, _ = make_activations(lin, seed=8)
    W16 = make_weight(lin, seed=8)
    X, W = to_dev(X16, dev), to_dev(W16, dev)
    layer = lib.Int8MixedLinear.from_fp16(W)
    ref = layer(X).clone()
    for _ in range(3):
        assert torch.equal(layer(X), ref)
    Y = torch.empty_like(ref)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        layer(X, Y=Y)
    torch.cuda.current_stream().wait_stream(s)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        layer(X, Y=Y)
    for _ in range(2):
        Y.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(Y, ref)


# ------------------------------------------------------------------ bias and GELU fused in the epilogue

@pytest.mark.parametrize("M,N,K,act", [(300, 520, 1040, "gelu_tanh"), (300, 520, 1040, None),
                                       (100, 384, 512, "gelu_tanh"), (5, 640, 1024, "gelu_tanh"),
                                       (32, 300, 2048, None), (7, 136, 96, "gelu_tanh"),
                                       (300, 520, 96, "gelu_tanh")])
def test_matmul_mixed_bias_activation(lib, dev, oracle_mod, M, N, K, act):
    """llmint8_matmul_mixed_ex: Y = fp16(act(linear + bias)) on every path
    (CTA-pair prefill, single-CTA prefill, fused decode; the K = 96 shapes send
    every column to the fp16 side, 96 columns in three chunks on the CTA-pair
    path). The tolerance is the linear's, carried
    through the activation: GELU's slope is at most 1.13, and the fp16
    rounding now happens after it."""
    lin = Linear("ba", M, N, K, 5, 60.0)
    X16, _ = make_activations(lin, seed=M + 3 * N)
    W16 = make_weight(lin, seed=K + 1)
    bias = np.random.default_rng(N).standard_normal(N).astype(np.float16)
    t = 1e-3 if K == 96 else 6.0
    X, W = to_dev(X16, dev), to_dev(W16, dev)
    CB, SCB, _ = lib.quantize_rowwise(W, 0.0)
    Y = lib.matmul_mixed(X, CB, SCB, W, t, bias=to_dev(bias, dev), activation=act)
    r = oracle_mod.matmul_mixed(X16, t, W=W16, bias=bias, activation=act)
    y = Y.cpu().numpy().astype(np.float64)
    pre = r["Y_lin"] + bias.astype(np.float64)[None, :]
    tol = 1.13 * (1e-2 + 2e-3 * np.abs(pre)) + 5e-4 * np.abs(r["Y"])
    bad = np.abs(y - r["Y"]) > tol
    assert not bad.any(), f"{bad.sum()} outside tolerance, worst {np.abs(y - r['Y']).max()}"


@pytest.mark.parametrize("M,N,K,nout,act,give_w16", [(300, 19000, 384, 40, "gelu_tanh", True),
                                                    (300, 19000, 384, 5, None, False)])
def test_stream_k_epilogue_variants(lib, dev, oracle_mod, M, N, K, nout, act, give_w16):
    """Stream-K (150 tiles on 74 pairs) under the other epilogue forms: more
    than 32 outlier columns (two chunks, the partial sums kept in TMEM between
    them) with a bias and GELU, and W's outlier columns recovered from CB with
    a bias only; against the oracle with the bias/activation tolerance."""
    if torch.cuda.get_device_properties(dev).multi_processor_count == 148:
        assert _takes_stream_k(M, N, K, 148)
    lin = Linear("ske", M, N, K, nout, 40.0)
    X16, _ = make_activations(lin, seed=nout)
    W16 = make_weight(lin, seed=nout)
    bias = np.random.default_rng(nout).standard_normal(N).astype(np.float16)
    X, W = to_dev(X16, dev), to_dev(W16, dev)
    CB, SCB, _ = lib.quantize_rowwise(W, 0.0)
    Y = lib.matmul_mixed(X, CB, SCB, W if give_w16 else None, 6.0, bias=to_dev(bias, dev), activation=act)
    r = oracle_mod.matmul_mixed(X16, 6.0, W=W16, use_fp16_weight_cols=give_w16, bias=bias, activation=act)
    assert r["O"].size == nout
    y = Y.cpu().numpy().astype(np.float64)
    pre = r["Y_lin"] + bias.astype(np.float64)[None, :]
    tol = 1.13 * (1e-2 + 2e-3 * np.abs(pre)) + 5e-4 * np.abs(r["Y"])
    bad = np.abs(y - r["Y"]) > tol
    assert not bad.any(), f"{bad.sum()} outside tolerance, worst {np.abs(y - r['Y']).max()}"


@pytest.mark.parametrize("M,N,K", [(300, 520, 1040), (4, 640, 1024), (64, 256, 4096), (300, 19000, 384)])
def test_fp16_weights_mode(lib, dev, oracle_mod, M, N, K):
    """llmint8_matmul_mixed_fp16w quantizes W on every call: its output is
    bit-identical to quantizing W once and calling matmul_mixed_ex, and its
    codes, outlier set and int32 products match the oracle exactly."""
    lin = Linear("fw", M, N, K, 4, 60.0)
    X16, _ = make_activations(lin, seed=M + N + K)
    W16 = make_weight(lin, seed=7)
    bias = np.random.default_rng(3).standard_normal(N).astype(np.float16)
    X, W, b = to_dev(X16, dev), to_dev(W16, dev), to_dev(bias, dev)
    dbg = dict(codes=torch.empty((M, K), dtype=torch.int8, device=dev),
               row_absmax=torch.empty(M, dtype=torch.float32, device=dev),
               col_idx=torch.empty(K, dtype=torch.int32, device=dev),
               count=torch.empty(1, dtype=torch.int32, device=dev),
               acc=torch.empty((M, N), dtype=torch.int32, device=dev))
    Y1 = lib.matmul_mixed_fp16w(X, W, 6.0, bias=b, activation="gelu_tanh", debug=dbg)
    CB, SCB, _ = lib.quantize_rowwise(W, 0.0)
    Y2 = lib.matmul_mixed(X, CB, SCB, W, 6.0, bias=b, activation="gelu_tanh")
    torch.cuda.synchronize()
    assert torch.equal(Y1, Y2)
    r = oracle_mod.matmul_mixed(X16, 6.0, W=W16, bias=bias, activation="gelu_tanh")
    n = int(dbg["count"].item())
    assert np.array_equal(dbg["col_idx"][:n].cpu().numpy(), r["O"])
    assert np.array_equal(dbg["codes"].cpu().numpy(), r["CX"])
    assert np.array_equal(dbg["acc"].cpu().numpy(), r["acc"])
    y = Y1.cpu().numpy().astype(np.float64)
    pre = r["Y_lin"] + bias.astype(np.float64)[None, :]
    assert np.all(np.abs(y - r["Y"]) <= 1.13 * (1e-2 + 2e-3 * np.abs(pre)) + 5e-4 * np.abs(r["Y"]))


def test_repeat_calls_identical(lib, dev):
    lin = Linear("t", 300, 600, 1024, 4, 60.0)
    X16, _ = make_activations(lin, seed=1)
    W16 = make_weight(lin, seed=1)
    X, W = to_dev(X16, dev), to_dev(W16, dev)
    layer = lib.Int8MixedLinear.from_fp16(W)
    y1 = layer(X).clone()
    y2 = layer(X)
    assert torch.equal(y1, y2)


def test_cuda_graph_capture(lib, dev):
    lin = Linear("t", 256, 512, 1024, 4, 60.0)
    X16, _ = make_activations(lin, seed=2)
    W16 = make_weight(lin, seed=2)
    X, W = to_dev(X16, dev), to_dev(W16, dev)
    layer = lib.Int8MixedLinear.from_fp16(W)
    ref = layer(X).clone()
    Y = torch.empty_like(ref)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        layer(X, Y=Y)
    torch.cuda.current_stream().wait_stream(s)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        layer(X, Y=Y)
    Y.zero_()
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(Y, ref)


# ------------------------------------------------------------------ full-size workloads, in full

def full_check(lib, dev, oracle_mod, X, W, t, give_w16, rows, cols, acc_ref="int_mm"):
    """Run the layer on device tensors X [M x K] and W [N x K] and compare it
    with the oracle on host copies, every element:
      - the outlier set, SX (fp32 bits), CX, CB and SB, against the oracle;
      - the int32 accumulators: acc_ref="oracle" against the oracle's own
        int8 product; acc_ref="int_mm" against torch._int_mm (cuBLAS, an
        independent library routine) applied to the ORACLE's CX and CB, with
        the oracle's own product checked on the sampled rows x columns;
      - Y against the oracle's output step (dequantization plus the outlier
        product, fp64) evaluated on that exact accumulator."""
    M, K = X.shape
    N = W.shape[0]
    CB, SCB, _ = lib.quantize_rowwise(W, 0.0)
    dbg = dict(codes=torch.empty((M, K), dtype=torch.int8, device=dev),
               row_absmax=torch.empty(M, dtype=torch.float32, device=dev),
               col_idx=torch.empty(K, dtype=torch.int32, device=dev),
               count=torch.empty(1, dtype=torch.int32, device=dev),
               acc=torch.empty((M, N), dtype=torch.int32, device=dev))
    Y = lib.matmul_mixed(X, CB, SCB, W if give_w16 else None, t, debug=dbg)
    torch.cuda.synchronize()
    Xh = X.cpu().numpy()
    O = oracle_mod.outlier_cols(Xh, t)
    n = int(dbg["count"].item())
    assert np.array_equal(dbg["col_idx"][:n].cpu().numpy(), O), "outlier columns"
    cx_ref, sx_ref = oracle_mod.quantize_rowwise(Xh, O)
    assert np.array_equal(dbg["row_absmax"].cpu().numpy().view(np.uint32), sx_ref.view(np.uint32)), "SX bits"
    assert np.array_equal(dbg["codes"].cpu().numpy(), cx_ref), "activation codes"
    del dbg["codes"]
    Wh = W.cpu().numpy()
    cb_ref, sb_ref = oracle_mod.quantize_weight(Wh)
    assert np.array_equal(CB.cpu().numpy(), cb_ref), "weight codes"
    assert np.array_equal(SCB.cpu().numpy().view(np.uint32), sb_ref.view(np.uint32)), "weight absmax bits"
    acc = dbg["acc"].cpu().numpy()
    del dbg["acc"]
    if acc_ref == "oracle":
        acc_full = oracle_mod.int8_matmul(cx_ref, cb_ref)
    else:
        assert oracle_mod.int8_matmul(cx_ref[rows], cb_ref[cols]).tolist() == acc[rows][:, cols].tolist(), \
            "int32 accumulators (oracle, sampled)"
        a_dev = torch.from_numpy(cx_ref).to(dev)
        b_dev = torch.from_numpy(cb_ref).to(dev).t().contiguous()
        acc_full = torch._int_mm(a_dev, b_dev).cpu().numpy()
        del a_dev, b_dev
    assert np.array_equal(acc, acc_full), "int32 accumulators"
    # W's outlier columns through the oracle, handed only those columns (a
    # gather, no arithmetic) so that it does not widen the whole weight again
    sel = np.arange(O.size, dtype=np.int64)
    wt = oracle_mod.outlier_weight(sel, N, O.size, W=np.ascontiguousarray(Wh[:, O]) if give_w16 else None,
                                   CB=np.ascontiguousarray(cb_ref[:, O]), SB=sb_ref)
    del Wh
    y_ref = oracle_mod.mixed_output(acc_full, sx_ref, sb_ref, Xh, O, wt)
    assert_y_close(Y.cpu().numpy(), y_ref, "Y")
    del CB, SCB, Y, dbg
    torch.cuda.empty_cache()
    return O


def _samples(M, N, seed, nrows=8, ncols=96):
    rng = np.random.default_rng(seed)
    rows = np.unique(np.concatenate([[0, M - 1], rng.choice(M, min(nrows, M), replace=False)]))
    cols = np.unique(np.concatenate([[0, N - 1], rng.choice(N, min(ncols, N), replace=False)]))
    return rows, cols


def test_prefill_workload_full(lib, dev, oracle_mod):
    """Prefill, 7B-class: X [2048 x 4096] with 4 columns x60, W [16384 x 4096],
    every output element; the accumulators against cuBLAS on the oracle's codes."""
    lin = synthetic.PREFILL_7B.linears[0]
    X16, cols = make_activations(lin, seed=0)
    W16 = make_weight(lin, seed=0)
    X, W = to_dev(X16, dev), to_dev(W16, dev)
    rows, jcols = _samples(lin.M, lin.N, 3)
    O = full_check(lib, dev, oracle_mod, X, W, 6.0, True, rows, jcols)
    assert set(cols.tolist()) <= set(O.tolist())


@pytest.mark.slow
def test_prefill_workload_full_oracle_product(lib, dev, oracle_mod):
    """The same prefill workload with the int32 accumulators compared in full
    against the oracle's own int8 product (137 G multiply-adds of plain C:
    about a minute)."""
    lin = synthetic.PREFILL_7B.linears[0]
    X16, _ = make_activations(lin, seed=0)
    W16 = make_weight(lin, seed=0)
    X, W = to_dev(X16, dev), to_dev(W16, dev)
    rows, jcols = _samples(lin.M, lin.N, 3)
    full_check(lib, dev, oracle_mod, X, W, 6.0, True, rows, jcols, acc_ref="oracle")


@pytest.mark.parametrize("M", [1, 8, 32])
def test_decode_workload_full(lib, dev, oracle_mod, M):
    """Decode at BLOOM width: X [M x 14336], W int8-prequantized [14336 x 14336]
    (outlier columns of W recovered as CB * SCB / 127), every output against
    the oracle's own int8 product."""
    lin = synthetic.decode_bloom(M).linears[0]
    X, W, cols = synthetic.torch_device_problem(lin, seed=M, device=dev)
    rows, jcols = _samples(lin.M, lin.N, M, ncols=160)
    O = full_check(lib, dev, oracle_mod, X, W, 6.0, False, rows, jcols, acc_ref="oracle")
    if M >= 16:
        assert set(cols.tolist()) <= set(O.tolist())
    del X, W
    torch.cuda.empty_cache()


@pytest.mark.parametrize("name", ["qkv", "attn_out", "fc1", "fc2"])
def test_bloom_block_linear_full(lib, dev, oracle_mod, name):
    """The four BLOOM-176B block linears at 2048 tokens, every element; the
    accumulators against cuBLAS on the oracle's codes, and against the
    oracle's own product on sampled rows x columns."""
    lin = {l.name: l for l in synthetic.BLOOM_BLOCK_2048.linears}[name]
    seed = {"qkv": 11, "attn_out": 12, "fc1": 13, "fc2": 14}[name]
    X, W, cols = synthetic.torch_device_problem(lin, seed=seed, device=dev)
    rows, jcols = _samples(lin.M, lin.N, 7, nrows=6, ncols=64)
    O = full_check(lib, dev, oracle_mod, X, W, 6.0, True, rows, jcols)
    assert set(cols.tolist()) <= set(O.tolist())
    del X, W
    torch.cuda.empty_cache()


def test_status_word_clean(lib, dev):
    """No kernel reported a timed-out wait during this module."""
    for ws in lib.workspaces():
        assert lib.read_status(ws, clear=False) == 0
