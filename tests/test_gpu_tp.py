"""GPU parity of the tensor-parallel pieces and layers (one GPU).

The library's per-GPU steps run on the GPU through the C ABI; the ranks of a
split are emulated in one process (tp_support.run_lockstep), each collective
done with torch ops between launches, so no kernel ever waits on another.
The bar is the one-GPU oracle: outlier set, row absmax (bits) and int8 codes
exact, the fp16 output within 1e-2 + 2e-3 |y|.
"""
import numpy as np
import pytest
import torch

from synthetic import Linear, make_activations, make_weight
from tp_support import mask_of, run_lockstep

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


def close(y, y_ref, what=""):
    err = np.abs(y.astype(np.float64) - y_ref)
    tol = ATOL + RTOL * np.abs(y_ref)
    assert np.all(err <= tol), f"{what}: {(err > tol).sum()} outside, worst {err.max():.4g}"


class Recording:
    """The library binding, keeping (codes, row absmax) of each quantization
    against a given outlier set."""

    def __init__(self, lib):
        self.lib = lib
        self.given = []

    def __getattr__(self, name):
        return getattr(self.lib, name)

    def quantize_rowwise_given(self, *a, **k):
        out = self.lib.quantize_rowwise_given(*a, **k)
        self.given.append((out[0], out[1]))
        return out


def problem(M, N, K, n_out=5, seed=1):
    lin = Linear("tp", M, N, K, n_out, 60.0)
    X16, cols = make_activations(lin, seed=seed)
    W16 = make_weight(lin, seed=seed)
    bias = (0.1 * np.random.default_rng(seed).standard_normal(N)).astype(np.float16)
    return X16, W16, bias


# ------------------------------------------------------------------ the pieces

@pytest.mark.parametrize("M,K,nbm,given", [(300, 1024, 3, False), (300, 1024, 1, True), (7, 4112, 2, False),
                                           (64, 160, 0, True), (0, 64, 1, False)])
def test_quantize_rowwise_given_matches_oracle(lib, dev, oracle_mod, M, K, nbm, given):
    X16, _, _ = problem(max(M, 1), 8, K)
    X16 = X16[:M]
    rng = np.random.default_rng(K)
    masks = [(rng.random(K) < 0.02).astype(np.uint8) for _ in range(nbm)]
    union = np.zeros(K, np.uint8)
    for m in masks:
        union |= m
    words = np.zeros((nbm, (K + 31) // 32), np.int32)
    for b, m in enumerate(masks):
        padded = np.zeros(words.shape[1] * 32, np.uint8)
        padded[:K] = m
        words[b] = np.packbits(padded, bitorder="little").view("<u4").astype(np.int32)
    c_ref, a_ref = oracle_mod.quantize_rowwise(X16, union)
    bms = to_dev(words, dev) if nbm else None
    if given:
        # a larger absmax than the row's own (as after a max over ranks): x2 of the fp16 value
        a_in = (2.0 * a_ref).astype(np.float32)
        xp = np.concatenate([X16.astype(np.float32), a_in[:, None]], axis=1)
        c_ref, a_chk = oracle_mod.quantize_rowwise(xp, np.concatenate([union, [0]]).astype(np.uint8))
        c_ref = c_ref[:, :K]
        codes, absmax, bm = lib.quantize_rowwise_given(to_dev(X16, dev), bms, row_absmax=to_dev(a_in, dev))
    else:
        codes, absmax, bm = lib.quantize_rowwise_given(to_dev(X16, dev), bms)
        assert np.array_equal(absmax.cpu().numpy().view(np.uint32), a_ref.view(np.uint32))
    torch.cuda.synchronize()
    assert np.array_equal(codes.cpu().numpy(), c_ref)
    assert np.array_equal(mask_of(bm.cpu().numpy(), K), union)


@pytest.mark.parametrize("M,N,K", [(300, 640, 1024), (2048, 1536, 4096), (24, 512, 1024), (9, 384, 512)])
def test_matmul_codes_matches_oracle(lib, dev, oracle_mod, M, N, K):
    """The GEMM on codes quantized beforehand, fp16 and fp32 outputs, bias and
    GELU; M <= 32 runs the swapped single-CTA form."""
    X16, W16, bias = problem(M, N, K, seed=M)
    X, W, b = to_dev(X16, dev), to_dev(W16, dev), to_dev(bias, dev)
    CB, SCB, _ = lib.quantize_rowwise(W, 0.0)
    cx, sx, bm = lib.quantize_rowwise(X, 6.0)
    col_idx, cnt, n = lib.find_outlier_cols(bm, K)
    y32 = lib.matmul_codes(cx, sx, X, CB, SCB, col_idx, cnt, W_f16=W, out_f32=True)
    y16 = lib.matmul_codes(cx, sx, X, CB, SCB, col_idx, cnt, W_f16=W, bias=b, activation="gelu_tanh")
    y16n = lib.matmul_codes(cx, sx, X, CB, SCB, col_idx, cnt)
    torch.cuda.synchronize()
    r = oracle_mod.matmul_mixed(X16, 6.0, W=W16)
    assert n == r["O"].size
    assert np.all(np.abs(y32.cpu().numpy().astype(np.float64) - r["Y"]) <= 1e-4 + 1e-5 * np.abs(r["Y"]))
    close(y16.cpu().numpy(), oracle_mod.bias_act(r["Y"], bias, "gelu_tanh"), "fp16 + bias + gelu")
    r2 = oracle_mod.matmul_mixed(X16, 6.0, W=W16, use_fp16_weight_cols=False)
    close(y16n.cpu().numpy(), r2["Y"], "fp16, outlier weights from CB")
    if M > 32:  # the same kernels as matmul_mixed: the same bits
        assert torch.equal(y16n, lib.matmul_mixed(X, CB, SCB, None, 6.0))


def test_bias_act_and_gather_blocks(lib, dev, oracle_mod):
    rng = np.random.default_rng(4)
    y32 = rng.standard_normal((37, 96)).astype(np.float32) * 3
    bias = (0.5 * rng.standard_normal(96)).astype(np.float16)
    out = lib.bias_act_to_f16(to_dev(y32, dev), to_dev(bias, dev), "gelu_tanh").cpu().numpy()
    close(out, oracle_mod.bias_act(y32.astype(np.float64), bias, "gelu_tanh"), "bias + gelu")
    blocks = to_dev(rng.standard_normal((3, 37, 64)).astype(np.float16), dev)
    g = lib.gather_column_blocks(blocks)
    assert torch.equal(g, torch.cat(list(blocks), dim=1))


# ------------------------------------------------------------------ the splits, ranks emulated

@pytest.mark.parametrize("world,M", [(2, 300), (4, 300), (4, 8)])
def test_column_split(lib, dev, oracle_mod, world, M):
    from int8_mixed_precision_rowwise_b200 import tp
    N, K = 1024, 1024
    X16, W16, bias = problem(M, N, K, seed=world)
    X, W, b = to_dev(X16, dev), to_dev(W16, dev), to_dev(bias, dev)
    layers = [tp.ColumnParallelInt8Linear.from_full_weight(W, world, r, bias=b, activation="gelu_tanh")
              for r in range(world)]
    outs = run_lockstep([l.steps(X) for l in layers])
    torch.cuda.synchronize()
    r = oracle_mod.matmul_mixed(X16, 6.0, W=W16, bias=bias, activation="gelu_tanh")
    for y in outs:
        close(y.cpu().numpy(), r["Y"], "column split")


@pytest.mark.parametrize("world,M,K", [(2, 300, 1024), (4, 300, 1040), (3, 8, 2064), (2, 2048, 4096)])
def test_row_split(lib, dev, oracle_mod, world, M, K):
    from int8_mixed_precision_rowwise_b200 import tp
    N = 768
    X16, W16, bias = problem(M, N, K, seed=K)
    r = oracle_mod.matmul_mixed(X16, 6.0, W=W16, bias=bias, activation="gelu_tanh")
    ops = Recording(lib)
    bounds = [tp.shard_bounds(K, world, i, 16) for i in range(world)]
    Ws = [to_dev(W16[:, lo:hi], dev) for lo, hi in bounds]
    preps = run_lockstep([tp.RowParallelInt8Linear.prepare_steps(w, ops=ops) for w in Ws])
    for (cb, sb), (lo, hi) in zip(preps, bounds):
        assert np.array_equal(cb.cpu().numpy(), r["CB"][:, lo:hi]), "weight codes of the shard"
        assert np.array_equal(sb.cpu().numpy().view(np.uint32), r["SB"].view(np.uint32)), "full-row absmax"
    b = to_dev(bias, dev)
    layers = [tp.RowParallelInt8Linear(cb, sb, w, b, "gelu_tanh", 6.0, ops=ops) for (cb, sb), w in zip(preps, Ws)]
    ops.given.clear()
    outs = run_lockstep([l.steps(to_dev(X16[:, lo:hi], dev)) for l, (lo, hi) in zip(layers, bounds)])
    torch.cuda.synchronize()
    assert len(ops.given) == world
    for _, sx in ops.given:
        assert np.array_equal(sx.cpu().numpy().view(np.uint32), r["SX"].view(np.uint32)), "row absmax"
    cx = np.concatenate([c.cpu().numpy() for c, _ in ops.given], axis=1)
    assert np.array_equal(cx, r["CX"]), "codes"
    for y in outs:
        close(y.cpu().numpy(), r["Y"], "row split")


@pytest.mark.parametrize("world,M", [(2, 300), (3, 40)])
def test_token_split(lib, dev, oracle_mod, world, M):
    """Including a column that crosses the threshold only in the last rank's
    rows while every rank's rows take their maximum in it."""
    from int8_mixed_precision_rowwise_b200 import tp
    N, K = 512, 1024
    X16, W16, bias = problem(M, N, K, seed=M)
    X16[:, 77] = np.float16(5.5)
    X16[M - 1, 77] = np.float16(40.0)
    r = oracle_mod.matmul_mixed(X16, 6.0, W=W16, bias=bias)
    assert 77 in r["O"]
    W, b = to_dev(W16, dev), to_dev(bias, dev)
    CB, SCB, _ = lib.quantize_rowwise(W, 0.0)
    ops = Recording(lib)
    bounds = [tp.shard_bounds(M, world, i) for i in range(world)]
    layers = [tp.TokenParallelInt8Linear(CB, SCB, W, b, None, 6.0, ops=ops) for _ in range(world)]
    outs = run_lockstep([l.steps(to_dev(X16[lo:hi], dev)) for l, (lo, hi) in zip(layers, bounds)])
    torch.cuda.synchronize()
    for y, (c, sx), (lo, hi) in zip(outs, ops.given, bounds):
        assert np.array_equal(sx.cpu().numpy().view(np.uint32), r["SX"][lo:hi].view(np.uint32))
        assert np.array_equal(c.cpu().numpy(), r["CX"][lo:hi])
        close(y.cpu().numpy(), r["Y"][lo:hi], "token split")


def test_tp_status_words_clean(lib, dev):
    for ws in lib.workspaces():
        assert lib.read_status(ws, clear=False) == 0
