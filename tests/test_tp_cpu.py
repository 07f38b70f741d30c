"""The tensor-parallel layers' host logic on CPU: shards, the collectives and
their order, checked against the oracle's one-GPU layer.

The per-GPU steps run in the oracle (tp_support.OracleOps), so no CUDA
library is needed. First the ranks are driven in one process (run_lockstep),
then as two gloo processes through the layers' own torch.distributed driver
(tp.run). The bar is the one-GPU result: the outlier set, row absmax and codes
exactly, the fp16 output within 1e-2 + 2e-3 |y|.

Splits (page "优化故事：Bloom 推理", section "支持 TP"): column (W's output rows
across ranks, output all-gathered), row (K across ranks: max all-reduce of
the row absmax, sum all-reduce of fp32 partial outputs), token (rows of X
across ranks, outlier bitmaps all-gathered so every rank uses the union).
"""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from conftest import ROOT
from synthetic import Linear, make_activations, make_weight
from tp_support import OracleOps, run_lockstep

ATOL, RTOL = 1e-2, 2e-3


def _problem(M=40, N=96, K=160, seed=3):
    lin = Linear("tp", M, N, K, 4, 60.0)
    X16, cols = make_activations(lin, seed=seed)
    W16 = make_weight(lin, seed=seed)
    bias = (0.1 * np.random.default_rng(seed).standard_normal(N)).astype(np.float16)
    return X16, W16, bias, cols


def _close(y, y_ref):
    err = np.abs(y.astype(np.float64) - y_ref)
    assert np.all(err <= ATOL + RTOL * np.abs(y_ref)), f"worst {err.max():.4g}"


def _column(tp, ops, X16, W16, bias, world, rank, drive):
    N = W16.shape[0]
    lin = tp.ColumnParallelInt8Linear.from_full_weight(torch.from_numpy(W16), world, rank,
                                                       bias=torch.from_numpy(bias), ops=ops,
                                                       activation="gelu_tanh", threshold=6.0)
    assert lin.CB.shape[0] == N // world
    return drive(lin.steps(torch.from_numpy(X16)))


def _row_prepare(tp, ops, W16, world, rank, drive):
    lo, hi = tp.shard_bounds(W16.shape[1], world, rank, 16)
    Wr = torch.from_numpy(np.ascontiguousarray(W16[:, lo:hi]))
    cb, sb = drive(tp.RowParallelInt8Linear.prepare_steps(Wr, ops=ops))
    return cb, sb, Wr, (lo, hi)


def _row(tp, ops, X16, W16, bias, world, rank, drive, prepared):
    cb, sb, Wr, (lo, hi) = prepared
    lin = tp.RowParallelInt8Linear(cb, sb, Wr, torch.from_numpy(bias), "gelu_tanh", 6.0, ops=ops)
    return drive(lin.steps(torch.from_numpy(np.ascontiguousarray(X16[:, lo:hi]))))


def _token(tp, ops, X16, W16, bias, world, rank, drive):
    import oracle
    CB, SB = oracle.quantize_weight(W16)
    lo, hi = tp.shard_bounds(X16.shape[0], world, rank)
    lin = tp.TokenParallelInt8Linear(torch.from_numpy(CB), torch.from_numpy(SB), torch.from_numpy(W16),
                                     None if bias is None else torch.from_numpy(bias), None, 6.0, ops=ops)
    return drive(lin.steps(torch.from_numpy(np.ascontiguousarray(X16[lo:hi])))), (lo, hi)


class RecordingOps(OracleOps):
    """OracleOps that keeps (codes, row absmax) of every quantization against
    a given outlier set, in call order."""

    def __init__(self):
        self.given = []

    def quantize_rowwise_given(self, X, outlier_bitmaps=None, row_absmax=None):
        out = super().quantize_rowwise_given(X, outlier_bitmaps, row_absmax)
        self.given.append((out[0], out[1]))
        return out


@pytest.mark.parametrize("world", [2, 3])
def test_splits_in_lockstep_match_one_gpu(oracle_mod, world):
    from int8_mixed_precision_rowwise_b200 import tp

    ops = RecordingOps()
    X16, W16, bias, cols = _problem()
    ref = oracle_mod.matmul_mixed(X16, 6.0, W=W16, bias=bias, activation="gelu_tanh")
    assert set(cols.tolist()) <= set(ref["O"].tolist())

    # column split: every rank ends with the whole output
    gens = [_column(tp, ops, X16, W16, bias, world, r, lambda g: g) for r in range(world)]
    outs = run_lockstep(gens)
    for y in outs:
        _close(y.numpy(), ref["Y"])

    # row split: weight preparation across ranks gives the one-GPU CB columns and SB bits
    preps = run_lockstep([tp.RowParallelInt8Linear.prepare_steps(
        torch.from_numpy(np.ascontiguousarray(W16[:, slice(*tp.shard_bounds(W16.shape[1], world, r, 16))])),
        ops=ops) for r in range(world)])
    for r, (cb, sb) in enumerate(preps):
        lo, hi = tp.shard_bounds(W16.shape[1], world, r, 16)
        assert np.array_equal(cb.numpy(), ref["CB"][:, lo:hi])
        assert np.array_equal(sb.numpy().view(np.uint32), ref["SB"].view(np.uint32))
    gens = []
    for r in range(world):
        lo, hi = tp.shard_bounds(W16.shape[1], world, r, 16)
        gens.append(_row(tp, ops, X16, W16, bias, world, r, lambda g: g,
                         (preps[r][0], preps[r][1], torch.from_numpy(np.ascontiguousarray(W16[:, lo:hi])), (lo, hi))))
    ops.given.clear()
    for y in run_lockstep(gens):
        _close(y.numpy(), ref["Y"])
    # every rank coded its columns with the full row absmax: the codes side by side are the one-GPU codes
    assert len(ops.given) == world
    for _, sx in ops.given:
        assert np.array_equal(sx.numpy().view(np.uint32), ref["SX"].view(np.uint32))
    assert np.array_equal(np.concatenate([c.numpy() for c, _ in ops.given], axis=1), ref["CX"])

    # token split: each rank's rows of the output
    ref_lin = oracle_mod.matmul_mixed(X16, 6.0, W=W16, bias=bias)
    pairs = [_token(tp, ops, X16, W16, bias, world, r, lambda g: g) for r in range(world)]
    outs = run_lockstep([g for g, _ in pairs])
    for y, (_, (lo, hi)) in zip(outs, pairs):
        _close(y.numpy(), ref_lin["Y"][lo:hi])


def test_token_split_uses_the_union_of_outlier_columns(oracle_mod):
    """A column crosses the threshold only in rank 1's rows, while rank 0's
    rows take their maximum in it: without the union rank 0 would keep the
    column in its int8 part with a different row absmax."""
    from int8_mixed_precision_rowwise_b200 import tp

    X16, W16, _, _ = _problem(M=16, seed=9)
    X16[:, 33] = np.float16(5.5)
    X16[12, 33] = np.float16(40.0)   # rank 1 of 2 holds rows 8..15
    ref = oracle_mod.matmul_mixed(X16, 6.0, W=W16)
    assert 33 in ref["O"]
    ops = RecordingOps()
    pairs = [_token(tp, ops, X16, W16, None, 2, r, lambda g: g) for r in range(2)]
    outs = run_lockstep([g for g, _ in pairs])
    for y, (_, (lo, hi)), (codes, sx) in zip(outs, pairs, ops.given):
        assert np.array_equal(sx.numpy().view(np.uint32), ref["SX"][lo:hi].view(np.uint32))
        assert np.array_equal(codes.numpy(), ref["CX"][lo:hi])
        _close(y.numpy(), ref["Y"][lo:hi])


def test_shard_bounds_cover_every_item_once():
    from int8_mixed_precision_rowwise_b200 import tp
    for n, world, mult in [(1040, 4, 16), (96, 3, 8), (10, 4, 1), (7, 8, 1), (0, 2, 16)]:
        parts = [tp.shard_bounds(n, world, r, mult) for r in range(world)]
        assert parts[0][0] == 0 and parts[-1][1] == n
        for (a, b), (c, d) in zip(parts, parts[1:]):
            assert b == c and a <= b
        for lo, hi in parts[:-1]:
            assert lo % mult == 0 and (hi - lo) % mult == 0


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _gloo_rank(rank, world, port, q):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    from datetime import timedelta
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        import oracle
        from int8_mixed_precision_rowwise_b200 import tp
        from tp_support import OracleOps
        oracle.build()
        ops = OracleOps()
        X16, W16, bias, _ = _problem()
        drive = tp.run
        ref = oracle.matmul_mixed(X16, 6.0, W=W16, bias=bias, activation="gelu_tanh")
        y_col = _column(tp, ops, X16, W16, bias, world, rank, drive).numpy()
        prep = _row_prepare(tp, ops, W16, world, rank, drive)
        y_row = _row(tp, ops, X16, W16, bias, world, rank, drive, prep).numpy()
        y_tok, (lo, hi) = _token(tp, ops, X16, W16, bias, world, rank, drive)
        ref_lin = oracle.matmul_mixed(X16, 6.0, W=W16, bias=bias)
        errs = []
        for name, y, r in [("column", y_col, ref["Y"]), ("row", y_row, ref["Y"]),
                           ("token", y_tok.numpy(), ref_lin["Y"][lo:hi])]:
            err = np.abs(y.astype(np.float64) - r)
            if not np.all(err <= ATOL + RTOL * np.abs(r)):
                errs.append(f"{name}: worst {err.max():.4g}")
        cb_lo, cb_hi = prep[3]
        if not np.array_equal(prep[0].numpy(), ref["CB"][:, cb_lo:cb_hi]):
            errs.append("row split weight codes")
        q.put((rank, errs))
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_splits_over_two_gloo_ranks():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_gloo_rank, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    got = {}
    for _ in range(world):
        rank, errs = q.get(timeout=180)
        got[rank] = errs
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert got == {0: [], 1: []}
