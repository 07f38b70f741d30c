"""Test support for the tensor-parallel layers (int8_mixed_precision_rowwise_b200.tp).

- ``run_lockstep``: drives the step generators of P emulated ranks in one
  process, doing each collective with plain torch ops on the ranks' tensors
  (the stand-in for NCCL when only one GPU, or none, is available). The ranks
  never wait on each other inside a kernel: every collective is a host step
  between launches.
- ``OracleOps``: the per-GPU steps of the layers computed by the CPU oracle on
  CPU tensors, so that the layers' host logic (shards, collectives, their
  order) runs on CPU ranks (gloo) without the CUDA library.
- ``bits_of`` / ``mask_of``: bitmap words <-> per-column masks.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle


def run_lockstep(gens):
    """Advance every rank's step generator to its next collective, perform it
    over all ranks, hand each rank its result; return the ranks' results."""
    n = len(gens)
    out = [None] * n

    def advance(i, value, first):
        try:
            return (next(gens[i]) if first else gens[i].send(value)), False
        except StopIteration as stop:
            out[i] = stop.value
            return None, True

    reqs = [advance(i, None, True) for i in range(n)]
    while True:
        fin = [r[1] for r in reqs]
        if all(fin):
            return out
        assert not any(fin), "ranks took different numbers of collective steps"
        ops = {r[0][0] for r in reqs}
        assert len(ops) == 1, f"ranks asked for different collectives: {ops}"
        op = ops.pop()
        ts = [r[0][1] for r in reqs]
        if op == "max":
            red = torch.stack(ts).amax(0)
            res = [red.clone() for _ in ts]
        elif op == "sum":
            red = torch.stack(ts).sum(0)
            res = [red.clone() for _ in ts]
        elif op == "gather":
            g = torch.stack(ts)
            res = [g.clone() for _ in ts]
        else:
            raise AssertionError(f"unknown collective {op}")
        reqs = [advance(i, res[i], False) for i in range(n)]


def mask_of(words, cols: int) -> np.ndarray:
    w = np.ascontiguousarray(np.asarray(words).astype("<u4"))
    bits = np.unpackbits(w.view(np.uint8), bitorder="little")
    return bits[:cols].astype(np.uint8)


def bits_of(mask: np.ndarray) -> np.ndarray:
    cols = mask.size
    nw = (cols + 31) // 32
    padded = np.zeros(nw * 32, dtype=np.uint8)
    padded[:cols] = mask
    return np.packbits(padded, bitorder="little").view("<u4").astype(np.int32)


class OracleOps:
    """The per-GPU steps the tensor-parallel layers call, computed by the
    oracle on the host. Inputs and outputs are CPU torch tensors with the
    binding's dtypes. Codes against a GIVEN row absmax come from the oracle's
    row quantizer run on the row with one more column holding that absmax:
    every other value of the row is at most it in magnitude, so the oracle
    takes it as the row's absmax and codes the real columns with it."""

    @staticmethod
    def _np(t):
        return t.detach().cpu().numpy()

    def quantize_rowwise(self, X, threshold, outlier_bitmap=None):
        x = self._np(X)
        mask = oracle.outlier_mask(x, threshold) if threshold > 0 else None
        codes, absmax = oracle.quantize_rowwise(x, mask)
        bm = torch.from_numpy(bits_of(mask)) if threshold > 0 else None
        return torch.from_numpy(codes), torch.from_numpy(absmax), bm

    def outlier_bitmap(self, X, threshold):
        x = self._np(X)
        mask = oracle.outlier_mask(x, threshold) if threshold > 0 else np.zeros(x.shape[1], np.uint8)
        return torch.from_numpy(bits_of(mask))

    def quantize_rowwise_given(self, X, outlier_bitmaps=None, row_absmax=None):
        x = self._np(X).astype(np.float32)
        rows, cols = x.shape
        mask = np.zeros(cols, np.uint8)
        if outlier_bitmaps is not None:
            words = self._np(outlier_bitmaps).reshape(-1, (cols + 31) // 32)
            for w in words:
                mask |= mask_of(w, cols)
        if row_absmax is None:
            codes, absmax = oracle.quantize_rowwise(x, mask)
        else:
            a = self._np(row_absmax).astype(np.float32)
            xp = np.concatenate([x, a[:, None]], axis=1)
            codes, absmax = oracle.quantize_rowwise(xp, np.concatenate([mask, [0]]).astype(np.uint8))
            assert np.array_equal(absmax.view(np.uint32), a.view(np.uint32))
            codes = np.ascontiguousarray(codes[:, :cols])
        return torch.from_numpy(codes), torch.from_numpy(absmax), torch.from_numpy(bits_of(mask))

    def find_outlier_cols(self, bitmap, cols, sync_count=True):
        idx = np.flatnonzero(mask_of(self._np(bitmap), cols)).astype(np.int32)
        col_idx = np.zeros(cols, np.int32)
        col_idx[:idx.size] = idx
        return torch.from_numpy(col_idx), torch.tensor([idx.size], dtype=torch.int32), idx.size

    def matmul_codes(self, CX, SX, X, CB, SCB, col_idx, d_count, W_f16=None, bias=None, activation=None,
                     out_f32=False):
        n = int(d_count[0])
        O = self._np(col_idx)[:n].astype(np.int64)
        cb, sb = self._np(CB), self._np(SCB)
        acc = oracle.int8_matmul(self._np(CX), cb)
        wt = oracle.outlier_weight(O, cb.shape[0], cb.shape[1], W=None if W_f16 is None else self._np(W_f16),
                                   CB=cb, SB=sb)
        y = oracle.mixed_output(acc, self._np(SX), sb, self._np(X), O, wt)
        if out_f32:
            return torch.from_numpy(y.astype(np.float32))
        if bias is not None or activation:
            y = oracle.bias_act(y, None if bias is None else self._np(bias), activation)
        return torch.from_numpy(y.astype(np.float16))

    def bias_act_to_f16(self, Y32, bias=None, activation=None):
        y = oracle.bias_act(self._np(Y32).astype(np.float64), None if bias is None else self._np(bias), activation)
        return torch.from_numpy(y.astype(np.float16))

    def gather_column_blocks(self, blocks):
        return torch.cat(list(blocks), dim=1).contiguous()

    def matmul_mixed(self, X, CB, SCB, W_f16, threshold, bias=None, activation=None):
        r = oracle.matmul_mixed(self._np(X), threshold, W=None if W_f16 is None else self._np(W_f16),
                                CB=self._np(CB), SB=self._np(SCB), use_fp16_weight_cols=W_f16 is not None,
                                bias=None if bias is None else self._np(bias), activation=activation)
        return torch.from_numpy(r["Y"].astype(np.float16))
