"""Tensor-parallel LLM.int8() linear layers: one process per GPU,
torch.distributed (NCCL) for the collectives, the library's kernels for every
step of the arithmetic.

The deployment follows the page "优化故事：Bloom 推理", section "支持 TP": every
GPU owns a part of the weights and the parts are combined with all-reduces
(section "唾手可得的优化" names ncclAllReduce as the step that then dominates).
The arithmetic is the LLM.int8() layer of the page "Hugging Face 将 LLM.int8()
8-bit 量化集成进 transformers 与 accelerate"; each split below reproduces the
one-GPU result: the same outlier columns, row absmax and int8 codes, and the
int32 products summed exactly within each GPU.

  ColumnParallelInt8Linear  W's output rows split across GPUs. No exchange
                            before the GEMM (every GPU sees the whole X); the
                            output stays split by columns or is all-gathered.
  RowParallelInt8Linear     K split across GPUs. A column's outlier status
                            depends on that column only, so each GPU finds its
                            own; the row absmax is a max all-reduce of the
                            per-GPU maxima; the fp32 partial products are
                            sum all-reduced, then bias, activation and the
                            single fp16 rounding.
  TokenParallelInt8Linear   rows of X split across GPUs, W replicated. The
                            outlier set is the union over GPUs (bitmaps
                            all-gathered) so that every GPU quantizes against
                            the same set as one GPU would.

Each layer's forward is a generator of steps (`steps(X)`): it yields a
collective request ("max" | "sum" | "gather", tensor) where an exchange is
needed and receives the result. `run(steps)` drives it with torch.distributed;
a caller may drive it another way (all ranks in one process, for instance).
The per-GPU kernels come from `ops` (the library binding by default).
"""
from __future__ import annotations

import int8_mixed_precision_rowwise_b200 as _lib

__all__ = ["run", "shard_bounds", "ColumnParallelInt8Linear", "RowParallelInt8Linear", "TokenParallelInt8Linear"]


def run(steps, group=None):
    """Drive a step generator with torch.distributed collectives on `group`:
    "max"/"sum" are all-reduces in place, "gather" an all-gather that returns
    a new tensor [world, *shape]. Returns the generator's result. Every rank
    must drive the same layer, so that the collectives match."""
    import torch
    import torch.distributed as dist

    try:
        req = next(steps)
        while True:
            op, t = req
            if op == "max":
                dist.all_reduce(t, op=dist.ReduceOp.MAX, group=group)
                res = t
            elif op == "sum":
                dist.all_reduce(t, op=dist.ReduceOp.SUM, group=group)
                res = t
            elif op == "gather":
                world = dist.get_world_size(group)
                t = t.contiguous()
                if dist.get_backend(group) == "nccl":
                    res = t.new_empty((world,) + tuple(t.shape))
                    dist.all_gather_into_tensor(res, t, group=group)
                else:
                    parts = [torch.empty_like(t) for _ in range(world)]
                    dist.all_gather(parts, t, group=group)
                    res = torch.stack(parts)
            else:
                raise ValueError(f"unknown collective {op!r}")
            req = steps.send(res)
    except StopIteration as stop:
        return stop.value


def shard_bounds(n: int, world: int, rank: int, multiple: int = 1):
    """[lo, hi) of rank's part of n items, split as evenly as whole groups of
    `multiple` allow (the last parts may be smaller or empty)."""
    groups = (n + multiple - 1) // multiple
    per = (groups + world - 1) // world
    lo = min(n, rank * per * multiple)
    hi = min(n, (rank + 1) * per * multiple)
    return lo, hi


class ColumnParallelInt8Linear:
    """This GPU's output rows [N_r x K] of an LLM.int8() linear (CB, SCB, and
    optionally the fp16 weight and bias rows). `steps(X)` runs the whole
    layer on the full X; with gather_output the column blocks of every GPU
    (equal N_r, a multiple of 8) are all-gathered and put in place."""

    def __init__(self, CB, SCB, W_f16=None, bias=None, activation=None, threshold=_lib.DEFAULT_THRESHOLD,
                 gather_output=True, ops=None):
        self.CB, self.SCB, self.W_f16, self.bias = CB, SCB, W_f16, bias
        self.activation, self.threshold, self.gather_output = activation, threshold, gather_output
        self.ops = ops or _lib

    @classmethod
    def from_full_weight(cls, W, world, rank, bias=None, keep_fp16_weights=True, ops=None, **kw):
        """Take rank's rows of the full fp16 W [N x K] and quantize them (per
        output row, as on one GPU: each row is whole on its GPU)."""
        ops = ops or _lib
        lo, hi = shard_bounds(W.shape[0], world, rank, 8)
        Wr = W[lo:hi].contiguous()
        CB, SCB, _ = ops.quantize_rowwise(Wr, 0.0)
        b = bias[lo:hi].contiguous() if bias is not None else None
        return cls(CB, SCB, Wr if keep_fp16_weights else None, b, ops=ops, **kw)

    def steps(self, X):
        Y = self.ops.matmul_mixed(X, self.CB, self.SCB, self.W_f16, self.threshold, bias=self.bias,
                                  activation=self.activation)
        if not self.gather_output:
            return Y
        blocks = yield ("gather", Y)
        return self.ops.gather_column_blocks(blocks)


class RowParallelInt8Linear:
    """This GPU's columns [N x K_r] of CB (and of the fp16 weight), with SCB
    over the FULL rows of W. `steps(X_r)` takes this GPU's columns of X
    [M x K_r] and returns the whole fp16 output [M x N] on every GPU."""

    def __init__(self, CB, SCB, W_f16=None, bias=None, activation=None, threshold=_lib.DEFAULT_THRESHOLD, ops=None):
        self.CB, self.SCB, self.W_f16, self.bias = CB, SCB, W_f16, bias
        self.activation, self.threshold = activation, threshold
        self.ops = ops or _lib

    @staticmethod
    def prepare_steps(W_r, ops=None):
        """Weight preparation across GPUs for this GPU's columns W_r [N x K_r]:
        the row absmax over the full rows (a max all-reduce of the per-GPU
        maxima), then W_r's codes with it. Returns (CB_r, SCB)."""
        ops = ops or _lib
        _, sb, _ = ops.quantize_rowwise(W_r, 0.0)
        sb = yield ("max", sb)
        cb, _, _ = ops.quantize_rowwise_given(W_r, None, row_absmax=sb)
        return cb, sb

    def steps(self, X_r):
        ops = self.ops
        K_r = X_r.shape[1]
        # this GPU's outlier columns and the row absmax over its other columns
        _, sx, bm = ops.quantize_rowwise(X_r, self.threshold)
        sx = yield ("max", sx)
        cx, _, bm = ops.quantize_rowwise_given(X_r, bm, row_absmax=sx)
        col_idx, count, _ = ops.find_outlier_cols(bm, K_r, sync_count=False)
        y = ops.matmul_codes(cx, sx, X_r, self.CB, self.SCB, col_idx, count, W_f16=self.W_f16, out_f32=True)
        y = yield ("sum", y)
        return ops.bias_act_to_f16(y, self.bias, self.activation)


class TokenParallelInt8Linear:
    """A replica of the whole weight on every GPU; `steps(X_r)` takes this
    GPU's rows of X and returns its rows of Y, quantized against the union of
    every GPU's outlier columns (one all-gather of the bitmaps)."""

    def __init__(self, CB, SCB, W_f16=None, bias=None, activation=None, threshold=_lib.DEFAULT_THRESHOLD, ops=None):
        self.CB, self.SCB, self.W_f16, self.bias = CB, SCB, W_f16, bias
        self.activation, self.threshold = activation, threshold
        self.ops = ops or _lib

    def steps(self, X_r):
        ops = self.ops
        K = X_r.shape[1]
        bm = ops.outlier_bitmap(X_r, self.threshold)
        all_bm = yield ("gather", bm)
        cx, sx, bm = ops.quantize_rowwise_given(X_r, all_bm)
        col_idx, count, _ = ops.find_outlier_cols(bm, K, sync_count=False)
        return ops.matmul_codes(cx, sx, X_r, self.CB, self.SCB, col_idx, count, W_f16=self.W_f16, bias=self.bias,
                                activation=self.activation)
