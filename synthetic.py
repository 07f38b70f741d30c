"""Seeded synthetic inputs for the LLM.int8() mixed-precision linear.

This module only draws random numbers and names shapes. It holds none of the
method's arithmetic (no quantization, no outlier detection, no matmul), so the
CPU oracle and the CUDA path can both take their inputs from here without
sharing any computation.

Draw order (numpy PCG64, ``default_rng(seed)``):

1. the outlier hidden columns, ``rng.choice(K, n, replace=False)`` (or a fixed
   list where the workload names the columns),
2. ``X = rng.standard_normal((M, K), float32)``,
3. ``X[:, cols] *= scale`` in fp32, then a round-to-nearest cast to fp16,
4. ``W = 0.02 * rng.standard_normal((N, K), float32)``, cast to fp16.

The workloads mirror the transformer shapes the LLM.int8() blog post talks
about (BLOOM-176B with hidden size 14336, a 7B-class model with hidden size
4096), with systematic large-magnitude hidden columns standing in for the
"emergent outlier features" the post describes (section "离群特征的重要性",
the importance of outlier features). Trained weights and real activations are
not available, so these draws stand in for them.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

THRESHOLD = 6.0  # the post's outlier threshold (section "MatMul 内部", inside the MatMul)


@dataclass(frozen=True)
class Linear:
    """One linear layer Y[M,N] = X[M,K] · W[N,K]^T."""

    name: str
    M: int
    N: int
    K: int
    n_outlier_cols: int = 0
    outlier_scale: float = 1.0
    fixed_cols: tuple = ()
    w_fp16_given: bool = True  # False: W reaches the layer only as int8 codes + row scales


@dataclass(frozen=True)
class Workload:
    name: str
    linears: tuple = field(default_factory=tuple)
    threshold: float = THRESHOLD


# Tiny single linear: 8 tokens x 64 hidden, columns 5 and 37 scaled x20.
TINY = Workload("tiny_8x64x128", (Linear("tiny", 8, 128, 64, 2, 20.0, fixed_cols=(5, 37)),))

# Quantizer only: 4096 x 4096, 8 random columns x40 (no W, N=0).
QUANT_4096 = Workload("quantizer_4096x4096", (Linear("quant", 4096, 0, 4096, 8, 40.0),))

# Prefill linear, 7B-class: X [2048 x 4096], W [16384 x 4096], 4 columns x60.
PREFILL_7B = Workload("prefill_2048x16384x4096", (Linear("ffn_up", 2048, 16384, 4096, 4, 60.0),))


def decode_bloom(M: int) -> Workload:
    """Decode shape at BLOOM-176B width: X [M x 14336], W int8-prequantized [14336 x 14336]."""
    return Workload(f"decode_bloom_M{M}",
                    (Linear("attn_out", M, 14336, 14336, 6, 60.0, w_fp16_given=False),))


# The four BLOOM-176B block linears at 2048 tokens; ~0.05% of hidden columns x60
# (7 columns at K=14336, 29 at K=57344).
BLOOM_BLOCK_2048 = Workload("bloom176b_block_2048tok", (
    Linear("qkv", 2048, 43008, 14336, 7, 60.0),
    Linear("attn_out", 2048, 14336, 14336, 7, 60.0),
    Linear("fc1", 2048, 57344, 14336, 7, 60.0),
    Linear("fc2", 2048, 14336, 57344, 29, 60.0),
))

WORKLOADS = {w.name: w for w in (TINY, QUANT_4096, PREFILL_7B, BLOOM_BLOCK_2048,
                                 decode_bloom(1), decode_bloom(8), decode_bloom(32))}


def outlier_columns(rng: np.random.Generator, lin: Linear) -> np.ndarray:
    if lin.fixed_cols:
        return np.array(sorted(lin.fixed_cols), dtype=np.int64)
    if lin.n_outlier_cols == 0:
        return np.zeros(0, dtype=np.int64)
    return np.sort(rng.choice(lin.K, lin.n_outlier_cols, replace=False)).astype(np.int64)


def make_activations(lin: Linear, seed: int = 0, rows: int | None = None):
    """X fp16 [M x K] ~N(0,1) with the workload's outlier columns scaled.

    Returns (X_fp16, cols). ``rows`` overrides M (same column draw, fewer rows).
    """
    rng = np.random.default_rng(seed)
    cols = outlier_columns(rng, lin)
    m = lin.M if rows is None else rows
    x = rng.standard_normal((m, lin.K), dtype=np.float32)
    if cols.size:
        x[:, cols] *= np.float32(lin.outlier_scale)
    return x.astype(np.float16), cols


def make_weight(lin: Linear, seed: int = 0, rows: int | None = None) -> np.ndarray:
    """W fp16 [N x K] ~N(0, 0.02). Drawn from a stream of its own (seed + 1) so
    that X and W can be made independently at any size."""
    rng = np.random.default_rng(seed + 1)
    n = lin.N if rows is None else rows
    w = np.float32(0.02) * rng.standard_normal((n, lin.K), dtype=np.float32)
    return w.astype(np.float16)


def make_problem(lin: Linear, seed: int = 0):
    """(X fp16, W fp16 or None, cols) for one linear, all on the host."""
    x, cols = make_activations(lin, seed)
    w = make_weight(lin, seed) if lin.N > 0 else None
    return x, w, cols


def make_random(shape, seed: int, scale: float = 1.0, dtype=np.float16) -> np.ndarray:
    """Plain N(0, scale^2) draw for property and edge-case tests."""
    rng = np.random.default_rng(seed)
    return (np.float32(scale) * rng.standard_normal(shape, dtype=np.float32)).astype(dtype)


def torch_device_problem(lin: Linear, seed: int, device):
    """Same distributions drawn on the GPU with a seeded torch generator, for
    the multi-GB BLOOM-shaped weights whose host draw would take minutes.
    Returns (X fp16, W fp16, cols) as device tensors (cols on the host)."""
    import torch

    rng = np.random.default_rng(seed)
    cols = outlier_columns(rng, lin)
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    x = torch.randn((lin.M, lin.K), generator=g, device=device, dtype=torch.float32)
    if cols.size:
        idx = torch.as_tensor(cols, device=device)
        x[:, idx] *= lin.outlier_scale
    x = x.half()
    w = (torch.randn((lin.N, lin.K), generator=g, device=device, dtype=torch.float32) * 0.02).half()
    return x, w, cols
