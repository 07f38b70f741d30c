"""Pins of the CPU oracle against what the source pages and mathematics fix.

Every test here runs on the CPU. Each one is chosen so that a plausible slip
in the oracle (a dropped term, a wrong sign or index, a transposed operand, a
wrong scale constant, > instead of >=) makes at least one of them fail.
Citations name the page "Hugging Face 将 LLM.int8() 8-bit 量化集成进
transformers 与 accelerate" and its section.
"""
import numpy as np
import pytest
import torch

from conftest import read_golden
from synthetic import Linear, make_activations, make_random, make_weight

pytestmark = pytest.mark.filterwarnings("ignore::DeprecationWarning")


# --- section "模型量化简介" (Introduction to model quantization) ---------------

def test_absmax_worked_example_decimal(oracle_mod):
    """absmax 5.4 -> factor 127/5.4 ~ 23.5 -> [28,-12,-101,28,-73,19,56,127]."""
    g = read_golden("absmax_worked_example.txt")
    x = np.array([g["input"]], dtype=np.float32)
    codes, absmax = oracle_mod.quantize_rowwise(x)
    assert codes[0].tolist() == [int(v) for v in g["codes"]]
    assert absmax[0] == np.float32(g["absmax"][0])
    assert round(127.0 / float(absmax[0]), 1) == g["scale_printed"][0]


def test_absmax_worked_example_fp16_inputs(oracle_mod):
    """The same codes when the vector first passes through fp16 (the layer's input type)."""
    g = read_golden("absmax_worked_example.txt")
    x = np.array([g["input"]], dtype=np.float16)
    codes, absmax = oracle_mod.quantize_rowwise(x)
    assert codes[0].tolist() == [int(v) for v in g["codes"]]
    assert absmax[0] == np.float32(np.float16(5.4))  # 5.3984375


def test_fixed_range_round_trip(oracle_mod):
    """Range -1..1 scaled by 127: 0.3 -> 38.1 -> 38 -> 38/127 = 0.2992."""
    g = read_golden("fixed_range_round_trip.txt")
    x = np.array([[g["value"][0], -g["range_absmax"][0]]], dtype=np.float32)
    codes, absmax = oracle_mod.quantize_rowwise(x)
    assert absmax[0] == 1.0
    assert round(float(np.float32(0.3) * np.float32(127.0 / absmax[0])), 1) == g["scaled_printed"][0]
    assert codes[0, 0] == int(g["code"][0]) and codes[0, 1] == -127
    # Recovery uses the same absmax/127 rule the weight path uses (CB * SCB / 127).
    wt = oracle_mod.outlier_weight(np.array([0]), 1, 2, CB=codes, SB=absmax)
    assert round(float(wt[0, 0]), 4) == g["dequant_printed"][0]
    assert abs(0.3 - float(wt[0, 0])) < 0.008


def test_round_half_to_even_ties(oracle_mod):
    """The pages say 'round' with no tie rule; the reading is half-to-even.
    absmax 127 gives s = 1 exactly, so x*s lands exactly on the .5 ties."""
    x = np.array([[127.0, 2.5, 3.5, -2.5, -0.5, 0.5, 1.5]], dtype=np.float32)
    codes, _ = oracle_mod.quantize_rowwise(x)
    assert codes[0].tolist() == [127, 2, 4, -2, 0, 0, 2]


# --- section "用法" (Usage): printed weights ----------------------------------

def _printed():
    g = read_golden("printed_weights.txt")
    w16 = np.array(g["fp16"], dtype=np.float16)
    q = np.array(g["int8"], dtype=np.int64)
    d = np.array(g["dequant"], dtype=np.float64)
    return w16, q, d


def _row_scale_interval(w, q):
    """Scales s with rint(w*s) == q for every visible entry of one row, assuming
    one scale per row; also s <= 127/max|w| since the row absmax bounds the
    visible values. Pure interval arithmetic on the printed numbers."""
    w = w.astype(np.float64)
    pos, neg = w > 0, w < 0
    lo = max(((q - 0.5) / w)[pos].max(), ((q + 0.5) / w)[neg].max())
    hi = min(((q + 0.5) / w)[pos].min(), ((q - 0.5) / w)[neg].min(), 127.0 / np.abs(w).max())
    return lo, hi


def _fillers(w16, q):
    """One fp16 absmax per row inside its feasible interval (the elided columns
    hold the row maximum; we stand in for it with this filler)."""
    out = []
    for r in range(w16.shape[0]):
        lo, hi = _row_scale_interval(w16[r], q[r])
        assert lo < hi, f"row {r}: printed codes admit no single per-row scale"
        b0 = int(np.float16(127.0 / hi).view(np.uint16)) - 1
        b1 = int(np.float16(127.0 / lo).view(np.uint16)) + 1
        cands = np.arange(b0, b1 + 1, dtype=np.uint16).view(np.float16).astype(np.float64)
        ok = [a for a in cands if lo + 0.05 < 127.0 / a < hi - 0.05]
        assert ok, f"row {r}: no fp16 absmax strictly inside the interval"
        out.append(ok[len(ok) // 2])
    return np.array(out, dtype=np.float16)


def test_printed_weights_per_output_row(oracle_mod):
    """The page prints W (fp16) and CB (int8) for Linear8bitLt(64, 64). With one
    absmax per OUTPUT ROW, the oracle reproduces all 36 visible codes."""
    w16, q, _ = _printed()
    a = _fillers(w16, q)
    W = np.concatenate([w16, a[:, None]], axis=1)
    codes, absmax = oracle_mod.quantize_rowwise(W)
    assert np.array_equal(codes[:, :6].astype(np.int64), q)
    assert np.array_equal(absmax, a.astype(np.float32))


def test_printed_weights_reject_per_column_scale(oracle_mod):
    """Negative control: quantizing the same matrix with one scale per column
    (a transposed operand) does not give the printed codes."""
    w16, q, _ = _printed()
    a = _fillers(w16, q)
    W = np.concatenate([w16, a[:, None]], axis=1)
    codes_t, _ = oracle_mod.quantize_rowwise(np.ascontiguousarray(W.T))
    assert not np.array_equal(codes_t.T[:, :6].astype(np.int64), q)


def test_printed_dequant_is_column_broadcast(oracle_mod):
    """The page's '(CB * SCB) / 127' printout: SCB has one entry per output row,
    but the printed matrix matches SCB broadcast along the LAST dim (column c
    scaled by row c's absmax) and not per row. The oracle recovers W's columns
    per output row (SCB[:, None]), as the code-to-weight ratio of each printed
    row requires; this pins both facts."""
    w16, q, d = _printed()
    a = _fillers(w16, q).astype(np.float32)
    wt = oracle_mod.outlier_weight(np.arange(6), 6, 6, CB=q.astype(np.int8), SB=a)
    col_bcast = q * a[None, :].astype(np.float64) / 127.0
    assert np.abs(col_bcast - d).max() < 5e-4            # the page's printed (bugged) output
    off = ~np.eye(6, dtype=bool)
    assert np.abs(wt.astype(np.float64) - d)[off].max() > 2e-3  # oracle differs off-diagonal
    assert np.abs(wt.astype(np.float64) - d)[~off].max() < 5e-4  # and agrees on the diagonal
    # per-row recovery is close to the printed fp16 weights themselves
    assert np.abs(wt.astype(np.float64) - w16.astype(np.float64)).max() < 6e-4


# --- sections "LLM.int8() 的简要总结" and "MatMul 内部" ---------------------------

def test_threshold_is_magnitude_6_or_greater(oracle_mod):
    """'all outliers of magnitude 6 or greater': |x| == 6 is an outlier, the
    largest fp16 below 6 is not; negative values count by magnitude."""
    below = float(np.nextafter(np.float16(6.0), np.float16(0.0)))
    x = np.array([[6.0, below, -6.0, 0.1], [0.0, 0.0, 0.0, 0.0]], dtype=np.float16)
    assert oracle_mod.outlier_cols(x, 6.0).tolist() == [0, 2]
    assert oracle_mod.outlier_cols(x, 0.0).tolist() == []     # t <= 0: no decomposition
    assert oracle_mod.outlier_cols(x, -1.0).tolist() == []


def test_row_absmax_excludes_outlier_columns(oracle_mod):
    """Column 0 is an outlier because of row 0; row 1 holds 5 there (below t).
    Row 1's absmax must come from its non-outlier columns (0.75), and its
    outlier-column code must be 0."""
    x = np.array([[100.0, 0.5, -0.25], [5.0, 0.75, -0.5]], dtype=np.float16)
    O = oracle_mod.outlier_cols(x, 6.0)
    assert O.tolist() == [0]
    codes, absmax = oracle_mod.quantize_rowwise(x, O)
    assert absmax.tolist() == [0.5, 0.75]
    assert codes.tolist() == [[0, 127, -64], [0, 127, -85]]


def test_zero_row_and_all_outlier_row(oracle_mod):
    x = np.array([[0.0, 0.0, 0.0, 0.0], [7.0, -8.0, 9.0, 10.0], [1.0, 2.0, 3.0, 4.0]], dtype=np.float16)
    O = oracle_mod.outlier_cols(x, 6.0)
    assert O.tolist() == [0, 1, 2, 3]
    codes, absmax = oracle_mod.quantize_rowwise(x, O)
    assert absmax.tolist() == [0.0, 0.0, 0.0] and not codes.any()
    codes, absmax = oracle_mod.quantize_rowwise(x[:1], None)
    assert absmax.tolist() == [0.0] and not codes.any()


def test_int8_matmul_matches_numpy_and_torch(oracle_mod):
    rng = np.random.default_rng(3)
    A = rng.integers(-127, 128, size=(37, 96), dtype=np.int8)
    B = rng.integers(-127, 128, size=(53, 96), dtype=np.int8)
    acc = oracle_mod.int8_matmul(A, B)
    ref = A.astype(np.int64) @ B.astype(np.int64).T
    assert np.array_equal(acc.astype(np.int64), ref)
    tm = torch._int_mm(torch.from_numpy(A[:32].copy()), torch.from_numpy(B[:48].T.copy()))
    assert np.array_equal(acc[:32, :48], tm.numpy())


def test_int8_matmul_int32_margin(oracle_mod):
    """K = 57344 with every code at +-127: |sum| = 57344*127^2 = 924,901,376 fits int32."""
    K = 57344
    A = np.full((2, K), 127, dtype=np.int8)
    A[1] = -127
    B = np.full((1, K), 127, dtype=np.int8)
    acc = oracle_mod.int8_matmul(A, B)
    assert acc[:, 0].tolist() == [K * 127 * 127, -K * 127 * 127]
    with pytest.raises(OverflowError):
        oracle_mod.int8_matmul(np.full((1, 140000), 127, np.int8), np.full((1, 140000), 127, np.int8))


def test_decomposition_is_identity_without_outliers(oracle_mod):
    """No |x| reaches the threshold: O is empty and the result is exactly plain
    vector-wise int8 (threshold off)."""
    X = make_random((17, 160), seed=11)          # N(0,1): max|x| ~ 4 < 6
    W = make_random((23, 160), seed=12, scale=0.02)
    assert np.abs(X.astype(np.float32)).max() < 6.0
    r6 = oracle_mod.matmul_mixed(X, 6.0, W=W)
    r0 = oracle_mod.matmul_mixed(X, 0.0, W=W)
    assert r6["O"].size == 0
    assert np.array_equal(r6["Y"], r0["Y"]) and np.array_equal(r6["CX"], r0["CX"])


def test_all_columns_outliers_gives_fp_product(oracle_mod):
    """Threshold below every |x|: all columns go to the fp16 side, the int8 part
    is empty, and Y equals X . W^T computed by a library fp64 matmul."""
    X = make_random((9, 48), seed=21)
    W = make_random((13, 48), seed=22, scale=0.02)
    r = oracle_mod.matmul_mixed(X, 1e-4, W=W)
    assert r["O"].size == 48 and not r["CX"].any() and not r["acc"].any()
    ref = X.astype(np.float64) @ W.astype(np.float64).T
    np.testing.assert_allclose(r["Y"], ref, rtol=1e-12, atol=1e-12)


def test_outlier_columns_recovered_from_int8_weight(oracle_mod):
    """All columns outliers and no fp16 W: Y = X . (CB * SB / 127)^T."""
    X = make_random((5, 32), seed=31)
    W = make_random((7, 32), seed=32, scale=0.02)
    CB, SB = oracle_mod.quantize_weight(W)
    r = oracle_mod.matmul_mixed(X, 1e-4, CB=CB, SB=SB)
    wt = CB.astype(np.float64) * SB.astype(np.float64)[:, None] / 127.0
    np.testing.assert_allclose(r["Y"], X.astype(np.float64) @ wt.T, rtol=1e-6, atol=1e-7)


def test_error_bound_against_exact_product(oracle_mod):
    """|Y - X.W^T| is bounded by the quantization error of the int8 part:
    sum over non-outlier c of |x|dw + |w|dx + dx*dw, with dx = SX/254 and
    dw = SB/254 (half a code step). A wrong dequant constant, a dropped outlier
    term or a sign slip breaks this by orders of magnitude."""
    from synthetic import Linear, make_activations, make_weight
    lin = Linear("t", 64, 96, 512, 5, 60.0)
    X, cols = make_activations(lin, seed=5)
    W = make_weight(lin, seed=5)
    r = oracle_mod.matmul_mixed(X, 6.0, W=W)
    assert set(cols.tolist()) <= set(r["O"].tolist())
    x = X.astype(np.float64)
    w = W.astype(np.float64)
    keep = np.ones(lin.K, dtype=bool)
    keep[r["O"]] = False
    dx = r["SX"].astype(np.float64)[:, None] / 254.0
    dw = r["SB"].astype(np.float64)[:, None] / 254.0
    ax, aw = np.abs(x[:, keep]), np.abs(w[:, keep])
    bound = ax @ (dw * np.ones_like(aw)).T + (dx * np.ones_like(ax)) @ aw.T + (dx @ dw.T) * keep.sum()
    err = np.abs(r["Y"] - x @ w.T)
    assert np.all(err <= bound * (1 + 1e-9) + 1e-9)
    assert err.max() > 0  # int8 is lossy: the test is not vacuous
    # the outlier part is large: dropping it would exceed the bound
    outl = np.abs(x[:, r["O"]] @ w[:, r["O"]].T)
    assert (outl > bound).mean() > 0.5


def test_codes_invariants(oracle_mod):
    X = make_random((40, 256), seed=41, scale=3.0)
    O = oracle_mod.outlier_cols(X, 6.0)
    codes, absmax = oracle_mod.quantize_rowwise(X, O)
    nz = absmax > 0
    assert (np.abs(codes.astype(np.int32)).max(axis=1)[nz] == 127).all()
    assert (codes != -128).all()
    assert not codes[:, O].any()


def test_power_of_two_scaling_invariance(oracle_mod):
    X = make_random((12, 64), seed=51)
    c0, a0 = oracle_mod.quantize_rowwise(X)
    for k in (-3, 1, 4):
        Xs = (X.astype(np.float32) * np.float32(2.0 ** k)).astype(np.float16)
        c, a = oracle_mod.quantize_rowwise(Xs)
        assert np.array_equal(c, c0)
        assert np.array_equal(a, a0 * np.float32(2.0 ** k))


def test_column_permutation_equivariance(oracle_mod):
    X = make_random((10, 64), seed=61, scale=2.5)
    perm = np.random.default_rng(62).permutation(64)
    O = oracle_mod.outlier_mask(X, 6.0)
    Op = oracle_mod.outlier_mask(X[:, perm], 6.0)
    assert np.array_equal(Op, O[perm])
    c, a = oracle_mod.quantize_rowwise(X, O)
    cp, ap = oracle_mod.quantize_rowwise(X[:, perm], Op)
    assert np.array_equal(cp, c[:, perm]) and np.array_equal(ap, a)


def test_brute_force_tiny_workload(oracle_mod):
    """The tiny workload: columns 5 and 37 scaled x20 are the outliers, and Y
    stays within the int8 error bound of the exact fp64 product."""
    from synthetic import TINY, make_problem
    lin = TINY.linears[0]
    X, W, cols = make_problem(lin, seed=0)
    r = oracle_mod.matmul_mixed(X, TINY.threshold, W=W)
    assert r["O"].tolist() == [5, 37]
    exact = X.astype(np.float64) @ W.astype(np.float64).T
    assert np.abs(r["Y"] - exact).max() < 0.05


# ------------------------------------------------------------------ bias and activation after the linear

def test_gelu_tanh_matches_library_routine(oracle_mod):
    """The oracle's BLOOM GELU (page "优化故事：Bloom 推理", section "唾手可得的优化")
    against torch's tanh-approximated GELU, an independent library routine.
    The page writes sqrt(2/pi) as 0.79788456 (torch: 0.7978845608...), a
    relative difference of 1e-9."""
    import torch
    y = np.linspace(-12.0, 12.0, 4801).reshape(1, -1)
    got = oracle_mod.bias_act(y, activation="gelu_tanh")
    ref = torch.nn.functional.gelu(torch.from_numpy(y), approximate="tanh").numpy()
    assert np.all(np.abs(got - ref) <= 1e-8 * (1.0 + np.abs(y)))


def test_gelu_tanh_identities(oracle_mod):
    """g(0) = 0, g(y) - g(-y) = y (tanh is odd), g(y) -> y for large y and
    -> 0 for very negative y."""
    y = np.concatenate([np.linspace(-8, 8, 1601), [0.0, 40.0, -40.0]]).reshape(1, -1)
    g = oracle_mod.bias_act(y, activation="gelu_tanh")[0]
    gm = oracle_mod.bias_act(-y, activation="gelu_tanh")[0]
    assert g[-3] == 0.0
    assert np.all(np.abs((g - gm) - y[0]) <= 1e-12 * (1.0 + np.abs(y[0])))
    assert abs(g[-2] - 40.0) < 1e-12 and abs(g[-1]) < 1e-12


def test_bias_is_added_per_output_feature(oracle_mod):
    """Y = linear + bias[j]: the bias follows the output feature (column of Y)."""
    lin = Linear("b", 6, 40, 64, 2, 20.0)
    X16, _ = make_activations(lin, seed=3)
    W16 = make_weight(lin, seed=4)
    bias = np.random.default_rng(5).standard_normal(40).astype(np.float16)
    r = oracle_mod.matmul_mixed(X16, 6.0, W=W16, bias=bias)
    diff = r["Y"] - r["Y_lin"]
    assert np.allclose(diff, np.broadcast_to(bias.astype(np.float64), diff.shape), rtol=0, atol=1e-12)
    # a per-row (token) bias would be a different matrix
    assert not np.allclose(diff, bias[:6].astype(np.float64)[:, None], atol=1e-3)


# ---- zero-point (unsigned int8) variant: section "模型量化简介" of the page
# "Hugging Face 将 LLM.int8() 8-bit 量化集成进 transformers 与 accelerate" --------

def test_asym_worked_vector_uses_the_full_unsigned_range(oracle_mod):
    """The absmax example vector under zero-point quantization: its minimum
    maps to q = 0 and its maximum to q = 255, and every value comes back
    within half a step (1 / (2 s)) of itself."""
    x = np.array([[1.2, -0.5, -4.3, 1.2, -3.1, 0.8, 2.4, 5.4]], dtype=np.float32)
    c, s, z = oracle_mod.quantize_rowwise_asym(x)
    q = c.astype(np.int32) + 128
    assert q[0, 2] == 0 and q[0, 7] == 255
    back = (q - z[:, None]) / s[:, None].astype(np.float64)
    assert np.all(np.abs(back - x) <= 0.5 / s[0] * (1 + 1e-6))


def test_asym_clamp_catches_the_code_one_past_the_range(oracle_mod):
    """The two separate roundings of the zero-point reading can step past
    [0, 255]: for the row [-1, 1] the range is 2, s = 127.5 exactly,
    z = rint(127.5) = 128 (half to even) and rint(1 * 127.5) = 128, so the
    maximum lands on 128 + 128 = 256 before the clamp. The oracle must count
    exactly that one clamp and store q = 255; the minimum lands on
    rint(-127.5) + 128 = 0 with no clamp. The absmax worked vector needs none."""
    x = np.array([[-1.0, 1.0, 0.0, 0.5]], dtype=np.float32)
    c, s, z, clamped = oracle_mod.quantize_rowwise_asym(x, return_clamped=True)
    q = c.astype(np.int32) + 128
    assert s[0] == np.float32(127.5) and z[0] == 128
    assert clamped == 1
    assert q[0].tolist() == [0, 255, 128, 192]     # 0.5 * 127.5 = 63.75 -> 64, + 128
    w = np.array([[1.2, -0.5, -4.3, 1.2, -3.1, 0.8, 2.4, 5.4]], dtype=np.float32)
    assert oracle_mod.quantize_rowwise_asym(w, return_clamped=True)[3] == 0


def test_asym_zero_is_exact_and_ranges_include_zero(oracle_mod):
    """0 is represented exactly (q = z dequantizes to 0) whatever the signs of
    the row, including all-positive and all-negative rows."""
    rows = np.array([[0.0, 1.5, 3.0, 0.25], [-2.0, -1.0, 0.0, -0.5], [0.0, -3.0, 7.0, 1.0]], dtype=np.float32)
    c, s, z = oracle_mod.quantize_rowwise_asym(rows)
    q = c.astype(np.int32) + 128
    for i in range(3):
        zero_cols = np.flatnonzero(rows[i] == 0)
        assert np.all(q[i, zero_cols] == z[i])
    assert z[0] == 0 and q[0].max() == 255          # non-negative row: lo = 0
    assert z[1] == 255 and q[1].min() == 0          # non-positive row: hi = 0


def test_asym_all_zero_row_and_outlier_columns(oracle_mod):
    """An all-zero row has scale 0; outlier columns carry q = z, so that they
    drop out once the zero point is taken off."""
    x = np.zeros((2, 16), dtype=np.float32)
    x[1] = np.linspace(-1, 2, 16)
    x[1, 5] = 40.0
    c, s, z = oracle_mod.quantize_rowwise_asym(x, outlier=[5])
    assert s[0] == 0 and z[0] == 0
    q = c.astype(np.int32) + 128
    assert q[1, 5] == z[1]
    # the outlier column did not set the range
    assert abs(255.0 / s[1] - 3.0) < 1e-5


def test_asym_linear_equals_the_dequantized_product(oracle_mod):
    """The oracle's asymmetric output, which goes through acc + (128 - z) R,
    equals the fp64 product of the dequantized operands formed directly from
    the codes (x~ = (q - z) / s, w~ = CB * SB / 127) plus the outlier part:
    a dropped or sign-flipped correction term fails here."""
    rng = np.random.default_rng(5)
    X = (rng.standard_normal((9, 48)) + 0.7).astype(np.float16)
    X[:, 11] *= 30
    W = (0.02 * rng.standard_normal((13, 48))).astype(np.float16)
    r = oracle_mod.matmul_mixed_asym(X, 6.0, W=W)
    O = r["O"]
    assert 11 in O
    q = r["CX"].astype(np.float64) + 128
    xt = (q - r["ZX"][:, None]) / r["SXs"].astype(np.float64)[:, None]
    wt = r["CB"].astype(np.float64) * r["SB"].astype(np.float64)[:, None] / 127.0
    keep = np.ones(48, bool)
    keep[O] = False
    ref = xt[:, keep] @ wt[:, keep].T + X.astype(np.float64)[:, O] @ W.astype(np.float64)[:, O].T
    assert np.allclose(r["Y"], ref, rtol=1e-9, atol=1e-9)


def test_asym_error_bound_against_exact_product(oracle_mod):
    """|Y - X W^T| is within the quantization steps of the two operands:
    sum_k |x| * SB / 254 + |w~| / (2 s) per output (plus fp32 slack)."""
    rng = np.random.default_rng(6)
    X = rng.standard_normal((7, 64)).astype(np.float16)
    W = (0.05 * rng.standard_normal((5, 64))).astype(np.float16)
    r = oracle_mod.matmul_mixed_asym(X, 0.0, W=W)
    x = X.astype(np.float64)
    w = W.astype(np.float64)
    wt = r["CB"].astype(np.float64) * r["SB"].astype(np.float64)[:, None] / 127.0
    bound = (np.abs(x) @ (r["SB"].astype(np.float64)[:, None] / 254.0 * np.ones((5, 64))).T
             + (0.5 / r["SXs"].astype(np.float64))[:, None] * np.abs(wt).sum(1)[None, :])
    err = np.abs(r["Y"] - x @ w.T)
    assert np.all(err <= bound * (1 + 1e-4) + 1e-6)
