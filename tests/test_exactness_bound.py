"""The integer paths' exactness guard, checked on the CPU.

The integer GEMV and the integer tensor-core GEMM round each token row to
fixed-point integers X = round(x 2^e) (|X| < 2^22; the rounding the library
states in include/wq.h, modelled here by wqtest_helpers.i8_fixed_point).  The
guard in their epilogues relies on

    |y_fixed[m][n] - y_exact[m][n]| <= max_k |w[n][k]| * 2^-e_m * R_m,
    R_m = sum_k |x[m][k] 2^e_m - X[m][k]|,

with max_k |w[n][k]| bounded by 128 s[n] (INT8) or by the largest
max(z, 15 - z) s over the weight (INT4), and recomputes every output whose
bound exceeds 2^-9 max(|y|, 1).  These tests check, against the oracle:
- that the fixed-point form alone misses the layer's tolerance on rows with
  an outlier 2^15 or 2^16 above the rest (so the guard is needed);
- that the bound holds on every output of ordinary, outlier and extreme rows;
- that on ordinary N(0,1) rows the guard never asks for a recompute, and on
  the outlier rows it does.
"""
import numpy as np
import pytest

import oracle
import wq_inputs as gen
from wqtest_helpers import extreme_rows, i8_fixed_point, outlier_rows

TOL = 1.0 / 512.0


def _residual_bound(x_bits):
    """2^-e_m R_m per row, in binary64 (exact: each term is a difference of
    two values on the 2^-e_m grid or finer)."""
    xq, e = i8_fixed_point(x_bits, with_exponents=True)
    x = oracle.bf16_to_f64(x_bits)
    return xq, np.abs(x - xq).sum(axis=1)


@pytest.fixture(scope="module")
def w8():
    K, N = 5120, 17408  # the W8A16 decode layer
    q, s = oracle.quant_int8(gen.W_f32(0, N, K))
    return K, q, s, oracle.dequant_int8(q, s), 128.0 * oracle.bf16_to_f64(s)


@pytest.fixture(scope="module")
def w4():
    K, N = 5120, 4096  # rows of the W4A16 decode layer
    q, s, z = oracle.quant_int4(gen.W_f32(0, N, K))
    zs = np.zeros(s.shape, np.int64)
    for g in range(s.shape[1]):
        zs[:, g] = (z[:, g // 8] >> np.uint32(4 * (g % 8))) & 0xF
    wmax = float(np.max(oracle.bf16_to_f64(s) * np.maximum(zs, 15 - zs)))
    w = oracle.dequant_int4(q, s, z, K)
    assert np.max(np.abs(w)) <= wmax
    return K, (q, s, z), w, np.full(N, wmax)


def _rows(kind, K):
    if kind == "normal":
        return gen.x_bf16(4, K)
    return outlier_rows(K) if kind == "outliers" else extreme_rows(K)


def test_fixed_point_alone_misses_outlier_rows(w8):
    K, q, s, w, _ = w8
    x = outlier_rows(K)
    y_ref = oracle.linear_int8(x, q, s)
    y_fixed = i8_fixed_point(x) @ w.T
    bad = np.abs(y_fixed - y_ref) > 1e-2 * np.maximum(np.abs(y_ref), 1.0)
    assert bad[2:].sum() > 0  # outliers 2^15 and 2^16


@pytest.mark.parametrize("kind", ["normal", "outliers", "extremes"])
def test_bound_holds_int8(w8, kind):
    K, q, s, w, wmax = w8
    x = _rows(kind, K)
    y_ref = oracle.linear_int8(x, q, s)
    xq, rb = _residual_bound(x)
    y_fixed = xq @ w.T
    bound = np.outer(rb, wmax)
    assert np.all(np.abs(y_fixed - y_ref) <= bound * (1 + 1e-12) + 1e-300)
    redo = ~(bound <= TOL * np.maximum(np.abs(y_fixed), 1.0))
    if kind == "normal":
        assert redo.sum() == 0
    else:
        assert redo.sum() > 0
    # every output the guard accepts is within the layer's tolerance after the bf16 rounding
    y_out = np.where(redo, y_ref, oracle.bf16_to_f64(oracle.bf16_rne_of(y_fixed)))
    assert np.all(np.abs(y_out - y_ref) <= 1e-2 * np.maximum(np.abs(y_ref), 1.0))


@pytest.mark.parametrize("kind", ["normal", "outliers"])
def test_bound_holds_int4(w4, kind):
    K, canon, w, wmax = w4
    x = _rows(kind, K)
    y_ref = oracle.linear_int4(x, *canon)
    xq, rb = _residual_bound(x)
    y_fixed = xq @ w.T
    bound = np.outer(rb, wmax)
    assert np.all(np.abs(y_fixed - y_ref) <= bound * (1 + 1e-12) + 1e-300)
    redo = ~(bound <= TOL * np.maximum(np.abs(y_fixed), 1.0))
    assert (redo.sum() == 0) if kind == "normal" else (redo.sum() > 0)
