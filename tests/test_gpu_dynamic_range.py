"""Parity of the integer paths at wide activation dynamic range.

The integer GEMV (GEMV_I8, both launch shapes) and the integer tensor-core
GEMM (I8MMA) write every token row as fixed-point integers X = round(x 2^e)
with |X| < 2^22, so an element far below its row's largest loses bits.  The
exactness guard of those kernels bounds the resulting error of every output
from the row's rounding residual and recomputes in binary64 every output the
bound cannot vouch for.  These tests feed the decode workloads' shapes rows
that defeat the fixed-point form alone:

- N(0,1) rows with one outlier of 2^12, 2^14, 2^15 or 2^16;
- rows mixing one value at bf16's largest normal with N(0,1) values and
  values at its smallest normal, subnormals included;
- rows of values around 2^-100, and a row that is zero but for one element
  at the smallest normal;

and compare every output with the CPU oracle at the layer's tolerance
|y - y_ref| <= 1e-2 max(|y_ref|, 1).  The fixed-point form without the guard
misses that tolerance on the outlier rows (tests/test_exactness_bound.py
shows it on the CPU), so the recompute is what the passing outputs rest on.
"""
import numpy as np
import pytest
import torch

import wq_inputs as gen
import weight_only_quantized_02_b200 as wq
from wqtest_helpers import (assert_parity, bf16_dev, extreme_rows, oracle_linear, outlier_rows, quantize_and_pack,
                            workspace, y_host)

pytestmark = pytest.mark.gpu

I8, GI = wq.WQ_VARIANT_I8MMA, wq.WQ_VARIANT_GEMV_I8

SHAPES = {
    "w8_decode_5120x17408": (8, 5120, 17408),
    "w4g128_decode_5120x25600": (4, 5120, 25600),
    "w8_vocab_5120x152064": (8, 5120, 152064),
}


@pytest.fixture(scope="module", params=list(SHAPES), ids=list(SHAPES))
def layer(request):
    bits, K, N = SHAPES[request.param]
    W = gen.W_f32(0, N, K)
    pw, canon = quantize_and_pack(W, bits)
    del W
    ws = workspace(4, K, N, 32)
    wq.wq_set_workspace(ws)
    yield request.param, bits, K, N, pw, canon
    wq.wq_set_workspace(None)
    del pw, ws
    torch.cuda.empty_cache()


def _integer_cases():
    return [(GI, 1), (GI, 2), (I8, 1), (wq.WQ_VARIANT_AUTO, 0)]


@pytest.mark.parametrize("rows", ["outliers", "extremes"])
def test_integer_paths_wide_range(layer, rows):
    name, bits, K, N, pw, canon = layer
    x = outlier_rows(K) if rows == "outliers" else extreme_rows(K)
    y_ref = oracle_linear(x, canon, bits)
    assert np.isfinite(y_ref).all()
    xd = bf16_dev(x)
    for variant, split in _integer_cases():
        y = wq.wq_linear_forced(xd, pw, variant, split)
        assert_parity(y_host(y), y_ref, f"{name} {rows} variant={variant} split={split}")
        # deterministic: the guard's decisions and recomputes repeat exactly
        y2 = wq.wq_linear_forced(xd, pw, variant, split)
        assert torch.equal(y.view(torch.int16), y2.view(torch.int16)), (variant, split)

