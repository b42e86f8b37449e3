"""The larger-M regime: wq_linear with more than 128 tokens (prefill chunks).

wq_linear runs M > 128 as consecutive chunks of 128 tokens, one kernel per
chunk, each chosen by the dispatcher for its own size (a ragged last chunk
can take another kernel).  These tests compare every output with the CPU
oracle at M = 129, 256, 512 and 2048 on shapes with ragged panels, through
the dispatcher and through every variant valid for a 128-token chunk, and
the W4A16 17408 x 5120 layer at M = 256 on sampled output channels.
Tolerance: |y - y_ref| <= 1e-2 max(|y_ref|, 1).
"""
import numpy as np
import pytest
import torch

import oracle
import wq_inputs as gen
import weight_only_quantized_02_b200 as wq
from wqtest_helpers import (assert_parity, bf16_dev, bits_u16, bits_u32, dev, oracle_linear, quantize_and_pack,
                            workspace, y_host)

pytestmark = pytest.mark.gpu

GEMM, GEMM_SK, GW4 = wq.WQ_VARIANT_GEMM, wq.WQ_VARIANT_GEMM_SK, wq.WQ_VARIANT_GEMM_W4
SHAPES = {8: (1120, 400), 4: (1152, 400)}


@pytest.fixture(scope="module", params=[8, 4], ids=["w8", "w4g128"])
def weight(request):
    bits = request.param
    K, N = SHAPES[bits]
    pw, canon = quantize_and_pack(gen.W_f32(0, N, K), bits)
    ws = workspace(2048, K, N, 32)
    wq.wq_set_workspace(ws)
    yield bits, K, N, pw, canon
    wq.wq_set_workspace(None)


@pytest.mark.parametrize("M", [129, 256, 512, 2048])
def test_large_m_matches_oracle(weight, M):
    bits, K, N, pw, canon = weight
    x = gen.x_bf16(M, K)
    y_ref = oracle_linear(x, canon, bits)
    xd = bf16_dev(x)
    assert_parity(y_host(wq.wq_linear(xd, pw)), y_ref, f"bits={bits} M={M} auto")
    cases = [(GEMM, 1), (GEMM, 4), (GEMM_SK, 1)] + ([(GW4, 1)] if bits == 4 else [])
    for variant, split in cases:
        y = wq.wq_linear_forced(xd, pw, variant, split)
        assert_parity(y_host(y), y_ref, f"bits={bits} M={M} variant={variant} split={split}")
    torch.cuda.synchronize()
    assert wq.wq_device_error() == 0


def test_large_m_limits(weight):
    bits, K, N, pw, canon = weight
    # the tuner and the table work on the chunk shape
    assert wq.wq_get_choice(300, K, N, bits, pw.group) == wq.wq_get_choice(128, K, N, bits, pw.group)
    # a variant that does not fit a 128-token chunk is refused before anything runs
    x = bf16_dev(gen.x_bf16(200, K))
    y = torch.empty((200, N), dtype=torch.bfloat16, device=dev())
    assert wq.wq_linear_status(x, pw, y, wq.WQ_VARIANT_GEMV_I8, 1) == -11  # WQ_ERR_VARIANT
    # beyond the largest M: WQ_ERR_SHAPE
    big = torch.empty((65537, 16), dtype=torch.bfloat16, device=dev())
    assert int(wq.lib.wq_linear(wq._p(big), 65537, K, wq._p(pw.wq), wq._p(pw.scales), wq._p(pw.zeros),
                                pw.group, N, wq._p(big), wq._s(None))) == -2


def test_prefill_layer_sampled():
    """The W4A16 17408 x 5120 layer at M = 256 (two chunks), on sampled
    output channels the oracle recomputes from its own quantization of the
    regenerated source rows (codes checked bit for bit)."""
    cfg = gen.workload("w4g128_prefill_17408x5120")
    K, N = cfg["K"], cfg["N"]
    W = torch.from_numpy(gen.W_f32(0, N, K)).to(dev())
    q, s, z = wq.wq_quantize_int4(W)
    pw = wq.wq_pack_int4(q, s, z)
    del W
    rows = gen.sample_rows(N, 64)
    q_ref, s_ref, z_ref = oracle.quant_int4(gen.W_rows(rows, K))
    idx = torch.from_numpy(rows).to(dev())
    assert np.array_equal(bits_u32(q.index_select(0, idx)), q_ref)
    assert np.array_equal(bits_u16(s.index_select(0, idx)), s_ref)
    assert np.array_equal(bits_u32(z.index_select(0, idx)), z_ref)
    ws = workspace(256, K, N, 32)
    wq.wq_set_workspace(ws)
    try:
        M = 256
        x = gen.x_bf16(M, K)
        y_ref = oracle.linear_int4(x, q_ref, s_ref, z_ref)
        y = wq.wq_linear(bf16_dev(x), pw)
        assert_parity(y_host(y.index_select(1, idx)), y_ref, "prefill M=256")
        assert torch.isfinite(y.float()).all()
    finally:
        wq.wq_set_workspace(None)
