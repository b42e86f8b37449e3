"""One workspace serves layers of different N in turn.

wq_set_workspace registers a single workspace that every later call uses,
whatever its shape, so a decode step runs its layers (different N) through
the same buffer.  The kernels' ticket counters must therefore sit where no
other shape's partial sums land: the counter region has one size for every
shape (include/wq.h, wq_workspace_bytes).  Here a small layer first fills
the workspace with partial sums through every split-K / stream-K kernel,
then larger layers run through every kernel that takes tickets (their
last-arriver fix-ups, the integer path's grid counter and residual sums)
and must still match the oracle -- the rows at the end of the layer
included, where the integer GEMV's shared row blocks lie -- and leave the
counter region at zero.
"""
import numpy as np
import pytest
import torch

import wq_inputs as gen
import weight_only_quantized_02_b200 as wq
from wqtest_helpers import assert_parity, bf16_dev, dev, oracle_linear, quantize_and_pack, workspace

pytestmark = pytest.mark.gpu

GEMV, GEMM, GEMM_SK, I8, GI, GW4 = (wq.WQ_VARIANT_GEMV, wq.WQ_VARIANT_GEMM, wq.WQ_VARIANT_GEMM_SK,
                                    wq.WQ_VARIANT_I8MMA, wq.WQ_VARIANT_GEMV_I8, wq.WQ_VARIANT_GEMM_W4)
COUNTER_BYTES = 262912  # the fixed counter region at the head of every workspace
K = 1024


def _rows(N):
    return np.unique(np.concatenate([np.arange(0, 64), np.arange(N // 2, N // 2 + 32), np.arange(N - 1024, N)]))


def test_layers_of_different_n_share_one_workspace():
    small8, _ = quantize_and_pack(gen.W_f32(0, 1024, K, seed=1), 8)
    big8, canon8 = quantize_and_pack(gen.W_f32(0, 65536, K, seed=2), 8)
    big4, canon4 = quantize_and_pack(gen.W_f32(0, 65536, K, seed=3), 4)
    ws = workspace(64, K, 65536, 8)
    wq.wq_set_workspace(ws)
    try:
        x = {M: gen.x_bf16(M, K) for M in (4, 16, 64)}
        xd = {M: bf16_dev(v) for M, v in x.items()}

        def dirty():  # the small layer: partial sums all over the workspace
            for M, v, s in ((64, GEMM, 8), (16, GEMM_SK, 1), (4, GEMV, 2), (4, GI, 1), (16, I8, 1)):
                wq.wq_linear_forced(xd[M], small8, v, s)

        for pw, canon, bits, runs in ((big8, canon8, 8, [(4, GI, 1), (4, GI, 2), (16, I8, 1), (4, GEMV, 2),
                                                         (64, GEMM, 4), (16, GEMM_SK, 1)]),
                                      (big4, canon4, 4, [(4, GI, 1), (16, GW4, 1), (64, GW4, 1), (16, I8, 1)])):
            for M, v, s in runs:
                dirty()
                y = torch.full((M, 65536), float("nan"), dtype=torch.bfloat16, device=dev())
                wq.wq_linear_forced(xd[M], pw, v, s, y=y)
                torch.cuda.synchronize()
                rows = _rows(65536)
                got = y[:, torch.from_numpy(rows).to(dev())].float().cpu().numpy().astype(np.float64)
                assert_parity(got, oracle_linear(x[M], canon, bits, rows=rows), f"W{bits} M={M} {v}/{s}")
                assert int(torch.count_nonzero(ws[:COUNTER_BYTES])) == 0, f"counters left set: W{bits} {v}/{s}"
    finally:
        wq.wq_set_workspace(None)
