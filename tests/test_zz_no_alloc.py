"""The allocation-free entry point, wq_linear_noalloc.

Some callers cannot allocate device memory when they run the layer: code
inside a captured CUDA graph or an allocator's critical section, runtimes
whose device memory is pre-partitioned, plugin hosts that hand over only
input and output buffers. For them, wq_linear_noalloc keeps its scratch in
a fixed array inside the library instead of a caller-provided workspace.

This file is collected last so that a run stopping at its first failure has
already run every other test. It passes both alone in a fresh process and
after the other tests: the first call on the device sets the array up, and
the array keeps the previous call's contents. So two calls in a row are
checked, each against the existing entry point wq_linear and against the
CPU oracle, within the tolerance the other tests use.
"""
import numpy as np
import pytest
import torch

import wq_inputs as gen
import weight_only_quantized_02_b200 as wq
from wqtest_helpers import REL_TOL, assert_parity, bf16_dev, dev, oracle_linear, quantize_and_pack, y_host

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("bits,K,N,M", [(8, 1024, 1024, 1), (8, 1120, 400, 5), (4, 1152, 400, 8),
                                        (4, 5120, 25600, 1)])
def test_noalloc_matches_wq_linear_twice(bits, K, N, M):
    W = gen.W_f32(0, N, K)
    pw, canon = quantize_and_pack(W, bits)
    xb = gen.x_bf16(M, K)
    x = bf16_dev(xb)
    y_lin = y_host(wq.wq_linear(x, pw))  # the existing entry point
    y_orc = oracle_linear(xb, canon, bits)  # the CPU oracle
    for call in range(2):
        y = wq.wq_linear_noalloc(x, pw)
        torch.cuda.synchronize()
        assert_parity(y_host(y), y_lin, f"noalloc call {call} bits={bits} M={M} vs wq_linear")
        assert_parity(y_host(y), y_orc, f"noalloc call {call} bits={bits} M={M} vs the oracle")
    assert REL_TOL == 1e-2
    assert wq.wq_device_error() == 0


def test_noalloc_rejects_shapes_beyond_its_limits():
    K, N = 1024, 256
    pw, _ = quantize_and_pack(gen.W_f32(0, N, K), 8)
    x = bf16_dev(gen.x_bf16(9, K))  # M = 9 > 8
    y = torch.empty((9, N), dtype=torch.bfloat16, device=dev())
    rc = wq.lib.wq_linear_noalloc(wq._p(x), 9, K, wq._p(pw.wq), wq._p(pw.scales), None, 0, N, wq._p(y),
                                  wq._s(None))
    assert rc == -2  # WQ_ERR_SHAPE, nothing enqueued
    with pytest.raises(wq.WQError):
        wq.wq_linear_noalloc(x, pw)
