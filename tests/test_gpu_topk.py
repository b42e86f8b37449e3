"""The vocabulary head's top-k (wq_linear_topk) against the layer and the oracle.

For every token row the call returns the k largest bf16 logits, descending,
and their indices, the lower index first among equal logits.  Checks:
- bit for bit against the top-k the host takes of the layer's own bf16
  logits (wq_linear, the same dispatcher choice): the selection adds no
  error and its tie rule makes the answer unique;
- against the CPU oracle: every returned logit is within the layer's
  tolerance of the oracle's value at its index, and no logit left out is
  larger than a returned one by more than the two tolerances (the set is a
  valid top-k of the exact logits);
- on the vocabulary-head shape 5120 x 152064 with INT8 per-channel and INT4
  group-128 heads, on ragged small shapes, on all-equal logits, and the
  argument limits.
"""
import numpy as np
import pytest
import torch

import oracle
import wq_inputs as gen
import weight_only_quantized_02_b200 as wq
from wqtest_helpers import bf16_dev, bits_u16, dev, oracle_linear, pack_canonical_int8, quantize_and_pack, workspace

pytestmark = pytest.mark.gpu


def host_topk(y_bits: np.ndarray, k: int):
    """Top-k of bf16 logits [M][N]: value descending, then index ascending."""
    y = oracle.bf16_to_f64(y_bits)
    vals, idx = [], []
    for m in range(y.shape[0]):
        order = np.lexsort((np.arange(y.shape[1]), -y[m]))[:k]
        idx.append(order)
        vals.append(y_bits[m, order])
    return np.array(vals, np.uint16), np.array(idx, np.int32)


def check_valid(vals_bits, idx, y_ref):
    v = oracle.bf16_to_f64(vals_bits)
    tol = lambda a: 1e-2 * np.maximum(np.abs(a), 1.0)  # noqa: E731
    for m in range(y_ref.shape[0]):
        ref_at = y_ref[m, idx[m]]
        assert np.all(np.abs(v[m] - ref_at) <= tol(ref_at)), m
        rest = np.ones(y_ref.shape[1], bool)
        rest[idx[m]] = False
        worst = np.argmin(ref_at)
        bound = ref_at[worst] + tol(ref_at[worst]) + tol(y_ref[m, rest])
        assert np.all(y_ref[m, rest] <= bound), m


def _run(pw, x_bits, k):
    M, N = x_bits.shape[0], pw.N
    ws = torch.zeros(wq.wq_topk_workspace_bytes(M, N, k), dtype=torch.uint8, device=dev())
    xd = bf16_dev(x_bits)
    vals, idx = wq.wq_linear_topk(xd, pw, k, ws)
    logits = wq.wq_linear(xd, pw)
    torch.cuda.synchronize()
    return bits_u16(vals.view(torch.int16)), idx.cpu().numpy(), bits_u16(logits.view(torch.int16))


@pytest.fixture(scope="module", params=[8, 4], ids=["int8_head", "int4g128_head"])
def head(request):
    bits = request.param
    K, N = 5120, 152064
    pw, canon = quantize_and_pack(gen.W_f32(0, N, K), bits)
    ws = workspace(16, K, N, 32)
    wq.wq_set_workspace(ws)
    yield bits, K, N, pw, canon
    wq.wq_set_workspace(None)
    del pw, ws
    torch.cuda.empty_cache()


@pytest.mark.parametrize("M,k", [(1, 1), (1, 64), (4, 8), (16, 64)])
def test_head_topk(head, M, k):
    bits, K, N, pw, canon = head
    x = gen.x_bf16(M, K)
    vals, idx, logits = _run(pw, x, k)
    hv, hi = host_topk(logits, k)
    assert np.array_equal(vals, hv) and np.array_equal(idx, hi)
    assert np.all(np.diff(oracle.bf16_to_f64(vals), axis=1) <= 0)
    if M <= 4:
        check_valid(vals, idx, oracle_linear(x, canon, bits))
    else:  # the oracle at the returned indices only
        rows = np.unique(idx)
        ref = oracle_linear(x, canon, bits, rows=rows)
        pos = {int(r): i for i, r in enumerate(rows)}
        v = oracle.bf16_to_f64(vals)
        for m in range(M):
            ref_at = ref[m, [pos[int(i)] for i in idx[m]]]
            assert np.all(np.abs(v[m] - ref_at) <= 1e-2 * np.maximum(np.abs(ref_at), 1.0))


@pytest.mark.parametrize("bits", [8, 4])
@pytest.mark.parametrize("M,k", [(1, 1), (3, 7), (9, 64), (33, 17)])
def test_small_ragged_topk(bits, M, k):
    K, N = (1120, 400) if bits == 8 else (1152, 400)
    pw, canon = quantize_and_pack(gen.W_f32(0, N, K), bits)
    ws = workspace(64, K, N, 32)
    wq.wq_set_workspace(ws)
    try:
        x = gen.x_bf16(M, K)
        vals, idx, logits = _run(pw, x, k)
        hv, hi = host_topk(logits, k)
        assert np.array_equal(vals, hv) and np.array_equal(idx, hi)
        check_valid(vals, idx, oracle_linear(x, canon, bits))
    finally:
        wq.wq_set_workspace(None)


def test_equal_logits_take_the_lowest_indices():
    K, N, M, k = 256, 96, 2, 20
    pw = pack_canonical_int8(np.zeros((N, K), np.int8), np.full(N, 0x3C00, np.uint16))  # every logit 0
    vals, idx, _ = _run(pw, gen.x_bf16(M, K), k)
    assert np.all(oracle.bf16_to_f64(vals) == 0.0)
    assert np.array_equal(idx, np.tile(np.arange(k, dtype=np.int32), (M, 1)))


def test_topk_limits():
    K, N = 256, 96
    pw = pack_canonical_int8(np.ones((N, K), np.int8), np.full(N, 0x3C00, np.uint16))
    x = bf16_dev(gen.x_bf16(2, K))
    assert wq.wq_topk_workspace_bytes(2, N, 0) == 0 and wq.wq_topk_workspace_bytes(2, N, 65) == 0
    assert wq.wq_topk_workspace_bytes(2, 40, 41) == 0 and wq.wq_topk_workspace_bytes(129, N, 4) == 0
    ws = torch.zeros(wq.wq_topk_workspace_bytes(2, N, 4), dtype=torch.uint8, device=dev())
    for k, st in [(0, -2), (65, -2), (N + 1, -2)]:
        with pytest.raises(wq.WQError) as e:
            wq.wq_linear_topk(x, pw, k, ws)
        assert e.value.status == st
    with pytest.raises(wq.WQError) as e:
        wq.wq_linear_topk(x, pw, 8, ws[:64])
    assert e.value.status == -6  # WQ_ERR_WORKSPACE
