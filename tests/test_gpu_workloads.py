"""The decode workloads at their full sizes, in the launch configurations the
benchmark times.

Inputs are the seeded synthetic tensors of ``wq_inputs``.  The oracle cannot
afford every output at these sizes, so it recomputes a sample of output
channels (first, last, panel edges and random ones): it regenerates those
rows of the fp32 source weights from their own counter-addressed streams,
quantizes them itself, checks that the device produced the same codes bit for
bit, and evaluates those outputs in fp64.
"""
import numpy as np
import pytest
import torch

import oracle
import wq_inputs as gen
import weight_only_quantized_02_b200 as wq
from wqtest_helpers import assert_parity, bf16_dev, bits_u16, bits_u32, dev, workspace, y_host

pytestmark = pytest.mark.gpu

GEMV, GEMM, GEMV_RB, GEMM_SK, I8, GI = (wq.WQ_VARIANT_GEMV, wq.WQ_VARIANT_GEMM, wq.WQ_VARIANT_GEMV_RB,
                                        wq.WQ_VARIANT_GEMM_SK, wq.WQ_VARIANT_I8MMA, wq.WQ_VARIANT_GEMV_I8)
GW4 = wq.WQ_VARIANT_GEMM_W4


def _build(name):
    cfg = gen.WORKLOADS[name]
    K, N, bits = cfg["K"], cfg["N"], cfg["bits"]
    if cfg.get("direct"):
        q, s = gen.direct_int8(K, N)
        pw = wq.wq_pack_int8(torch.from_numpy(q).to(dev()), torch.from_numpy(s.view(np.int16)).to(dev()))
        return cfg, pw, ("direct", q, s)
    W = torch.from_numpy(gen.W_f32(0, N, K)).to(dev())
    if bits == 8:
        q, s = wq.wq_quantize_int8(W)
        pw = wq.wq_pack_int8(q, s)
        dev_codes = (q, s)
    else:
        q, s, z = wq.wq_quantize_int4(W)
        pw = wq.wq_pack_int4(q, s, z)
        dev_codes = (q, s, z)
    del W
    torch.cuda.empty_cache()
    return cfg, pw, ("quantized", dev_codes)


def _oracle_rows(cfg, src, rows):
    """Oracle codes for the sampled rows, checked bit-exact against the device's."""
    K, bits = cfg["K"], cfg["bits"]
    if src[0] == "direct":
        return (src[1][rows], src[2][rows])
    Wr = gen.W_rows(rows, K)
    idx = torch.from_numpy(rows).to(dev())
    if bits == 8:
        q_ref, s_ref = oracle.quant_int8(Wr)
        q_d, s_d = src[1]
        assert np.array_equal(q_d.index_select(0, idx).cpu().numpy(), q_ref)
        assert np.array_equal(bits_u16(s_d.index_select(0, idx)), s_ref)
        return (q_ref, s_ref)
    q_ref, s_ref, z_ref = oracle.quant_int4(Wr)
    q_d, s_d, z_d = src[1]
    assert np.array_equal(bits_u32(q_d.index_select(0, idx)), q_ref)
    assert np.array_equal(bits_u16(s_d.index_select(0, idx)), s_ref)
    assert np.array_equal(bits_u32(z_d.index_select(0, idx)), z_ref)
    return (q_ref, s_ref, z_ref)


def _ref(cfg, x, codes):
    if cfg["bits"] == 8:
        return oracle.linear_int8(x, codes[0], codes[1])
    return oracle.linear_int4(x, codes[0], codes[1], codes[2])


def _variants(M, K, bits):
    out = []
    if M <= 32:
        out += [(GEMV, c) for c in (1, 2, 3)]
        out += [(GEMV_RB, ks) for ks in (1, 2, 4, 8)]
    out += [(GEMM, s) for s in (1, 2, 4, 8, 16, 32) if s <= (K + 127) // 128]
    out += [(GEMM_SK, c) for c in (1, 2)]
    if M <= (64 if bits == 8 else 32):  # integer tensor-core path: W8A16 M <= 64, W4A16 M <= 32
        out += [(I8, 1)]
    if M <= 8:  # integer GEMV
        out += [(GI, c) for c in (1, 2)]
    if bits == 4:  # role-split W4A16 GEMM
        out += [(GW4, 1)]
    return out


@pytest.mark.parametrize("name", list(gen.WORKLOADS))
def test_workload_full_size(name):
    cfg, pw, src = _build(name)
    K, N = cfg["K"], cfg["N"]
    assert wq.wq_check_packed(pw) == 0
    rows = gen.sample_rows(N, 96)
    codes = _oracle_rows(cfg, src, rows)
    Mmax = max(cfg["Ms"])
    ws = workspace(Mmax, K, N, 32)
    wq.wq_set_workspace(ws)
    idx = torch.from_numpy(rows).to(dev())
    try:
        for M in cfg["Ms"]:
            x = gen.x_bf16(M, K)
            y_ref = _ref(cfg, x, codes)
            xd = bf16_dev(x)
            y = torch.empty((M, N), dtype=torch.bfloat16, device=dev())
            for variant, split in _variants(M, K, cfg["bits"]):
                wq.wq_linear_forced(xd, pw, variant, split, y=y)
                assert_parity(y_host(y.index_select(1, idx)), y_ref, f"{name} M={M} {variant}/{split}")
            y.zero_()
            wq.wq_linear(xd, pw, y=y)
            assert_parity(y_host(y.index_select(1, idx)), y_ref, f"{name} M={M} auto")
            # property at any size: every output is finite and was written
            assert torch.isfinite(y.float()).all()
        torch.cuda.synchronize()
        assert wq.wq_device_error() == 0
    finally:
        wq.wq_set_workspace(None)
