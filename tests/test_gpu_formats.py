"""More weight and activation formats: INT4 groups of 32 and 64 k, INT4
with one scale and zero point per channel, and fp16 activations (the
validation matrix of the Marlin register and launch scheduling benchmark,
"Validation and limits": FP16/BF16, INT4/INT8, per-channel and groups
32/64/128).

- The device quantizer and packer are bit-exact with the oracle for every
  group (codes, scales, zero points, unpacked and dequantized weights).
- The layer matches the oracle within |y - y_ref| <= 1e-2 max(|y_ref|, 1)
  on ragged shapes: groups of 32 and 64 through the row-block GEMV (the one
  kernel that reads them, 32 tokens per launch), per-channel INT4 through
  every kernel (stored as group 128 with the row's pair repeated), and fp16
  activations through wq_linear_f16 for INT8 and every INT4 group.
- Closed forms, bit for bit: identity weights give y = x, one-hot
  activations pick the weights, in fp16 as in bf16.
"""
import numpy as np
import pytest
import torch

import oracle
import wq_inputs as gen
import weight_only_quantized_02_b200 as wq
from wqtest_helpers import assert_parity, bf16_dev, bits_u16, bits_u32, dev, to_dev, workspace

pytestmark = pytest.mark.gpu

GEMV, GEMM, GEMV_RB, GEMM_SK, I8, GI, GW4 = (wq.WQ_VARIANT_GEMV, wq.WQ_VARIANT_GEMM, wq.WQ_VARIANT_GEMV_RB,
                                             wq.WQ_VARIANT_GEMM_SK, wq.WQ_VARIANT_I8MMA, wq.WQ_VARIANT_GEMV_I8,
                                             wq.WQ_VARIANT_GEMM_W4)
K4, N4 = 1152, 400  # ragged: 3 full panels + a 16-row tail


def _adversarial(K, N):
    g = gen.generator("misc", 31)
    rows = [np.zeros(K, np.float32), np.abs(g.normal(0, 0.02, K)).astype(np.float32),
            np.full(K, -0.01, np.float32), (g.integers(-8, 8, K) * 2.0 ** -7).astype(np.float32),
            (g.standard_cauchy(K) * 0.01).astype(np.float32)]
    return np.concatenate([np.stack(rows), gen.W_f32(0, N - len(rows), K)])


def _quantize(W, G):
    q, s, z = wq.wq_quantize_int4(torch.from_numpy(W).to(dev()), G)
    return q, s, z, wq.wq_pack_int4(q, s, z, G)


def _f16_dev(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.float16).to(dev())


def _host16(t):
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


@pytest.fixture(scope="module")
def ws():
    t = workspace(128, K4, N4, 32)
    wq.wq_set_workspace(t)
    yield t
    wq.wq_set_workspace(None)


@pytest.mark.parametrize("G", [32, 64, K4])
def test_quantize_pack_bit_exact(G):
    W = _adversarial(K4, N4)
    q, s, z, pw = _quantize(W, G)
    q_ref, s_ref, z_ref = oracle.quant_int4(W, G)
    assert np.array_equal(bits_u32(q), q_ref) and np.array_equal(bits_u16(s), s_ref)
    assert np.array_equal(bits_u32(z), z_ref)
    assert wq.wq_check_packed(pw) == 0
    qd, zd = wq.wq_unpack_debug(pw)
    assert np.array_equal(qd.cpu().numpy(), oracle.unpack_int4(q_ref).astype(np.int8))
    zn = np.stack([(z_ref[:, gi // 8] >> np.uint32(4 * (gi % 8))) & 0xF for gi in range(K4 // G)], axis=1)
    assert np.array_equal(zd.cpu().numpy(), zn.astype(np.int8))
    w = wq.wq_dequant_debug(pw).cpu().numpy().astype(np.float64)
    assert np.array_equal(w, oracle.dequant_int4(q_ref, s_ref, z_ref, K4, G))


def _variants(G, M):
    if G in (32, 64):  # the row-block GEMV, 32 tokens per launch
        return [(GEMV_RB, ks) for ks in (1, 2, 4, 8)]
    out = [(GEMM, 1), (GEMM, 4), (GEMM_SK, 1), (GW4, 1)]  # per channel: every group-128 kernel
    if M <= 32:
        out += [(GEMV, 2), (GEMV_RB, 2)]
    if M <= 32:
        out += [(I8, 1)]
    if M <= 8:
        out += [(GI, 1), (GI, 2)]
    return out


@pytest.mark.parametrize("G", [32, 64, K4])
@pytest.mark.parametrize("M", [1, 7, 32, 33, 100])
def test_groups_and_per_channel_match_oracle(ws, G, M):
    W = gen.W_f32(0, N4, K4)
    q, s, z, pw = _quantize(W, G)
    x = gen.x_bf16(M, K4)
    y_ref = oracle.linear_int4(x, bits_u32(q), bits_u16(s), bits_u32(z), G)
    xd = bf16_dev(x)
    assert_parity(wq.wq_linear(xd, pw).float().cpu().numpy().astype(np.float64), y_ref, f"G={G} M={M} auto")
    for variant, split in _variants(G, M):
        y = wq.wq_linear_forced(xd, pw, variant, split)
        assert_parity(y.float().cpu().numpy().astype(np.float64), y_ref, f"G={G} M={M} {variant}/{split}")


def test_groups_refuse_other_kernels(ws):
    q, s, z, pw = _quantize(gen.W_f32(0, N4, K4), 64)
    x = bf16_dev(gen.x_bf16(4, K4))
    y = torch.empty((4, N4), dtype=torch.bfloat16, device=dev())
    for variant in (GEMM, GEMM_SK, GW4, I8, GI, GEMV):
        assert wq.wq_linear_status(x, pw, y, variant, 1) == -11  # WQ_ERR_VARIANT
    with pytest.raises(wq.WQError):
        wq.wq_linear_noalloc(x, pw)  # the stream-K GEMV reads group 128 only


@pytest.mark.parametrize("fmt", ["w8", 32, 64, 128, K4])
@pytest.mark.parametrize("M", [1, 8, 33])
def test_fp16_activations_match_oracle(fmt, M):
    g = np.random.default_rng(90 + M)
    if fmt == "w8":
        K, N = 1120, N4
        q, s = wq.wq_quantize_int8(torch.from_numpy(gen.W_f32(0, N, K)).to(dev()))
        pw = wq.wq_pack_int8(q, s)
    else:
        K, N = K4, N4
        q, s, z, pw = _quantize(gen.W_f32(0, N, K), fmt)
    xh = g.normal(0, 1, (M, K)).astype(np.float16).view(np.uint16)
    y = wq.wq_linear_f16(_f16_dev(xh), pw)
    assert y.dtype == torch.float16
    if fmt == "w8":
        y_ref = oracle.linear_int8(xh, q.cpu().numpy(), bits_u16(s), act="fp16")
    else:
        y_ref = oracle.linear_int4(xh, bits_u32(q), bits_u16(s), bits_u32(z), fmt, act="fp16")
    assert_parity(oracle.f16_to_f64(_host16(y)), y_ref, f"fp16 {fmt} M={M}")


def test_fp16_closed_forms():
    """Identity INT4 weights (q = 9 on the diagonal, 8 elsewhere, z = 8,
    s = 1) give y = x exactly; one-hot fp16 activations pick each weight
    s (q - z), rounded once to fp16."""
    K = N = 256
    qn = np.full((N, K), 8, np.uint32)
    np.fill_diagonal(qn, 9)
    qw = np.zeros((N, K // 8), np.uint32)
    for k in range(K):
        qw[:, k // 8] |= qn[:, k] << np.uint32(4 * (k % 8))
    for G in (32, 64, 128):
        z = np.zeros((N, oracle.zero_words_per_row(K, G)), np.uint32)
        for gi in range(K // G):
            z[:, gi // 8] |= np.uint32(8) << np.uint32(4 * (gi % 8))
        pw = wq.wq_pack_int4(to_dev(qw), to_dev(np.full((N, K // G), 0x3F80, np.uint16)), to_dev(z), G)
        xh = np.random.default_rng(G).normal(0, 1, (5, K)).astype(np.float16).view(np.uint16)
        y = _host16(wq.wq_linear_f16(_f16_dev(xh), pw))
        assert np.array_equal(y, xh), G
    # one-hot activations on quantized weights: y[m][n] = fp16(w[n][k_m])
    W = gen.W_f32(0, N4, K4)
    q, s, z, pw = _quantize(W, 64)
    ks = [0, 63, 64, 1151]
    xh = np.zeros((len(ks), K4), np.uint16)
    for m, k in enumerate(ks):
        xh[m, k] = 0x3C00  # fp16 1.0
    w = oracle.dequant_int4(bits_u32(q), bits_u16(s), bits_u32(z), K4, 64)
    want = oracle.f64_to_f16(w[:, ks].T)
    assert np.array_equal(_host16(wq.wq_linear_f16(_f16_dev(xh), pw)), want)
