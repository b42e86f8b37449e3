"""Bit-exact checks of the device quantizers, packers and the packed layout
against the CPU oracle (integer, byte and exact-fp work: no tolerance)."""
import numpy as np
import pytest
import torch

import oracle
import wq_inputs as gen
import weight_only_quantized_02_b200 as wq
from wqtest_helpers import bits_u16, bits_u32, dev, pack_canonical_int4, pack_canonical_int8, to_dev

pytestmark = pytest.mark.gpu


def _adversarial(K, N):
    """Seeded rows that hit the quantizers' corner cases: all-zero, one-signed,
    constant, exact grid values with ties, tiny and heavy-tailed rows."""
    g = gen.generator("misc", 7)
    rows = [
        np.zeros(K, np.float32),
        np.abs(g.normal(0, 0.02, K)).astype(np.float32),
        -np.abs(g.normal(0, 0.02, K)).astype(np.float32),
        np.full(K, 0.01, np.float32),
        (g.integers(-8, 8, K) * 2.0 ** -7).astype(np.float32),
        (g.integers(-127, 128, K) * 2.0 ** -9).astype(np.float32),
        (g.normal(0, 1, K) * 1e-30).astype(np.float32),
        (g.standard_cauchy(K) * 0.01).astype(np.float32),
    ]
    W = gen.W_f32(0, N - len(rows), K)
    return np.concatenate([np.stack(rows), W])


@pytest.mark.parametrize("K,N", [(1024, 64), (5120, 48)])
def test_quantize_int8_bit_exact(K, N):
    W = _adversarial(K, N)
    q, s = wq.wq_quantize_int8(torch.from_numpy(W).to(dev()))
    q_ref, s_ref = oracle.quant_int8(W)
    assert np.array_equal(bits_u16(s), s_ref)
    assert np.array_equal(q.cpu().numpy(), q_ref)


@pytest.mark.parametrize("K,N", [(1024, 64), (17408, 32)])
def test_quantize_int4_bit_exact(K, N):
    W = _adversarial(K, N)
    q, s, z = wq.wq_quantize_int4(torch.from_numpy(W).to(dev()))
    q_ref, s_ref, z_ref = oracle.quant_int4(W)
    assert np.array_equal(bits_u16(s), s_ref)
    assert np.array_equal(bits_u32(z), z_ref)
    assert np.array_equal(bits_u32(q), q_ref)


@pytest.mark.parametrize("K,N", [(1024, 1024), (1120, 400), (96, 16)])
def test_pack_unpack_int8_bit_exact(K, N):
    g = gen.generator("misc", 11)
    q = g.integers(-128, 128, size=(N, K), dtype=np.int8)
    s = gen.f32_to_bf16_bits(g.uniform(1e-3, 2e-2, N).astype(np.float32))
    pw = pack_canonical_int8(q, s)
    assert wq.wq_check_packed(pw) == 0
    qd, _ = wq.wq_unpack_debug(pw)
    assert np.array_equal(qd.cpu().numpy(), oracle.unpack_int8(q.view(np.uint8)).astype(np.int8))
    w = wq.wq_dequant_debug(pw).cpu().numpy()
    w_ref = oracle.dequant_int8(q, s)
    assert np.array_equal(w.astype(np.float64), w_ref)  # s*q is exact in fp32


@pytest.mark.parametrize("K,N", [(1024, 1024), (1152, 400), (128, 16)])
def test_pack_unpack_int4_bit_exact(K, N):
    g = gen.generator("misc", 12)
    q = g.integers(0, 2**32, size=(N, K // 8), dtype=np.uint64).astype(np.uint32)
    s = gen.f32_to_bf16_bits(g.uniform(1e-3, 3e-2, size=(N, K // 128)).astype(np.float32))
    zw = oracle.zero_words_per_row(K)
    z = g.integers(0, 2**32, size=(N, zw), dtype=np.uint64).astype(np.uint32)
    # unused high zero nibbles of the last word are not part of the format
    ng = K // 128
    if ng % 8:
        z[:, -1] &= np.uint32((1 << (4 * (ng % 8))) - 1)
    pw = pack_canonical_int4(q, s, z)
    assert wq.wq_check_packed(pw) == 0
    qd, zd = wq.wq_unpack_debug(pw)
    assert np.array_equal(qd.cpu().numpy().astype(np.uint8), oracle.unpack_int4(q))
    z_ref = oracle.unpack_int4(z)[:, :ng]
    assert np.array_equal(zd.cpu().numpy().astype(np.uint8), z_ref)
    w = wq.wq_dequant_debug(pw).cpu().numpy()
    w_ref = oracle.dequant_int4(q, s, z, K)
    assert np.array_equal(w.astype(np.float64), w_ref)  # s*(q-z) is exact in fp32


def test_trailer_mismatch_is_reported():
    g = gen.generator("misc", 13)
    K, N = 256, 32
    q = g.integers(-127, 128, size=(N, K), dtype=np.int8)
    s = gen.f32_to_bf16_bits(np.full(N, 0.01, np.float32))
    pw = pack_canonical_int8(q, s)
    assert wq.wq_check_packed(pw) == 0
    bad = wq.PackedWeight(pw.wq, pw.scales, None, 8, K, N - 16, 0)
    assert wq.wq_check_packed(bad) == -5  # WQ_ERR_HEADER
    bad = wq.PackedWeight(pw.wq, pw.scales, None, 8, K - 32, N, 0)
    assert wq.wq_check_packed(bad) == -5


def _trailer_word(pw, i):
    """32-bit word i of the 64-byte trailer after the packed weights."""
    wb = pw.wq.numel() - 64
    return int(pw.wq[wb + 4 * i: wb + 4 * i + 4].cpu().numpy().view(np.uint32)[0])


@pytest.mark.parametrize("bits", [8, 4])
def test_trailer_weight_bound(bits):
    """The trailer's bound on max |w| that the integer paths' exactness guard
    reads: INT8 the largest 128 s, INT4 the largest max(z, 15 - z) s of any
    group; either way at least the largest dequantized magnitude."""
    K, N = (1024, 272) if bits == 8 else (1152, 272)
    W = _adversarial(K, N)
    Wd = torch.from_numpy(W).to(dev())
    if bits == 8:
        q, s = wq.wq_quantize_int8(Wd)
        pw = wq.wq_pack_int8(q, s)
        s_h = oracle.bf16_to_f64(bits_u16(s))
        want = np.float32(np.max(128.0 * s_h))
        w = oracle.dequant_int8(q.cpu().numpy(), bits_u16(s))
    else:
        q, s, z = wq.wq_quantize_int4(Wd)
        pw = wq.wq_pack_int4(q, s, z)
        s_h = oracle.bf16_to_f64(bits_u16(s))
        zw = bits_u32(z)
        zs = np.stack([(zw[:, g // 8] >> np.uint32(4 * (g % 8))) & 0xF for g in range(K // 128)], axis=1)
        want = np.float32(np.max(s_h * np.maximum(zs, 15 - zs)))
        w = oracle.dequant_int4(bits_u32(q), bits_u16(s), zw, K)
    got = np.uint32(_trailer_word(pw, 8)).view(np.float32)
    assert got == want
    assert np.max(np.abs(w)) <= float(got)
    assert _trailer_word(pw, 1) == 3  # layout version
