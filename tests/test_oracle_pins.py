"""Pins of the CPU oracle against things other than itself (CPU only).

The pages print no worked example, so each part of the oracle is pinned by
hand-derived fixtures (tests/golden), closed forms, special cases, exact
rational brute force, library routines (torch's fp32 -> bf16 conversion,
numpy's fp64 matmul) and invariants.  A plausible mistake anywhere in the
oracle -- a dropped zero point, a wrong group index, a transposed operand, a
swapped nibble order, double rounding in the output conversion -- fails at
least one test here.
"""
import os
import struct
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
import wq_inputs as gen

pytestmark = pytest.mark.filterwarnings("ignore::DeprecationWarning")


def f32_from_bits(u):
    return struct.unpack("<f", struct.pack("<I", u))[0]


def bf16_bits_to_fraction(b):
    return Fraction(f32_from_bits(int(b) << 16))


# ---------------------------------------------------------------------------
# bf16 rounding
# ---------------------------------------------------------------------------

def _read_rows(path, maxsplit=-1):
    rows = []
    for line in open(path):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        rows.append([p.strip() for p in line.split(";", maxsplit)])
    return rows


def test_bf16_rounding_hand_fixture(golden_dir):
    for v, mode, want, _why in _read_rows(os.path.join(golden_dir, "bf16_rounding.txt"), 3):
        got = oracle.f64_to_bf16(np.array([float.fromhex(v)]), mode)[0]
        assert got == int(want, 16), (v, mode, hex(got), want)


def test_bf16_rne_matches_torch_on_fp32_values():
    """torch's fp32 -> bf16 conversion is an independent RNE implementation;
    every fp32 value is exactly a binary64 value."""
    g = np.random.default_rng(1)
    bits = g.integers(0, 2**32, size=200000, dtype=np.uint64).astype(np.uint32)
    f = bits.view(np.float32)
    f = f[np.isfinite(f)]
    # add every midpoint of a sample of bf16 neighbours, plus tiny/huge values
    b = g.integers(0, 0x7F7F, size=20000, dtype=np.uint32)
    mids = ((b << 16) | 0x8000).view(np.float32)
    extra = np.array([0.0, -0.0, 1e-45, -1e-45, 3.3e38, -3.3e38, 1.0, -1.0], np.float32)
    f = np.concatenate([f, mids, -mids, extra])
    want = torch.from_numpy(f.copy()).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = oracle.f64_to_bf16(f.astype(np.float64), "rne")
    assert np.array_equal(got, want)


def test_bf16_roundtrip_every_pattern():
    pats = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    vals = oracle.bf16_to_f64(pats)
    ref = torch.from_numpy(pats.view(np.int16).copy()).view(torch.bfloat16).to(torch.float64).numpy()
    finite = np.isfinite(ref)
    assert np.array_equal(vals[finite], ref[finite])
    back = oracle.f64_to_bf16(vals[finite], "rne")
    assert np.array_equal(back, pats[finite])


def test_bf16_round_up_is_ceiling():
    g = np.random.default_rng(2)
    v = np.concatenate([g.uniform(1e-6, 1.0, 20000), 10.0 ** g.uniform(-30, 30, 20000)])
    up = oracle.f64_to_bf16(v, "up")
    upv = oracle.bf16_to_f64(up)
    prev = oracle.bf16_to_f64((up.astype(np.int32) - 1).astype(np.uint16))
    assert np.all(upv >= v)
    assert np.all(prev < v)
    exact = oracle.bf16_to_f64(oracle.f64_to_bf16(v, "rne"))
    assert np.array_equal(oracle.f64_to_bf16(exact, "up"), oracle.f64_to_bf16(exact, "rne"))


# ---------------------------------------------------------------------------
# unpack
# ---------------------------------------------------------------------------

def test_unpack_int4_hand_words(golden_dir):
    for word, elems in _read_rows(os.path.join(golden_dir, "unpack_int4_words.txt")):
        got = oracle.unpack_int4(np.array([int(word, 16)], np.uint32))
        assert got.tolist() == [int(e) for e in elems.split()], word


def test_unpack_int8_two_complement():
    b = np.array([0x00, 0x01, 0x7F, 0x80, 0x81, 0xFF, 0xFE], np.uint8)
    assert oracle.unpack_int8(b).tolist() == [0, 1, 127, -128, -127, -1, -2]


def test_unpack_int4_roundtrip_numpy_pack():
    g = np.random.default_rng(3)
    q = g.integers(0, 16, size=(7, 64), dtype=np.uint32)
    # pack element k = 8c + j into nibble j of word c
    words = np.zeros((7, 8), np.uint32)
    for k in range(64):
        words[:, k // 8] |= q[:, k] << np.uint32(4 * (k % 8))
    assert np.array_equal(oracle.unpack_int4(words).astype(np.uint32), q)


# ---------------------------------------------------------------------------
# quantizers + dequant, hand-derived
# ---------------------------------------------------------------------------

def _parse_kv(field, conv):
    out = {}
    for tok in field.split()[1:]:
        k, v = tok.split(":")
        out[k] = conv(v)
    return out


def test_int8_quant_and_dequant_by_hand(golden_dir):
    K = 32
    for row in _read_rows(os.path.join(golden_dir, "int8_quant_by_hand.txt")):
        name, s_f, W_f, q_f, w_f = row
        W = np.zeros((1, K), np.float32)
        for k, v in _parse_kv(W_f, lambda v: int(v, 16)).items():
            W[0, int(k)] = f32_from_bits(v)
        q, s = oracle.quant_int8(W)
        assert s[0] == int(s_f.split()[1], 16), name
        want_q = np.zeros(K, np.int8)
        for k, v in _parse_kv(q_f, int).items():
            want_q[int(k)] = v
        assert np.array_equal(q[0], want_q), name
        w = oracle.dequant_int8(q, s)
        want_w = np.zeros(K)
        for k, v in _parse_kv(w_f, float).items():
            want_w[int(k)] = v
        assert np.array_equal(w[0], want_w), name


def test_int4_quant_and_dequant_by_hand(golden_dir):
    G = 128
    rows = _read_rows(os.path.join(golden_dir, "int4_quant_by_hand.txt"))
    K = G * len(rows)
    W = np.zeros((1, K), np.float32)
    want_s, want_z, want_q, want_w = [], [], np.zeros(K, np.uint8), np.zeros(K)
    for g, (name, s_f, z_f, W_f, q_f, w_f) in enumerate(rows):
        for k, v in _parse_kv(W_f, lambda v: int(v, 16)).items():
            W[0, g * G + int(k)] = f32_from_bits(v)
        want_s.append(int(s_f.split()[1], 16))
        want_z.append(int(z_f.split()[1]))
        qd = _parse_kv(q_f, int)
        wd = _parse_kv(w_f, float)
        for k in range(G):
            want_q[g * G + k] = qd.get(str(k), qd.get("rest"))
            want_w[g * G + k] = wd.get(str(k), wd.get("rest"))
    q, s, z = oracle.quant_int4(W, G)
    assert s[0].tolist() == want_s
    assert oracle.unpack_int4(z)[0][: len(rows)].tolist() == want_z
    assert np.array_equal(oracle.unpack_int4(q)[0], want_q)
    w = oracle.dequant_int4(q, s, z, K, G)
    assert np.array_equal(w[0], want_w)


# ---------------------------------------------------------------------------
# invariants of the quantizers: |s (q - z) - W| <= s/2
# ---------------------------------------------------------------------------

def _adversarial_rows(K):
    g = np.random.default_rng(5)
    rows = [
        np.zeros(K, np.float32),                        # degenerate: all zero
        np.abs(g.normal(0, 0.02, K)).astype(np.float32),   # all >= 0 (lo = 0)
        -np.abs(g.normal(0, 0.02, K)).astype(np.float32),  # all <= 0 (hi = 0)
        np.full(K, 0.01, np.float32),                   # constant
        (g.integers(-8, 8, K) * 2.0 ** -7).astype(np.float32),  # exact grid, ties likely
        (g.normal(0, 1, K) * 1e-30).astype(np.float32),  # tiny scale
        (g.standard_cauchy(K) * 0.01).astype(np.float32),  # heavy tails
    ]
    return np.stack(rows)


@pytest.mark.parametrize("K", [128, 1024])
def test_quant_int8_error_bound(K):
    W = np.concatenate([gen.W_f32(0, 64, K), _adversarial_rows(K)])
    q, s = oracle.quant_int8(W)
    sd = oracle.bf16_to_f64(s)
    w = oracle.dequant_int8(q, s)
    err = np.abs(w - W.astype(np.float64))
    bound = sd[:, None] / 2 * (1 + 2.0 ** -40)
    ok = (err <= bound) | (sd[:, None] == 0) & (W == 0)
    assert np.all(ok)
    assert np.all(np.abs(q) <= 127)


@pytest.mark.parametrize("K", [128, 1024])
def test_quant_int4_error_bound(K):
    G = 128
    W = np.concatenate([gen.W_f32(0, 64, K), _adversarial_rows(K)])
    q, s, z = oracle.quant_int4(W, G)
    w = oracle.dequant_int4(q, s, z, K, G)
    sd = np.repeat(oracle.bf16_to_f64(s), G, axis=1)
    err = np.abs(w - W.astype(np.float64))
    ok = (err <= sd / 2 * (1 + 2.0 ** -40)) | ((sd == 0) & (W == 0))
    assert np.all(ok)
    qn = oracle.unpack_int4(q)
    assert qn.max() <= 15


# ---------------------------------------------------------------------------
# linear: exact rational brute force on tiny shapes
# ---------------------------------------------------------------------------

def _rand_int4(g, N, K, G):
    q = g.integers(0, 2**32, size=(N, K // 8), dtype=np.uint64).astype(np.uint32)
    s = gen.f32_to_bf16_bits(g.uniform(1e-3, 3e-2, size=(N, K // G)).astype(np.float32))
    zw = oracle.zero_words_per_row(K, G)
    z = g.integers(0, 2**32, size=(N, zw), dtype=np.uint64).astype(np.uint32)
    return q, s, z


def _exact_int4(x, q, s, z, G):
    """Exact rational evaluation of the definition, element by element."""
    M, K = x.shape
    N = q.shape[0]
    xf = [[bf16_bits_to_fraction(x[m, k]) for k in range(K)] for m in range(M)]
    out = [[Fraction(0)] * N for _ in range(M)]
    for n in range(N):
        w = []
        for k in range(K):
            qn = (int(q[n, k // 8]) >> (4 * (k % 8))) & 15
            gidx = k // G
            zn = (int(z[n, gidx // 8]) >> (4 * (gidx % 8))) & 15
            w.append(bf16_bits_to_fraction(s[n, gidx]) * (qn - zn))
        for m in range(M):
            out[m][n] = sum(xf[m][k] * w[k] for k in range(K))
    return out


def _exact_int8(x, q, s):
    M, K = x.shape
    N = q.shape[0]
    out = [[Fraction(0)] * N for _ in range(M)]
    for n in range(N):
        sn = bf16_bits_to_fraction(s[n])
        for m in range(M):
            out[m][n] = sum(bf16_bits_to_fraction(x[m, k]) * sn * int(q[n, k]) for k in range(K))
    return out


def _check_against_exact(y, exact, x, wabs_sum):
    M, N = y.shape
    K = x.shape[1]
    for m in range(M):
        for n in range(N):
            bound = K * 2.0 ** -53 * wabs_sum[m, n] * 1.01
            assert abs(Fraction(y[m, n]) - exact[m][n]) <= Fraction(bound), (m, n)


@pytest.mark.parametrize("M,K,N", [(1, 128, 8), (2, 256, 16), (3, 256, 8)])
def test_linear_int4_exact_bruteforce(M, K, N):
    g = np.random.default_rng(10 + M)
    G = 128
    x = gen.f32_to_bf16_bits(g.normal(0, 1, (M, K)).astype(np.float32))
    q, s, z = _rand_int4(g, N, K, G)
    y = oracle.linear_int4(x, q, s, z, G)
    exact = _exact_int4(x, q, s, z, G)
    w = oracle.dequant_int4(q, s, z, K, G)
    absw = np.abs(oracle.bf16_to_f64(x)) @ np.abs(w).T
    _check_against_exact(y, exact, x, absw)


@pytest.mark.parametrize("M,K,N", [(1, 32, 8), (2, 64, 16), (3, 96, 8)])
def test_linear_int8_exact_bruteforce(M, K, N):
    g = np.random.default_rng(20 + M)
    x = gen.f32_to_bf16_bits(g.normal(0, 1, (M, K)).astype(np.float32))
    q = g.integers(-128, 128, size=(N, K), dtype=np.int8)
    s = gen.f32_to_bf16_bits(g.uniform(1e-3, 2e-2, N).astype(np.float32))
    y = oracle.linear_int8(x, q, s)
    exact = _exact_int8(x, q, s)
    w = oracle.dequant_int8(q, s)
    absw = np.abs(oracle.bf16_to_f64(x)) @ np.abs(w).T
    _check_against_exact(y, exact, x, absw)


def test_linear_matches_numpy_matmul():
    """Library fp64 matmul (BLAS, different summation order) on the oracle's
    own dequantized weights: within the fp64 error bound."""
    g = np.random.default_rng(30)
    M, K, N, G = 4, 1024, 64, 128
    x = gen.x_bf16(M, K)
    q, s, z = _rand_int4(g, N, K, G)
    y = oracle.linear_int4(x, q, s, z, G)
    # independent unpack + dequant with numpy bit operations
    shifts = np.uint32(4) * np.arange(8, dtype=np.uint32)
    qn = ((q[:, :, None] >> shifts) & np.uint32(15)).reshape(N, K).astype(np.float64)
    zn = ((z[:, :, None] >> shifts) & np.uint32(15)).reshape(N, -1)[:, : K // G].astype(np.float64)
    sd = torch.from_numpy(s.view(np.int16).copy()).view(torch.bfloat16).double().numpy()
    w = np.repeat(sd, G, axis=1) * (qn - np.repeat(zn, G, axis=1))
    xd = torch.from_numpy(x.view(np.int16).copy()).view(torch.bfloat16).double().numpy()
    ref = xd @ w.T
    bound = 2 * K * 2.0 ** -53 * (np.abs(xd) @ np.abs(w).T)
    assert np.all(np.abs(y - ref) <= bound)


# ---------------------------------------------------------------------------
# special cases with closed forms
# ---------------------------------------------------------------------------

def test_one_hot_activation_picks_a_weight():
    g = np.random.default_rng(40)
    M, K, N, G = 3, 256, 16, 128
    q, s, z = _rand_int4(g, N, K, G)
    ks = [0, 130, 255]
    x = np.zeros((M, K), np.uint16)
    for m, k in enumerate(ks):
        x[m, k] = 0x3F80  # 1.0
    y = oracle.linear_int4(x, q, s, z, G)
    w = oracle.dequant_int4(q, s, z, K, G)
    for m, k in enumerate(ks):
        assert np.array_equal(y[m], w[:, k])


def test_identity_weights_reproduce_x():
    K = N = 256
    x = gen.x_bf16(2, K)
    xd = oracle.bf16_to_f64(x)
    # INT8: q = 64 I, s = 2^-6  -> w = I
    q8 = (np.eye(N) * 64).astype(np.int8)
    s8 = np.full(N, 0x3C80, np.uint16)  # 2^-6
    assert np.array_equal(oracle.linear_int8(x, q8, s8), xd)
    # INT4: q = 9 on the diagonal, 8 elsewhere, z = 8, s = 1 -> w = I
    G = 128
    qn = np.full((N, K), 8, np.uint32)
    np.fill_diagonal(qn, 9)
    q4 = np.zeros((N, K // 8), np.uint32)
    for k in range(K):
        q4[:, k // 8] |= qn[:, k] << np.uint32(4 * (k % 8))
    z4 = np.zeros((N, oracle.zero_words_per_row(K, G)), np.uint32)
    for gi in range(K // G):
        z4[:, gi // 8] |= np.uint32(8) << np.uint32(4 * (gi % 8))
    s4 = np.full((N, K // G), 0x3F80, np.uint16)
    assert np.array_equal(oracle.linear_int4(x, q4, s4, z4, G), xd)


def test_zero_scales_give_zero():
    g = np.random.default_rng(50)
    M, K, N, G = 2, 256, 16, 128
    x = gen.x_bf16(M, K)
    q, _, z = _rand_int4(g, N, K, G)
    s = np.zeros((N, K // G), np.uint16)
    assert np.all(oracle.linear_int4(x, q, s, z, G) == 0)
    q8 = g.integers(-127, 128, (N, K), dtype=np.int8)
    assert np.all(oracle.linear_int8(x, q8, np.zeros(N, np.uint16)) == 0)


def test_int8_and_int4_agree_when_representable():
    """A weight with values in -8..7 and one scale per row is both an INT8
    per-channel weight and an INT4 group weight (q4 = q8 + 8, z = 8).  Catches
    group-index and zero-point mistakes in either path."""
    g = np.random.default_rng(60)
    M, K, N, G = 2, 384, 16, 128
    x = gen.x_bf16(M, K)
    q8 = g.integers(-8, 8, (N, K), dtype=np.int8)
    s = gen.f32_to_bf16_bits(g.uniform(1e-3, 2e-2, N).astype(np.float32))
    q4 = np.zeros((N, K // 8), np.uint32)
    for k in range(K):
        q4[:, k // 8] |= (q8[:, k].astype(np.int32) + 8).astype(np.uint32) << np.uint32(4 * (k % 8))
    z4 = np.zeros((N, oracle.zero_words_per_row(K, G)), np.uint32)
    for gi in range(K // G):
        z4[:, gi // 8] |= np.uint32(8) << np.uint32(4 * (gi % 8))
    s4 = np.repeat(s[:, None], K // G, axis=1)
    assert np.array_equal(oracle.linear_int8(x, q8, s), oracle.linear_int4(x, q4, s4, z4, G))


def test_scaling_and_row_permutation():
    g = np.random.default_rng(70)
    M, K, N, G = 2, 256, 24, 128
    x = gen.x_bf16(M, K)
    q, s, z = _rand_int4(g, N, K, G)
    y = oracle.linear_int4(x, q, s, z, G)
    s2 = (s.astype(np.uint32) + (1 << 7)).astype(np.uint16)  # exponent + 1: exactly 2 s
    assert np.array_equal(oracle.linear_int4(x, q, s2, z, G), 2 * y)
    perm = g.permutation(N)
    assert np.array_equal(oracle.linear_int4(x, q[perm], s[perm], z[perm], G), y[:, perm])
    rows = np.array([5, 0, 23, 5])
    assert np.array_equal(oracle.linear_int4(x, q, s, z, G, rows=rows), y[:, rows])


def test_result_independent_of_threads():
    M, K, N = 2, 1024, 96
    x = gen.x_bf16(M, K)
    q, s = oracle.quant_int8(gen.W_f32(0, N, K))
    n0 = oracle.get_threads()
    oracle.set_threads(1)
    y1 = oracle.linear_int8(x, q, s)
    oracle.set_threads(max(n0, 4))
    y2 = oracle.linear_int8(x, q, s)
    oracle.set_threads(n0)
    assert np.array_equal(y1, y2)


# ---------------------------------------------------------------------------
# generator properties (no method arithmetic there, only addressing)
# ---------------------------------------------------------------------------

def test_generator_rows_are_addressable():
    K = 128
    a = gen.W_f32(250, 600, K)
    b = gen.W_rows(np.arange(250, 600), K)
    assert np.array_equal(a, b)
    x4 = gen.x_bf16(4, K)
    assert np.array_equal(gen.x_bf16(1, K), x4[:1])
    q, s = gen.direct_int8(64, 16)
    assert q.min() >= -127 and q.max() <= 127
    sd = oracle.bf16_to_f64(s)
    assert np.all((sd >= 1e-3 * (1 - 2**-8)) & (sd <= 2e-2 * (1 + 2**-8)))


# ---------------------------------------------------------------------------
# groups of 32 and 64 k and one pair per channel (G = K); fp16 activations
# (the validation matrix of the Marlin register and launch scheduling
# benchmark, "Validation and limits")
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("G", [32, 64, 512])
def test_quant_int4_error_bound_groups(G):
    K = 512  # G = K: one scale and zero point per row
    W = np.concatenate([gen.W_f32(0, 64, K), _adversarial_rows(K)])
    q, s, z = oracle.quant_int4(W, G)
    assert s.shape == (W.shape[0], K // G)
    w = oracle.dequant_int4(q, s, z, K, G)
    sd = np.repeat(oracle.bf16_to_f64(s), G, axis=1)
    err = np.abs(w - W.astype(np.float64))
    assert np.all((err <= sd / 2 * (1 + 2.0 ** -40)) | ((sd == 0) & (W == 0)))


@pytest.mark.parametrize("G", [32, 64, 256])
def test_linear_int4_exact_bruteforce_groups(G):
    g = np.random.default_rng(50 + G)
    M, K, N = 2, 256, 8
    x = gen.f32_to_bf16_bits(g.normal(0, 1, (M, K)).astype(np.float32))
    q, s, z = _rand_int4(g, N, K, G)
    y = oracle.linear_int4(x, q, s, z, G)
    exact = _exact_int4(x, q, s, z, G)
    w = oracle.dequant_int4(q, s, z, K, G)
    _check_against_exact(y, exact, x, np.abs(oracle.bf16_to_f64(x)) @ np.abs(w).T)


def test_f16_decode_every_pattern():
    """binary16 -> binary64 on all 65536 patterns against numpy's float16."""
    h = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ours = oracle.f16_to_f64(h)
    ref = h.view(np.float16).astype(np.float64)
    both_nan = np.isnan(ours) & np.isnan(ref)
    assert np.all(both_nan | (ours == ref))
    assert np.all(np.signbit(ours[~both_nan]) == np.signbit(ref[~both_nan]))


def test_f16_rounding_against_numpy():
    """binary64 -> binary16 round to nearest even against numpy's float16
    conversion: random values over the whole range, exact ties between
    neighbours (normal and subnormal), and the overflow edge."""
    g = np.random.default_rng(60)
    v = np.concatenate([
        g.normal(0, 1, 20000), g.normal(0, 3e4, 20000), g.normal(0, 1e-5, 20000), g.normal(0, 1e-7, 5000),
        np.ldexp(g.integers(0, 4096, 20000) + 0.5, -12),           # ties at quantum 2^-11 .. (normal)
        np.ldexp(g.integers(0, 1024, 4000) + 0.5, -24),            # ties between subnormals
        [65504.0, 65519.999, 65520.0, 65536.0, 1e9, 2.0 ** -24, 2.0 ** -25, 2.0 ** -25 * 1.0001, 0.0, -0.0],
    ])
    v = np.concatenate([v, -v])
    ours = oracle.f64_to_f16(v)
    ref = v.astype(np.float16).view(np.uint16)
    assert np.array_equal(ours, ref)


def test_linear_fp16_activations_match_numpy():
    """fp16 activations: the oracle's linear against numpy's float16 decode
    and fp64 matmul on the oracle's own dequantized weights, both formats."""
    g = np.random.default_rng(70)
    M, K, N = 3, 512, 32
    xh = g.normal(0, 1, (M, K)).astype(np.float16).view(np.uint16)
    xd = xh.view(np.float16).astype(np.float64)
    q8 = g.integers(-127, 128, size=(N, K), dtype=np.int8)
    s8 = gen.f32_to_bf16_bits(g.uniform(1e-3, 2e-2, N).astype(np.float32))
    w8 = oracle.dequant_int8(q8, s8)
    y8 = oracle.linear_int8(xh, q8, s8, act="fp16")
    assert np.all(np.abs(y8 - xd @ w8.T) <= 2 * K * 2.0 ** -53 * (np.abs(xd) @ np.abs(w8).T))
    q4, s4, z4 = _rand_int4(g, N, K, 64)
    w4 = oracle.dequant_int4(q4, s4, z4, K, 64)
    y4 = oracle.linear_int4(xh, q4, s4, z4, 64, act="fp16")
    assert np.all(np.abs(y4 - xd @ w4.T) <= 2 * K * 2.0 ** -53 * (np.abs(xd) @ np.abs(w4).T))
