"""Parity of the CUDA layer with the CPU oracle, element by element.

Shapes span several 16-row blocks, 128-row panels and 128-k blocks with a
ragged tail (N not a multiple of 128, INT8 K not a multiple of 128), every
token-tile boundary of both kernels (M = 1, 7, 8, 9, 16, 17, 32, 33, 64, 65,
100, 128), every GEMV K-slice count and every GEMM split factor.
Tolerance: |y_gpu - y_ref| <= 1e-2 * max(|y_ref|, 1).  Closed-form special
cases (one-hot activations, one-hot and identity weights, zero scales,
power-of-two scaling) are compared bit for bit.
"""
import os

import time

import numpy as np
import pytest
import torch

import oracle
import wq_inputs as gen
import weight_only_quantized_02_b200 as wq
from wqtest_helpers import (assert_parity, bf16_dev, dev, extreme_rows, i8_fixed_point, oracle_linear, outlier_rows,
                            pack_canonical_int4, pack_canonical_int8, quantize_and_pack, to_dev, workspace, y_host)

pytestmark = pytest.mark.gpu

GEMV, GEMM, GEMV_RB, GEMM_SK, I8, GI = (wq.WQ_VARIANT_GEMV, wq.WQ_VARIANT_GEMM, wq.WQ_VARIANT_GEMV_RB,
                                        wq.WQ_VARIANT_GEMM_SK, wq.WQ_VARIANT_I8MMA, wq.WQ_VARIANT_GEMV_I8)
GW4 = wq.WQ_VARIANT_GEMM_W4
INTEGER = (I8, GI)  # the integer paths: fixed-point activations
SHAPES = {8: (1120, 400), 4: (1152, 400)}  # (K, N): 3 full panels + a 16-row tail
M_ALL = [1, 7, 8, 9, 16, 17, 32, 33, 64, 65, 100, 128]


@pytest.fixture(scope="module")
def ws():
    t = workspace(128, 1152, 1024, 32)
    wq.wq_set_workspace(t)
    yield t
    wq.wq_set_workspace(None)


@pytest.fixture(scope="module", params=[8, 4], ids=["w8", "w4g128"])
def weight(request):
    bits = request.param
    K, N = SHAPES[bits]
    W = gen.W_f32(0, N, K)
    pw, canon = quantize_and_pack(W, bits)
    return bits, K, N, pw, canon


def _cases(M, K, bits):
    kb = (K + 127) // 128
    out = []
    if M <= 32:
        out += [(GEMV, c) for c in (1, 2, 3)]
        out += [(GEMV_RB, ks) for ks in (1, 2, 4, 8)]
    out += [(GEMM, s) for s in (1, 2, 4, 8, 16, 32) if s <= kb]
    out += [(GEMM_SK, c) for c in (1, 2)]
    if M <= (64 if bits == 8 else 32):  # integer tensor-core path: W8A16 M <= 64, W4A16 M <= 32
        out += [(I8, 1)]
    if M <= 8:  # integer GEMV
        out += [(GI, c) for c in (1, 2)]
    if bits == 4:  # role-split W4A16 GEMM
        out += [(GW4, 1)]
    return out


@pytest.mark.parametrize("M", M_ALL)
def test_linear_parity_all_variants(weight, ws, M):
    bits, K, N, pw, canon = weight
    x = gen.x_bf16(M, K)
    y_ref = oracle_linear(x, canon, bits)
    xd = bf16_dev(x)
    for variant, split in _cases(M, K, bits):
        y = wq.wq_linear_forced(xd, pw, variant, split)
        assert_parity(y_host(y), y_ref, f"bits={bits} M={M} variant={variant} split={split}")
    # the dispatcher's own choice
    assert_parity(y_host(wq.wq_linear(xd, pw)), y_ref, f"bits={bits} M={M} auto")


def test_deterministic_and_splits_agree(weight, ws):
    bits, K, N, pw, canon = weight
    x = bf16_dev(gen.x_bf16(24, K))
    for variant, split in _cases(24, K, bits):
        a = wq.wq_linear_forced(x, pw, variant, split)
        b = wq.wq_linear_forced(x, pw, variant, split)
        assert torch.equal(a.view(torch.int16), b.view(torch.int16)), (variant, split)


def test_repeated_dispatch_resets_tickets(weight, ws):
    """Many split-K and stream-K calls in a row reuse the workspace counters;
    each must leave them at zero for the next (different variant, split, M)."""
    bits, K, N, pw, canon = weight
    runs = [(GEMM, 16, 2), (GEMM, 16, 8), (GEMM_SK, 40, 2), (GEMV, 5, 3), (GEMM, 40, 4), (GEMM, 128, 9),
            (I8, 5, 1), (I8, 40 if bits == 8 else 30, 1), (GEMV, 3, 2), (I8, 1, 1), (GI, 1, 2), (GI, 8, 1),
            (GEMM_SK, 7, 1), (GI, 4, 1), (I8, 3, 1), (GI, 6, 2)]
    runs += [(GEMM, 16, 2)]
    # a workspace of its own inside a larger buffer: 4 KiB of canaries on each
    # side catch any partial or counter written outside the declared size (the
    # stream-K fix-ups index partials by computed contributor ids)
    need = wq.wq_workspace_bytes(128, K, N, 32)
    buf = torch.full((need + 8192,), 0xA5, dtype=torch.uint8, device=dev())
    own = buf[4096:4096 + need]
    own.zero_()
    for variant, M, split in runs:
        x = gen.x_bf16(M, K)
        y = wq.wq_linear_ex(bf16_dev(x), pw, variant, split, ws=own)
        assert_parity(y_host(y), oracle_linear(x, canon, bits), f"variant={variant} M={M} split={split}")
    torch.cuda.synchronize()
    # tickets, the integer path's grid counters and its residual sums (one 64-bit word per token row)
    counters = own[: 4 * (8 * ((N + 127) // 128) + 2 + 2 * 64)].view(torch.int32)
    assert int(counters.abs().sum()) == 0
    assert bool((buf[:4096] == 0xA5).all()) and bool((buf[4096 + need:] == 0xA5).all())


# ---------------------------------------------------------------------------
# closed-form special cases, bit for bit
# ---------------------------------------------------------------------------

def _all_cases(M, K, bits):
    return _cases(M, K, bits)


def _i8_want_one_hot(x_bits, q, s):
    """y of an INT8 weight with one nonzero per row, on the integer path's
    fixed-point activations: bf16_rne(s[n] * q[n][c] * xq[m][c]), exact in
    binary64 (8 + 8 + 22 significant bits)."""
    xq = i8_fixed_point(x_bits)
    y = xq @ (q.astype(np.float64).T * oracle.bf16_to_f64(s)[None, :])
    return oracle.bf16_to_f64(oracle.bf16_rne_of(y))


@pytest.mark.parametrize("bits", [8, 4])
def test_one_hot_activations_pick_weights_exactly(bits, ws):
    K, N = SHAPES[bits]
    M = 5
    g = gen.generator("misc", 21)
    W = gen.W_f32(0, N, K)
    pw, canon = quantize_and_pack(W, bits)
    ks = [0, 127, 128, 641, K - 1]
    x = np.zeros((M, K), np.uint16)
    for m, k in enumerate(ks):
        x[m, k] = 0x3F80  # 1.0
    want = oracle.bf16_to_f64(oracle.bf16_rne_of(oracle_linear(x, canon, bits)))
    for variant, split in _all_cases(M, K, bits):  # the integer path included: 1.0 and 0 are exact
        y = y_host(wq.wq_linear_forced(bf16_dev(x), pw, variant, split))
        assert np.array_equal(y, want), (variant, split)


def test_one_hot_int8_weights_exact(ws):
    K, N, M = 1120, 400, 9
    g = gen.generator("misc", 22)
    q = np.zeros((N, K), np.int8)
    cols = g.integers(0, K, N)
    q[np.arange(N), cols] = g.integers(-128, 128, N).astype(np.int8)
    s = gen.f32_to_bf16_bits(g.uniform(1e-3, 2e-2, N).astype(np.float32))
    pw = pack_canonical_int8(q, s)
    x = gen.x_bf16(M, K)
    want = oracle.bf16_to_f64(oracle.bf16_rne_of(oracle.linear_int8(x, q, s)))
    for variant, split in _all_cases(M, K, 8):
        y = y_host(wq.wq_linear_forced(bf16_dev(x), pw, variant, split))
        if variant in INTEGER:
            # exact on its fixed-point activations (or, where the exactness guard
            # recomputed an output, the oracle's value), and within the layer's
            # tolerance of the oracle
            assert np.all((y == _i8_want_one_hot(x, q, s)) | (y == want)), (variant, split)
            assert_parity(y, oracle.linear_int8(x, q, s), "one-hot int8 weights, integer path")
        else:
            assert np.array_equal(y, want), (variant, split)


def test_one_hot_int4_weights_exact(ws):
    """q = z except one (n, k) per row.  Power-of-two scales keep s*(q - z)
    exact in bf16, so the GEMM's bf16 weight tile is exact too."""
    K, N, M = 1152, 400, 9
    G = 128
    g = gen.generator("misc", 23)
    zn = g.integers(0, 16, size=(N, K // G))
    qn = np.repeat(zn, G, axis=1).astype(np.int64)
    cols = g.integers(0, K, N)
    qn[np.arange(N), cols] = g.integers(0, 16, N)
    q = np.zeros((N, K // 8), np.uint32)
    for k in range(K):
        q[:, k // 8] |= qn[:, k].astype(np.uint32) << np.uint32(4 * (k % 8))
    z = np.zeros((N, oracle.zero_words_per_row(K)), np.uint32)
    for gi in range(K // G):
        z[:, gi // 8] |= zn[:, gi].astype(np.uint32) << np.uint32(4 * (gi % 8))
    s = (0x3F80 + (g.integers(-9, 3, size=(N, K // G)) << 7)).astype(np.uint16)  # 2^e
    pw = pack_canonical_int4(q, s, z)
    x = gen.x_bf16(M, K)
    want = oracle.bf16_to_f64(oracle.bf16_rne_of(oracle.linear_int4(x, q, s, z)))
    # integer path: per group s * fp32((q - z) X) with X the fixed-point activations
    xq, e = i8_fixed_point(x, with_exponents=True)
    X = np.ldexp(xq, e[:, None])                                   # exact integers
    d = (qn[np.arange(N), cols] - zn[np.arange(N), cols // G]).astype(np.float64)
    prod = np.float32(X[:, cols] * d[None, :]).astype(np.float64)  # one binary32 rounding
    sc = oracle.bf16_to_f64(s[np.arange(N), cols // G])
    want_i8 = oracle.bf16_to_f64(oracle.bf16_rne_of(np.ldexp(prod * sc[None, :], -e[:, None])))
    # integer GEMV: per digit plane s * fp32((q - z) d_i), exact here, recombined in binary64; a row
    # block split between warps passes through one binary32 partial before the bf16 rounding
    exact = np.ldexp(X[:, cols] * d[None, :] * sc[None, :], -e[:, None])
    want_gi = oracle.bf16_to_f64(oracle.bf16_rne_of(exact))
    want_gi32 = oracle.bf16_to_f64(oracle.bf16_rne_of(np.float32(exact).astype(np.float64)))
    for variant, split in _all_cases(M, K, 4):
        y = y_host(wq.wq_linear_forced(bf16_dev(x), pw, variant, split))
        if variant == I8:
            assert np.all((y == want_i8) | (y == want)), (variant, split)
            assert_parity(y, oracle.linear_int4(x, q, s, z), "one-hot int4 weights, integer path")
        elif variant == GI:
            assert np.all((y == want_gi) | (y == want_gi32) | (y == want)), (variant, split)
            assert_parity(y, oracle.linear_int4(x, q, s, z), "one-hot int4 weights, integer GEMV")
        else:
            assert np.array_equal(y, want), (variant, split)


@pytest.mark.parametrize("bits", [8, 4])
def test_identity_weights_reproduce_x(bits, ws):
    K = N = 384 if bits == 8 else 512
    M = 33
    x = gen.x_bf16(M, K)
    if bits == 8:
        pw = pack_canonical_int8((np.eye(N) * 64).astype(np.int8), np.full(N, 0x3C80, np.uint16))
    else:
        qn = np.full((N, K), 8, np.uint32)
        np.fill_diagonal(qn, 9)
        q = np.zeros((N, K // 8), np.uint32)
        for k in range(K):
            q[:, k // 8] |= qn[:, k] << np.uint32(4 * (k % 8))
        z = np.zeros((N, oracle.zero_words_per_row(K)), np.uint32)
        for gi in range(K // 128):
            z[:, gi // 8] |= np.uint32(8) << np.uint32(4 * (gi % 8))
        pw = pack_canonical_int4(q, np.full((N, K // 128), 0x3F80, np.uint16), z)
    want = oracle.bf16_to_f64(x)
    want_i8 = oracle.bf16_to_f64(oracle.bf16_rne_of(i8_fixed_point(x)))
    for variant, split in _all_cases(M, K, bits):
        y = y_host(wq.wq_linear_forced(bf16_dev(x), pw, variant, split))
        if variant in INTEGER:
            # The integer paths round activations more than 2^14 below their
            # row's largest to the row's fixed-point grid, so y = x holds
            # bit for bit only for the others: here y is x on that grid (or
            # x itself where the exactness guard recomputed the output), and
            # within the layer's tolerance of the oracle's y = x.
            assert np.all((y == want_i8) | (y == want)), (variant, split)
            assert_parity(y, want, f"identity weights, integer path variant={variant} split={split}")
        else:
            assert np.array_equal(y, want), (variant, split)


@pytest.mark.parametrize("M", [4, 16, 64])
def test_wide_range_rows_all_variants(weight, ws, M):
    """Rows with outliers 2^12 .. 2^16 above N(0,1) values, rows around
    2^-100 and zero rows, through every variant and split; the integer
    variants also on rows holding bf16's largest and smallest normals (the
    fp32-accumulating kernels keep x q within the binary32 range, which such
    rows leave)."""
    bits, K, N, pw, canon = weight
    x = outlier_rows(K, M)
    x[1::4] = gen.f32_to_bf16_bits(oracle.bf16_to_f64(x[1::4]).astype(np.float32) * np.float32(2.0 ** -100))
    x[3::8] = 0
    y_ref = oracle_linear(x, canon, bits)
    xd = bf16_dev(x)
    for variant, split in _cases(M, K, bits):
        y = wq.wq_linear_forced(xd, pw, variant, split)
        assert_parity(y_host(y), y_ref, f"wide range bits={bits} M={M} variant={variant} split={split}")
    xe = np.concatenate([extreme_rows(K)] * ((M + 3) // 4))[:M]
    ye_ref = oracle_linear(xe, canon, bits)
    xed = bf16_dev(xe)
    for variant, split in _cases(M, K, bits):
        if variant in INTEGER:
            y = wq.wq_linear_forced(xed, pw, variant, split)
            assert_parity(y_host(y), ye_ref, f"extremes bits={bits} M={M} variant={variant} split={split}")


@pytest.mark.parametrize("bits", [8, 4])
def test_zero_scales_give_zero(bits, ws):
    K, N = SHAPES[bits]
    g = gen.generator("misc", 24)
    if bits == 8:
        pw = pack_canonical_int8(g.integers(-127, 128, (N, K), dtype=np.int8), np.zeros(N, np.uint16))
    else:
        q = g.integers(0, 2**32, size=(N, K // 8), dtype=np.uint64).astype(np.uint32)
        z = g.integers(0, 2**32, size=(N, oracle.zero_words_per_row(K)), dtype=np.uint64).astype(np.uint32)
        pw = pack_canonical_int4(q, np.zeros((N, K // 128), np.uint16), z)
    x = bf16_dev(gen.x_bf16(17, K))
    for variant, split in _all_cases(17, K, bits):
        y = y_host(wq.wq_linear_forced(x, pw, variant, split))
        assert np.all(y == 0), (variant, split)


def test_power_of_two_scaling_is_exact(weight, ws):
    bits, K, N, pw, canon = weight
    x = gen.x_bf16(9, K)
    xd = bf16_dev(x)
    x2 = bf16_dev((x.astype(np.uint32) + (1 << 7)).astype(np.uint16))  # 2x exactly (no zeros in x)
    assert np.all((x & 0x7F80) != 0)
    for variant, split in _cases(9, K, bits):
        a = y_host(wq.wq_linear_forced(xd, pw, variant, split))
        b = y_host(wq.wq_linear_forced(x2, pw, variant, split))
        assert np.array_equal(2 * a, b), (variant, split)


# ---------------------------------------------------------------------------
# boundary behaviour: canaries, argument errors, graphs, tuner
# ---------------------------------------------------------------------------

def test_output_canaries_untouched(weight, ws):
    bits, K, N, pw, canon = weight
    for M in (1, 17, 100):
        x = gen.x_bf16(M, K)
        pad = 4096
        buf = torch.full((M * N + 2 * pad,), -1234, dtype=torch.int16, device=dev())
        y = buf[pad:pad + M * N].view(torch.bfloat16).view(M, N)
        for variant, split in _cases(M, K, bits):
            wq.wq_linear_forced(bf16_dev(x), pw, variant, split, y=y)
            torch.cuda.synchronize()
            assert int((buf[:pad] != -1234).sum()) == 0 and int((buf[-pad:] != -1234).sum()) == 0, (variant, split)
            assert_parity(y_host(y), oracle_linear(x, canon, bits), f"canary M={M} {variant}/{split}")


def test_argument_errors(weight, ws):
    bits, K, N, pw, canon = weight
    x = bf16_dev(gen.x_bf16(4, K))
    y = torch.empty((4, N), dtype=torch.bfloat16, device=dev())
    assert wq.wq_linear_status(x, pw, y, GEMV_RB, 3) == -11       # split not 1/2/4/8
    assert wq.wq_linear_status(x, pw, y, GEMV, 5) == -11          # CTAs per SM 1..4
    assert wq.wq_linear_status(x, pw, y, GEMM, 33) == -11         # split above 32
    assert wq.wq_linear_status(x, pw, y, 7, 1) == -11             # unknown variant
    assert wq.wq_linear_status(x, pw, y, I8, 2) == -11            # one CTA per SM only
    assert wq.wq_linear_status(x, pw, y, GI, 3) == -11            # integer GEMV: split 1 or 2
    assert wq.wq_linear_status(x, pw, y, GI, 0) == 0              # 0: the default
    assert wq.wq_linear_status(x, pw, y, GW4, 2) == -11           # role-split W4A16 GEMM: split 1 only
    assert wq.wq_linear_status(x, pw, y, GW4, 1) == (-11 if bits == 8 else 0)  # W4A16 only
    xc = bf16_dev(gen.x_bf16(65, K))
    yc = torch.empty((65, N), dtype=torch.bfloat16, device=dev())
    assert wq.wq_linear_status(xc, pw, yc, I8, 1) == -11          # integer path takes M <= 64 (W4A16: 32)
    xd33 = bf16_dev(gen.x_bf16(33, K))
    yd33 = torch.empty((33, N), dtype=torch.bfloat16, device=dev())
    assert wq.wq_linear_status(xd33, pw, yd33, I8, 1) == (0 if bits == 8 else -11)
    x9 = bf16_dev(gen.x_bf16(9, K))
    y9 = torch.empty((9, N), dtype=torch.bfloat16, device=dev())
    assert wq.wq_linear_status(x9, pw, y9, GI, 1) == -11          # integer GEMV takes M <= 8
    xb = bf16_dev(gen.x_bf16(40, K))
    yb = torch.empty((40, N), dtype=torch.bfloat16, device=dev())
    assert wq.wq_linear_status(xb, pw, yb, GEMV, 1) == -11        # GEMV takes M <= 32
    assert wq.wq_linear_status(xb, pw, yb, GEMV_RB, 1) == -11
    # misaligned output pointer
    raw = torch.empty(4 * N + 8, dtype=torch.bfloat16, device=dev())
    assert wq.wq_linear_status(x, pw, raw[1:1 + 4 * N].view(4, N), GEMV_RB, 1) == -3
    # split > 1 without a workspace
    wq.wq_set_workspace(None)
    try:
        assert wq.wq_linear_status(x, pw, y, GEMM, 4) == -6
        assert wq.wq_linear_status(x, pw, y, GEMV, 1) == -6
        assert wq.wq_linear_status(x, pw, y, I8, 1) == -6
        assert wq.wq_linear_status(x, pw, y, GI, 2) == -6
        assert wq.wq_linear_status(x, pw, y, GEMM, 1) == 0
        assert wq.wq_linear_status(x, pw, y, GEMV_RB, 2) == 0
        assert wq.wq_linear_status(x, pw, y) == 0  # dispatcher falls back to the row-block GEMV
        xm = bf16_dev(gen.x_bf16(40, K))
        ym = torch.empty((40, N), dtype=torch.bfloat16, device=dev())
        assert wq.wq_linear_status(xm, pw, ym) == 0  # ... and to the unsplit GEMM
    finally:
        wq.wq_set_workspace(ws)
    small = torch.zeros(512, dtype=torch.uint8, device=dev())
    with pytest.raises(wq.WQError):
        wq.wq_linear_ex(x, pw, GEMM, 4, small)
    torch.cuda.synchronize()
    assert wq.wq_device_error() == 0


def test_explicit_workspace_on_two_streams(weight):
    bits, K, N, pw, canon = weight
    x = gen.x_bf16(48, K)
    xd = bf16_dev(x)
    s1, s2 = torch.cuda.Stream(), torch.cuda.Stream()
    w1, w2 = workspace(48, K, N, 8), workspace(48, K, N, 8)
    torch.cuda.synchronize()
    with torch.cuda.stream(s1):
        y1 = wq.wq_linear_ex(xd, pw, GEMM, 8, w1, stream=s1)
    with torch.cuda.stream(s2):
        y2 = wq.wq_linear_ex(xd, pw, GEMM, 4, w2, stream=s2)
    torch.cuda.synchronize()
    ref = oracle_linear(x, canon, bits)
    assert_parity(y_host(y1), ref, "stream 1")
    assert_parity(y_host(y2), ref, "stream 2")


def test_cuda_graph_replay(weight, ws):
    bits, K, N, pw, canon = weight
    runs = [(1, GEMV, 2), (1, GEMV_RB, 4), (16, GEMM, 4), (128, GEMM, 2), (1, I8, 1), (16, I8, 1), (1, GI, 2),
            (7, GI, 1)]
    for M, variant, split in runs:
        x = gen.x_bf16(M, K)
        xd = bf16_dev(x)
        y = torch.empty((M, N), dtype=torch.bfloat16, device=dev())
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            wq.wq_linear_forced(xd, pw, variant, split, y=y, stream=s)  # warm (attributes, tensor map fn)
        torch.cuda.current_stream().wait_stream(s)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            wq.wq_linear_forced(xd, pw, variant, split, y=y)
        y.zero_()
        for _ in range(3):
            g.replay()
        torch.cuda.synchronize()
        assert_parity(y_host(y), oracle_linear(x, canon, bits), f"graph M={M}")


def test_tuner_and_table_roundtrip(weight, ws, tmp_path):
    bits, K, N, pw, canon = weight
    wq.wq_clear_tuning()
    M = 16
    x = gen.x_bf16(M, K)
    y = torch.empty((M, N), dtype=torch.bfloat16, device=dev())
    v, s = wq.wq_tune(bf16_dev(x), pw, y, warmup=1, iters=3)
    assert (v, s) in _cases(M, K, bits)
    assert_parity(y_host(wq.wq_linear(bf16_dev(x), pw)), oracle_linear(x, canon, bits), "tuned")
    path = str(tmp_path / "table.txt")
    wq.wq_save_tuning(path)
    wq.wq_clear_tuning()
    assert wq.wq_load_tuning(path) == 0
    assert wq.wq_get_choice(M, K, N, bits, 0 if bits == 8 else 128) == (v, s)
    wq.wq_set_choice(M, K, N, bits, 0 if bits == 8 else 128, GEMV_RB, 8)
    assert wq.wq_get_choice(M, K, N, bits, 0 if bits == 8 else 128) == (GEMV_RB, 8)
    wq.wq_clear_tuning()


@pytest.mark.gpu
def test_bounded_wait_runs_out_and_reports():
    """Failure detection: a bounded wait on an mbarrier that nothing completes
    gives up, the kernel records a timeout and returns; the host reads it as
    WQ_ERR_TIMEOUT, the error word is cleared, and the context stays usable."""
    assert wq.wq_device_error() == 0
    t0 = time.perf_counter()
    wq.wq_wait_selftest(50000)  # 50 ms
    assert wq.wq_device_error() == -9  # WQ_ERR_TIMEOUT
    assert time.perf_counter() - t0 < 5.0
    assert wq.wq_device_error() == 0  # read and cleared
    # the context still runs work
    z = torch.ones(1024, device=dev())
    assert float(z.sum()) == 1024.0
    assert wq.lib.wq_wait_selftest(0, None) == -2  # limit out of range
