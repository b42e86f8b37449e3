"""CPU oracle for the weight-only quantized linear layer (test infrastructure).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product package never imports it,
and it never imports the product package.

Every function is a thin numpy/ctypes wrapper around ``wq_oracle.c``, which
holds all of the arithmetic (plain loops in IEEE binary64).  What each
function computes, and the page passage it restates, is documented in that
file.  Parity pins live in ``tests/test_oracle_pins.py``.
"""
import ctypes
import os

import numpy as np

from . import build as _build

_lib = None


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        P = ctypes.c_void_p
        I64 = ctypes.c_int64
        L.wqo_bf16_to_f64.restype = ctypes.c_double
        L.wqo_bf16_to_f64.argtypes = [ctypes.c_uint16]
        L.wqo_f64_to_bf16_rne.restype = ctypes.c_uint16
        L.wqo_f64_to_bf16_rne.argtypes = [ctypes.c_double]
        L.wqo_f64_to_bf16_up.restype = ctypes.c_uint16
        L.wqo_f64_to_bf16_up.argtypes = [ctypes.c_double]
        L.wqo_bf16_round_array.argtypes = [P, I64, ctypes.c_int, P]
        L.wqo_bf16_to_f64_array.argtypes = [P, I64, P]
        L.wqo_set_threads.argtypes = [ctypes.c_int]
        L.wqo_get_threads.restype = ctypes.c_int
        L.wqo_unpack_int4.argtypes = [P, I64, P]
        L.wqo_unpack_int8.argtypes = [P, I64, P]
        L.wqo_dequant_int8.argtypes = [P, P, I64, I64, P, I64, P]
        L.wqo_dequant_int4.argtypes = [P, P, P, I64, I64, I64, P, I64, P]
        L.wqo_linear_int8.argtypes = [P, I64, I64, P, P, I64, P, I64, P]
        L.wqo_linear_int4.argtypes = [P, I64, I64, P, P, P, I64, I64, P, I64, P]
        L.wqo_linear_int8_fmt.argtypes = [P, ctypes.c_int, I64, I64, P, P, I64, P, I64, P]
        L.wqo_linear_int4_fmt.argtypes = [P, ctypes.c_int, I64, I64, P, P, P, I64, I64, P, I64, P]
        L.wqo_f16_to_f64.restype = ctypes.c_double
        L.wqo_f16_to_f64.argtypes = [ctypes.c_uint16]
        L.wqo_f64_to_f16_rne.restype = ctypes.c_uint16
        L.wqo_f64_to_f16_rne.argtypes = [ctypes.c_double]
        L.wqo_f16_to_f64_array.argtypes = [P, I64, P]
        L.wqo_f16_round_array.argtypes = [P, I64, P]
        L.wqo_quant_int8.argtypes = [P, I64, I64, P, P]
        L.wqo_quant_int4.argtypes = [P, I64, I64, I64, P, P, P]
        _lib = L
    return _lib


def _c(a, dtype):
    a = np.ascontiguousarray(a, dtype=dtype)
    return a, a.ctypes.data_as(ctypes.c_void_p)


def _rows_arg(rows, N):
    if rows is None:
        return None, None, N
    r, p = _c(np.asarray(rows), np.int64)
    return r, p, len(r)


def set_threads(n: int) -> None:
    lib().wqo_set_threads(int(n))


def get_threads() -> int:
    return int(lib().wqo_get_threads())


# ---- bf16 -----------------------------------------------------------------

def bf16_to_f64(b):
    b, pb = _c(b, np.uint16)
    out = np.empty(b.shape, np.float64)
    lib().wqo_bf16_to_f64_array(pb, b.size, out.ctypes.data_as(ctypes.c_void_p))
    return out


def f64_to_bf16(v, mode: str = "rne"):
    """Round binary64 values to bf16 bit patterns (uint16); mode 'rne' or 'up'."""
    v, pv = _c(v, np.float64)
    out = np.empty(v.shape, np.uint16)
    lib().wqo_bf16_round_array(pv, v.size, 0 if mode == "rne" else 1,
                               out.ctypes.data_as(ctypes.c_void_p))
    return out


# ---- unpack / dequant -----------------------------------------------------

def unpack_int4(words):
    words, pw = _c(words, np.uint32)
    out = np.empty(words.shape[:-1] + (words.shape[-1] * 8,), np.uint8)
    lib().wqo_unpack_int4(pw, words.size, out.ctypes.data_as(ctypes.c_void_p))
    return out


def unpack_int8(q):
    q8 = np.ascontiguousarray(q).view(np.uint8)
    out = np.empty(q8.shape, np.int32)
    lib().wqo_unpack_int8(q8.ctypes.data_as(ctypes.c_void_p), q8.size,
                          out.ctypes.data_as(ctypes.c_void_p))
    return out


def dequant_int8(q, s, rows=None):
    q, pq = _c(q, np.int8)
    s, ps = _c(s, np.uint16)
    N, K = q.shape
    r, pr, nr = _rows_arg(rows, N)
    out = np.empty((nr, K), np.float64)
    lib().wqo_dequant_int8(pq, ps, K, N, pr, nr, out.ctypes.data_as(ctypes.c_void_p))
    return out


def dequant_int4(q_words, s, z_words, K, G=128, rows=None):
    q_words, pq = _c(q_words, np.uint32)
    s, ps = _c(s, np.uint16)
    z_words, pz = _c(z_words, np.uint32)
    N = q_words.shape[0]
    r, pr, nr = _rows_arg(rows, N)
    out = np.empty((nr, K), np.float64)
    lib().wqo_dequant_int4(pq, ps, pz, K, N, G, pr, nr, out.ctypes.data_as(ctypes.c_void_p))
    return out


# ---- linear ---------------------------------------------------------------

def f16_to_f64(h):
    """IEEE binary16 bit patterns -> binary64 (exact)."""
    h, ph = _c(h, np.uint16)
    out = np.empty(h.shape, np.float64)
    lib().wqo_f16_to_f64_array(ph, h.size, out.ctypes.data_as(ctypes.c_void_p))
    return out


def f64_to_f16(v):
    """binary64 -> IEEE binary16 bit patterns, round to nearest even."""
    v, pv = _c(v, np.float64)
    out = np.empty(v.shape, np.uint16)
    lib().wqo_f16_round_array(pv, v.size, out.ctypes.data_as(ctypes.c_void_p))
    return out


_FMT = {"bf16": 0, "fp16": 1}


def linear_int8(x_bf16, q, s, rows=None, act="bf16"):
    """y[m][i] = sum_k x[m][k] * s[n] * q[n][k], n = rows[i]; binary64 [M][len(rows)].
    x: bf16 bit patterns, or fp16 ones with act='fp16'."""
    x, px = _c(x_bf16, np.uint16)
    q, pq = _c(q, np.int8)
    s, ps = _c(s, np.uint16)
    M, K = x.shape
    N = q.shape[0]
    assert q.shape[1] == K
    r, pr, nr = _rows_arg(rows, N)
    y = np.empty((M, nr), np.float64)
    lib().wqo_linear_int8_fmt(px, _FMT[act], M, K, pq, ps, N, pr, nr, y.ctypes.data_as(ctypes.c_void_p))
    return y


def linear_int4(x_bf16, q_words, s, z_words, G=128, rows=None, act="bf16"):
    x, px = _c(x_bf16, np.uint16)
    q_words, pq = _c(q_words, np.uint32)
    s, ps = _c(s, np.uint16)
    z_words, pz = _c(z_words, np.uint32)
    M, K = x.shape
    N = q_words.shape[0]
    assert q_words.shape[1] * 8 == K
    r, pr, nr = _rows_arg(rows, N)
    y = np.empty((M, nr), np.float64)
    lib().wqo_linear_int4_fmt(px, _FMT[act], M, K, pq, ps, pz, G, N, pr, nr, y.ctypes.data_as(ctypes.c_void_p))
    return y


# ---- quantizers -----------------------------------------------------------

def quant_int8(W):
    W, pw = _c(W, np.float32)
    N, K = W.shape
    q = np.empty((N, K), np.int8)
    s = np.empty((N,), np.uint16)
    lib().wqo_quant_int8(pw, K, N, q.ctypes.data_as(ctypes.c_void_p),
                         s.ctypes.data_as(ctypes.c_void_p))
    return q, s


def zero_words_per_row(K, G=128):
    return (K // G + 7) // 8


def quant_int4(W, G=128):
    W, pw = _c(W, np.float32)
    N, K = W.shape
    assert K % G == 0 and K % 8 == 0
    q = np.zeros((N, K // 8), np.uint32)
    s = np.empty((N, K // G), np.uint16)
    z = np.zeros((N, zero_words_per_row(K, G)), np.uint32)
    lib().wqo_quant_int4(pw, K, N, G, q.ctypes.data_as(ctypes.c_void_p),
                         s.ctypes.data_as(ctypes.c_void_p), z.ctypes.data_as(ctypes.c_void_p))
    return q, s, z


def bf16_rne_of(y):
    """Output rounding of the layer: binary64 -> bf16 (round to nearest even)."""
    return f64_to_bf16(y, "rne")
