"""Seeded synthetic inputs for the weight-only quantized linear layer.

This module holds random draws and workload shapes only -- no unpacking,
dequantization, matmul, quantization or output rounding.  It is the one
module that both the CPU oracle side and the CUDA side take inputs from.

Every draw comes from its own counter-addressed numpy PCG64 stream
(``SeedSequence(entropy=seed, spawn_key=(stream, chunk))``), so any block of
rows can be regenerated on its own: the oracle can rebuild just the rows it
samples from a full-size workload, with the same values the device got.

Value distributions (the workloads of the decode-time linear layers these
kernels serve):
  * activations x: bf16 of an fp32 N(0, 1) draw (round to nearest even, done
    by torch's fp32 -> bf16 conversion);
  * source weights W: fp32 N(0, 0.02^2), quantized afterwards;
  * the direct W8A16 correctness case: int8 codes uniform on [-127, 127] and
    a bf16 per-channel scale uniform on [1e-3, 2e-2].
"""
from __future__ import annotations

import concurrent.futures as _cf
import os

import numpy as np

SEED = 0
ROW_CHUNK = 256  # rows of W per independent stream chunk
W_STD = 0.02

_STREAMS = {"x": 1, "W": 2, "q8": 3, "s8": 4, "misc": 5}

# Workloads: (name, bits, K, N, group, M values).  group 0 = per-channel.
WORKLOADS = {
    "w8_gemv_1024": dict(bits=8, K=1024, N=1024, group=0, Ms=(1,), direct=True),
    "w8_decode_5120x17408": dict(bits=8, K=5120, N=17408, group=0, Ms=(1, 2, 4)),
    "w4g128_decode_5120x25600": dict(bits=4, K=5120, N=25600, group=128, Ms=(1, 4, 8)),
    "w4g128_splitk_17408x5120": dict(bits=4, K=17408, N=5120, group=128, Ms=(16, 32, 64, 128),
                                     splits=(1, 2, 4, 8, 16, 32)),
    "w8_vocab_5120x152064": dict(bits=8, K=5120, N=152064, group=0, Ms=(1, 4, 16)),
}


# Beyond the five decode workloads: the same W4A16 layer at prefill-sized M
# (the larger-M regime; wq_linear runs M > 128 in chunks of 128 tokens).
EXTRA_WORKLOADS = {
    "w4g128_prefill_17408x5120": dict(bits=4, K=17408, N=5120, group=128, Ms=(256, 2048)),
}


def workload(name: str) -> dict:
    """The workload of that name, from WORKLOADS or EXTRA_WORKLOADS."""
    return WORKLOADS[name] if name in WORKLOADS else EXTRA_WORKLOADS[name]


def generator(stream: str, chunk: int = 0, seed: int = SEED) -> np.random.Generator:
    ss = np.random.SeedSequence(entropy=seed, spawn_key=(_STREAMS[stream], int(chunk)))
    return np.random.Generator(np.random.PCG64(ss))


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 bit patterns, round to nearest even (torch's conversion)."""
    import torch

    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32))
    return t.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16).copy()


def x_bf16(M: int, K: int, seed: int = SEED) -> np.ndarray:
    """Activations [M][K] as bf16 bit patterns; row m has its own stream, so
    the first rows of a larger M are the rows of a smaller M."""
    rows = [generator("x", m, seed).standard_normal(K, dtype=np.float32) for m in range(M)]
    a = np.stack(rows) if M else np.zeros((0, K), np.float32)
    return f32_to_bf16_bits(a)


def _w_chunk(c: int, K: int, seed: int) -> np.ndarray:
    a = generator("W", c, seed).standard_normal((ROW_CHUNK, K), dtype=np.float32)
    a *= np.float32(W_STD)
    return a


def W_f32(n0: int, n1: int, K: int, seed: int = SEED, threads: int | None = None) -> np.ndarray:
    """Source weights W[n0:n1][K], fp32 N(0, 0.02^2), addressed by row."""
    if n1 <= n0:
        return np.zeros((0, K), np.float32)
    c0, c1 = n0 // ROW_CHUNK, (n1 - 1) // ROW_CHUNK + 1
    chunks = list(range(c0, c1))
    out = np.empty(((c1 - c0) * ROW_CHUNK, K), np.float32)
    threads = threads or min(16, os.cpu_count() or 1)

    def fill(i_c):
        i, c = i_c
        out[i * ROW_CHUNK:(i + 1) * ROW_CHUNK] = _w_chunk(c, K, seed)

    if len(chunks) > 4 and threads > 1:
        with _cf.ThreadPoolExecutor(threads) as ex:
            list(ex.map(fill, enumerate(chunks)))
    else:
        for ic in enumerate(chunks):
            fill(ic)
    off = n0 - c0 * ROW_CHUNK
    return out[off:off + (n1 - n0)]


def W_rows(rows, K: int, seed: int = SEED) -> np.ndarray:
    """Source weight rows W[rows][K] for an arbitrary list of row indices."""
    rows = np.asarray(rows, np.int64)
    out = np.empty((len(rows), K), np.float32)
    cache = {}
    for i, n in enumerate(rows):
        c = int(n) // ROW_CHUNK
        if c not in cache:
            cache[c] = _w_chunk(c, K, seed)
        out[i] = cache[c][int(n) % ROW_CHUNK]
    return out


def direct_int8(K: int, N: int, seed: int = SEED):
    """The direct W8A16 case: q int8 [N][K] uniform on [-127, 127] and bf16
    scales [N] uniform on [1e-3, 2e-2]; no zero point."""
    q = generator("q8", 0, seed).integers(-127, 128, size=(N, K), dtype=np.int8)
    s32 = generator("s8", 0, seed).uniform(1e-3, 2e-2, size=N).astype(np.float32)
    return q, f32_to_bf16_bits(s32)


def sample_rows(N: int, count: int, seed: int = SEED) -> np.ndarray:
    """A sorted sample of output channels that always includes the first and
    last channel and the edges of a 128-row panel."""
    g = generator("misc", N, seed)
    base = {0, N - 1, min(127, N - 1), min(128, N - 1), max(N - 128, 0)}
    extra = g.choice(N, size=min(count, N), replace=False)
    return np.array(sorted(base | set(int(v) for v in extra)), np.int64)
