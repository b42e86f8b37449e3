"""Shared helpers of the GPU tests: moving seeded inputs to the device,
building packed weights through the library, and the parity check.

The expected values always come from the CPU oracle (``oracle``) on inputs
from ``wq_inputs``; nothing expected is ever read back from the CUDA path.
"""
import numpy as np
import torch

import oracle
import weight_only_quantized_02_b200 as wq
import wq_inputs as gen

# The layer's parity bar: |y_gpu - y_ref| <= 1e-2 * max(|y_ref|, 1) elementwise,
# y_ref the fp64 oracle, y_gpu the bf16 output (fp32 accumulation).
REL_TOL = 1e-2


def dev():
    return torch.device("cuda:0")


def bf16_dev(x_bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(x_bits).view(np.int16)).view(torch.bfloat16).to(dev())


def to_dev(a: np.ndarray) -> torch.Tensor:
    a = np.ascontiguousarray(a)
    view = {np.dtype(np.uint16): np.int16, np.dtype(np.uint32): np.int32, np.dtype(np.uint8): np.uint8}
    if a.dtype in view:
        a = a.view(view[a.dtype])
    return torch.from_numpy(a).to(dev())


def y_host(y: torch.Tensor) -> np.ndarray:
    return y.float().cpu().numpy().astype(np.float64)


def bits_u16(t: torch.Tensor) -> np.ndarray:
    return t.cpu().numpy().view(np.uint16)


def bits_u32(t: torch.Tensor) -> np.ndarray:
    return t.cpu().numpy().view(np.uint32)


def assert_parity(y_gpu: np.ndarray, y_ref: np.ndarray, what: str = "") -> float:
    assert y_gpu.shape == y_ref.shape, (y_gpu.shape, y_ref.shape)
    err = np.abs(y_gpu - y_ref)
    bound = REL_TOL * np.maximum(np.abs(y_ref), 1.0)
    bad = err > bound
    if bad.any():
        i = np.argwhere(bad)[0]
        raise AssertionError(f"{what}: {bad.sum()} elements out of tolerance; first at {tuple(i)}: "
                             f"gpu {y_gpu[tuple(i)]} ref {y_ref[tuple(i)]}")
    return float(np.sqrt(np.mean((y_gpu - y_ref) ** 2) / max(np.mean(y_ref ** 2), 1e-300)))


def pack_canonical_int8(q: np.ndarray, s: np.ndarray) -> wq.PackedWeight:
    return wq.wq_pack_int8(to_dev(q), to_dev(s))


def pack_canonical_int4(q: np.ndarray, s: np.ndarray, z: np.ndarray) -> wq.PackedWeight:
    return wq.wq_pack_int4(to_dev(q), to_dev(s), to_dev(z))


def quantize_and_pack(W: np.ndarray, bits: int):
    """fp32 W [N][K] -> device quantizer -> packer.  Returns the packed weight
    and the device's canonical codes (host copies) for the bit-exact checks."""
    Wd = torch.from_numpy(np.ascontiguousarray(W)).to(dev())
    if bits == 8:
        q, s = wq.wq_quantize_int8(Wd)
        pw = wq.wq_pack_int8(q, s)
        canon = (q.cpu().numpy(), bits_u16(s))
    else:
        q, s, z = wq.wq_quantize_int4(Wd)
        pw = wq.wq_pack_int4(q, s, z)
        canon = (bits_u32(q), bits_u16(s), bits_u32(z))
    del Wd
    return pw, canon


def oracle_linear(x_bits: np.ndarray, canon, bits: int, rows=None) -> np.ndarray:
    if bits == 8:
        return oracle.linear_int8(x_bits, canon[0], canon[1], rows=rows)
    return oracle.linear_int4(x_bits, canon[0], canon[1], canon[2], 128, rows=rows)


def workspace(M: int, K: int, N: int, max_split: int = 32) -> torch.Tensor:
    nbytes = wq.wq_workspace_bytes(M, K, N, max_split)
    return torch.zeros(nbytes, dtype=torch.uint8, device=dev())


def i8_fixed_point(x_bits: np.ndarray, with_exponents: bool = False):
    """The activations as the integer tensor-core path represents them, from
    the library's stated contract (include/wq.h): per token row, e = 21 - E
    with E the binary exponent of the row's largest magnitude (2^E <= max|x|
    < 2^(E+1); subnormal rows use E = -126), at most 127, and
    x -> round(x * 2^e) * 2^-e, ties to even.  Every element within 2^14 of
    the row's largest is unchanged.  Returns binary64 values (and the
    exponents e per row when asked)."""
    x = oracle.bf16_to_f64(x_bits)
    out = np.zeros_like(x)
    es = np.zeros(x.shape[0], np.int64)
    for m in range(x.shape[0]):
        amax = np.max(np.abs(x[m])) if x.shape[1] else 0.0
        if amax == 0.0:
            continue
        E = max(int(np.frexp(amax)[1]) - 1, -126)  # amax = f * 2^(E+1), f in [0.5, 1)
        e = min(21 - E, 127)
        es[m] = e
        out[m] = np.rint(np.ldexp(x[m], e)) * np.ldexp(1.0, -e)  # exact: |X| < 2^22
    return (out, es) if with_exponents else out


# ---------------------------------------------------------------------------
# activation rows of wide dynamic range (the integer paths' exactness guard)
# ---------------------------------------------------------------------------
BF16_MAX = 0x7F7F      # largest finite bf16, 3.3895e38
BF16_MIN_NORMAL = 0x0080
BF16_MIN_SUB = 0x0001


def _bits_of(v: np.ndarray) -> np.ndarray:
    return gen.f32_to_bf16_bits(np.asarray(v, np.float32))


def outlier_rows(K: int, M: int = 4) -> np.ndarray:
    """M N(0,1) rows, row m with one element at +-2^(12, 14, 15, 16)[m % 4]."""
    x = oracle.bf16_to_f64(gen.x_bf16(M, K)).astype(np.float32)
    for m in range(M):
        p = (12, 14, 15, 16)[m % 4]
        x[m, (977 * m + 5) % K] = (-1.0) ** m * 2.0 ** p
    return _bits_of(x)


def extreme_rows(K: int) -> np.ndarray:
    """Row 0: N(0,1) with one element at bf16 max and a few at the smallest
    normal and subnormals.  Row 1: N(0,1) scaled by 2^-100.  Row 2: zero but
    for one element at the smallest normal.  Row 3: N(0,1) with one element at
    -bf16 max.  One huge element per row: two of opposite products would
    cancel, and the sum of what is left then depends on the order of the
    binary64 additions (the oracle's among them) by more than the tolerance."""
    base = gen.x_bf16(4, K)
    x = base.copy()
    x[0, 11] = BF16_MAX
    for j, b in enumerate((BF16_MIN_NORMAL, BF16_MIN_SUB, BF16_MIN_NORMAL | 0x8000, 0x0003)):
        x[0, 100 + 37 * j] = b
    x[1] = _bits_of(oracle.bf16_to_f64(base[1:2]).astype(np.float32) * np.float32(2.0 ** -100))[0]
    x[2] = 0
    x[2, K - 1] = BF16_MIN_NORMAL
    x[3, 7] = BF16_MAX | 0x8000
    return x


