"""Python binding of libwq.so, the B200 weight-only quantized linear layer.

Argument marshalling only: every step of the layer runs in the library's
CUDA kernels.  torch supplies device memory and streams.  The names follow
the C ABI in ``include/wq.h`` (``wq_linear``, ``wq_pack_int4``, ...); the
binding takes torch tensors where the C functions take pointers and raises
``WQError`` where they return a negative status.

There is no fallback: if libwq.so is missing or was built for another
architecture, importing this package or calling a kernel fails loudly.
"""
from __future__ import annotations

import ctypes
import os
import re
from dataclasses import dataclass
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libwq.so")
HEADER_PATH = os.path.join(os.path.dirname(_HERE), "include", "wq.h")

WQ_VARIANT_AUTO = -1
WQ_VARIANT_GEMV = 0     # stream-K GEMV (needs the workspace), M <= 32
WQ_VARIANT_GEMM = 1     # tcgen05 split-K GEMM, M <= 128
WQ_VARIANT_GEMV_RB = 2  # row-block GEMV, no workspace, M <= 32
WQ_VARIANT_GEMM_SK = 3  # stream-K tcgen05 GEMM (needs the workspace), M <= 128
WQ_VARIANT_I8MMA = 4    # tcgen05 kind::i8 (needs the workspace): W8A16 M <= 64, W4A16 M <= 32
WQ_VARIANT_GEMV_I8 = 5  # integer GEMV, mma.sync m16n8k32 s8 on the packed codes (needs the workspace), M <= 8
WQ_VARIANT_GEMM_W4 = 6  # W4A16 stream-K tcgen05 GEMM, one role-split CTA per SM (needs the workspace), M <= 128

STATUS = {
    0: "WQ_OK", -1: "WQ_ERR_NULL", -2: "WQ_ERR_SHAPE", -3: "WQ_ERR_ALIGN", -4: "WQ_ERR_GROUP",
    -5: "WQ_ERR_HEADER", -6: "WQ_ERR_WORKSPACE", -7: "WQ_ERR_CUDA", -8: "WQ_ERR_TUNING",
    -9: "WQ_ERR_TIMEOUT", -10: "WQ_ERR_ARCH", -11: "WQ_ERR_VARIANT",
}


class WQError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {STATUS.get(status, status)} ({strerror(status)})")


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with `python -m weight_only_quantized_02_b200.build` "
            "(nvcc, sm_100a). There is no CPU fallback.")
    L = ctypes.CDLL(LIB_PATH)
    P, I, SZ = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
    sig = {
        "wq_strerror": (ctypes.c_char_p, [I]),
        "wq_version": (I, []),
        "wq_packed_bytes": (I, [I, I, I, I, P, P, P]),
        "wq_quantize_int8": (I, [P, I, I, P, P, P]),
        "wq_quantize_int4": (I, [P, I, I, I, P, P, P, P]),
        "wq_pack_int8": (I, [P, P, I, I, P, P, P]),
        "wq_pack_int4": (I, [P, P, P, I, I, I, P, P, P, P]),
        "wq_check_packed": (I, [P, I, I, I, I, P]),
        "wq_linear": (I, [P, I, I, P, P, P, I, I, P, P]),
        "wq_linear_forced": (I, [P, I, I, P, P, P, I, I, P, I, I, P]),
        "wq_linear_ex": (I, [P, I, I, P, P, P, I, I, P, I, I, P, SZ, P]),
        "wq_linear_noalloc": (I, [P, I, I, P, P, P, I, I, P, P]),
        "wq_linear_topk": (I, [P, I, I, P, P, P, I, I, I, P, P, P, SZ, P]),
        "wq_linear_f16": (I, [P, I, I, P, P, P, I, I, P, P]),
        "wq_topk_workspace_bytes": (SZ, [I, I, I]),
        "wq_workspace_bytes": (SZ, [I, I, I, I]),
        "wq_set_workspace": (I, [P, SZ]),
        "wq_tune": (I, [P, I, I, P, P, P, I, I, P, I, I, P]),
        "wq_get_choice": (I, [I, I, I, I, I, P, P]),
        "wq_set_choice": (I, [I, I, I, I, I, I, I]),
        "wq_clear_tuning": (I, []),
        "wq_save_tuning": (I, [ctypes.c_char_p]),
        "wq_load_tuning": (I, [ctypes.c_char_p]),
        "wq_unpack_debug": (I, [P, P, I, I, I, I, P, P, P]),
        "wq_dequant_debug": (I, [P, P, P, I, I, I, I, P, P]),
        "wq_device_error": (I, [P]),
        "wq_wait_selftest": (I, [I, P]),
        "wq_gemv_i8_plan": (I, [I, I, I, I, I, P, P]),
        "wq_gemv_i8_contributors": (I, [I, I, I, I, I, I, P, P, P]),
        "wq_stream_k_plan": (I, [ctypes.c_longlong, I, I, P, P, P, P]),
    }
    for name, (res, args) in sig.items():
        f = getattr(L, name)
        f.restype = res
        f.argtypes = args
    return L


lib = _load()


def header_functions() -> list:
    """Names of the functions declared in include/wq.h."""
    text = open(HEADER_PATH).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(wq_[a-z0-9_]+)\s*\(", text)))


def strerror(status: int) -> str:
    return lib.wq_strerror(int(status)).decode()


wq_strerror = strerror


def wq_version() -> int:
    return int(lib.wq_version())


def _check(rc: int, what: str) -> None:
    if rc != 0:
        raise WQError(rc, what)


def _p(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _s(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _bits(group: int) -> int:
    return 8 if group == 0 else 4


# ---------------------------------------------------------------------------
# sizes
# ---------------------------------------------------------------------------

def wq_packed_bytes(bits: int, K: int, N: int, group: int):
    a, b, c = ctypes.c_size_t(), ctypes.c_size_t(), ctypes.c_size_t()
    _check(lib.wq_packed_bytes(bits, K, N, group, ctypes.byref(a), ctypes.byref(b), ctypes.byref(c)),
           "wq_packed_bytes")
    return a.value, b.value, c.value


def wq_workspace_bytes(M: int, K: int, N: int, max_split: int) -> int:
    return int(lib.wq_workspace_bytes(M, K, N, max_split))


# ---------------------------------------------------------------------------
# quantize / pack
# ---------------------------------------------------------------------------

def wq_quantize_int8(W: torch.Tensor, stream=None):
    N, K = W.shape
    q = torch.empty((N, K), dtype=torch.int8, device=W.device)
    s = torch.empty((N,), dtype=torch.int16, device=W.device)
    _check(lib.wq_quantize_int8(_p(W), K, N, _p(q), _p(s), _s(stream)), "wq_quantize_int8")
    return q, s


def wq_quantize_int4(W: torch.Tensor, group: int = 128, stream=None):
    N, K = W.shape
    q = torch.empty((N, K // 8), dtype=torch.int32, device=W.device)
    s = torch.empty((N, K // group), dtype=torch.int16, device=W.device)
    z = torch.empty((N, (K // group + 7) // 8), dtype=torch.int32, device=W.device)
    _check(lib.wq_quantize_int4(_p(W), K, N, group, _p(q), _p(s), _p(z), _s(stream)), "wq_quantize_int4")
    return q, s, z


@dataclass
class PackedWeight:
    """The three packed buffers of one weight plus its shape."""
    wq: torch.Tensor
    scales: torch.Tensor
    zeros: Optional[torch.Tensor]
    bits: int
    K: int
    N: int
    group: int

    @property
    def nbytes_algorithmic(self) -> int:
        """Bytes the layer must read for the weight: codes + scales + zeros (no padding)."""
        if self.bits == 8:
            return self.N * self.K + self.N * 2
        g = self.K // self.group
        return self.N * self.K // 2 + self.N * g * 2 + self.N * g // 2


def wq_pack_int8(q: torch.Tensor, s: torch.Tensor, stream=None) -> PackedWeight:
    N, K = q.shape
    wb, sb, _ = wq_packed_bytes(8, K, N, 0)
    wq = torch.empty(wb, dtype=torch.uint8, device=q.device)
    sp = torch.empty(sb // 2, dtype=torch.int16, device=q.device)
    _check(lib.wq_pack_int8(_p(q), _p(s), K, N, _p(wq), _p(sp), _s(stream)), "wq_pack_int8")
    return PackedWeight(wq, sp, None, 8, K, N, 0)


def wq_pack_int4(q: torch.Tensor, s: torch.Tensor, z: torch.Tensor, group: int = 128, stream=None) -> PackedWeight:
    N = q.shape[0]
    K = q.shape[1] * 8
    wb, sb, zb = wq_packed_bytes(4, K, N, group)
    wq = torch.empty(wb, dtype=torch.uint8, device=q.device)
    sp = torch.empty(sb // 2, dtype=torch.int16, device=q.device)
    zp = torch.empty(zb, dtype=torch.uint8, device=q.device)
    _check(lib.wq_pack_int4(_p(q), _p(s), _p(z), K, N, group, _p(wq), _p(sp), _p(zp), _s(stream)),
           "wq_pack_int4")
    return PackedWeight(wq, sp, zp, 4, K, N, group)


def wq_check_packed(pw: PackedWeight, stream=None) -> int:
    return int(lib.wq_check_packed(_p(pw.wq), pw.bits, pw.K, pw.N, pw.group, _s(stream)))


# ---------------------------------------------------------------------------
# the layer
# ---------------------------------------------------------------------------

def _y_for(x: torch.Tensor, N: int, y: Optional[torch.Tensor]) -> torch.Tensor:
    if y is None:
        y = torch.empty((x.shape[0], N), dtype=torch.bfloat16, device=x.device)
    return y


def wq_linear(x: torch.Tensor, pw: PackedWeight, y: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """y = x . dequant(W)^T; x bf16 [M][K] on the device."""
    M, K = x.shape
    y = _y_for(x, pw.N, y)
    _check(lib.wq_linear(_p(x), M, K, _p(pw.wq), _p(pw.scales), _p(pw.zeros), pw.group, pw.N, _p(y),
                         _s(stream)), "wq_linear")
    return y


def wq_linear_forced(x: torch.Tensor, pw: PackedWeight, variant: int, split: int,
                     y: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    M, K = x.shape
    y = _y_for(x, pw.N, y)
    _check(lib.wq_linear_forced(_p(x), M, K, _p(pw.wq), _p(pw.scales), _p(pw.zeros), pw.group, pw.N, _p(y),
                                variant, split, _s(stream)), "wq_linear_forced")
    return y


def wq_linear_ex(x: torch.Tensor, pw: PackedWeight, variant: int, split: int, ws: Optional[torch.Tensor],
                 y: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    M, K = x.shape
    y = _y_for(x, pw.N, y)
    nbytes = 0 if ws is None else ws.numel() * ws.element_size()
    _check(lib.wq_linear_ex(_p(x), M, K, _p(pw.wq), _p(pw.scales), _p(pw.zeros), pw.group, pw.N, _p(y),
                            variant, split, _p(ws), nbytes, _s(stream)), "wq_linear_ex")
    return y


def wq_linear_noalloc(x: torch.Tensor, pw: PackedWeight, y: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """wq_linear without any device allocation by the library (M <= 8).  Its
    scratch is a fixed array inside the library; see include/wq.h."""
    M, K = x.shape
    y = _y_for(x, pw.N, y)
    _check(lib.wq_linear_noalloc(_p(x), M, K, _p(pw.wq), _p(pw.scales), _p(pw.zeros), pw.group, pw.N, _p(y),
                                 _s(stream)), "wq_linear_noalloc")
    return y


def wq_linear_f16(x: torch.Tensor, pw: PackedWeight, y: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """y = x . dequant(W)^T with fp16 activations and outputs; x fp16 [M][K]."""
    M, K = x.shape
    if y is None:
        y = torch.empty((M, pw.N), dtype=torch.float16, device=x.device)
    _check(lib.wq_linear_f16(_p(x), M, K, _p(pw.wq), _p(pw.scales), _p(pw.zeros), pw.group, pw.N, _p(y),
                             _s(stream)), "wq_linear_f16")
    return y


def wq_topk_workspace_bytes(M: int, N: int, k: int) -> int:
    return int(lib.wq_topk_workspace_bytes(M, N, k))


def wq_linear_topk(x: torch.Tensor, pw: PackedWeight, k: int, ws: torch.Tensor, stream=None):
    """The k largest logits of every token row and their indices: (vals bf16
    [M][k] descending, idx int32 [M][k]); ws a device scratch of at least
    wq_topk_workspace_bytes(M, N, k) bytes."""
    M, K = x.shape
    vals = torch.empty((M, k), dtype=torch.bfloat16, device=x.device)
    idx = torch.empty((M, k), dtype=torch.int32, device=x.device)
    _check(lib.wq_linear_topk(_p(x), M, K, _p(pw.wq), _p(pw.scales), _p(pw.zeros), pw.group, pw.N, k, _p(vals),
                              _p(idx), _p(ws), ws.numel() * ws.element_size(), _s(stream)), "wq_linear_topk")
    return vals, idx


def wq_linear_status(x, pw: PackedWeight, y, variant=WQ_VARIANT_AUTO, split=0, stream=None) -> int:
    """Raw status of wq_linear_forced, for the argument-checking tests."""
    M, K = x.shape if x is not None else (1, pw.K)
    return int(lib.wq_linear_forced(_p(x), M, K, _p(pw.wq), _p(pw.scales), _p(pw.zeros), pw.group, pw.N,
                                    _p(y), variant, split, _s(stream)))


def wq_set_workspace(ws: Optional[torch.Tensor]) -> None:
    nbytes = 0 if ws is None else ws.numel() * ws.element_size()
    _check(lib.wq_set_workspace(_p(ws), nbytes), "wq_set_workspace")


# ---------------------------------------------------------------------------
# dispatcher
# ---------------------------------------------------------------------------

def wq_tune(x: torch.Tensor, pw: PackedWeight, y: torch.Tensor, warmup: int = 3, iters: int = 9, stream=None):
    M, K = x.shape
    _check(lib.wq_tune(_p(x), M, K, _p(pw.wq), _p(pw.scales), _p(pw.zeros), pw.group, pw.N, _p(y), warmup,
                       iters, _s(stream)), "wq_tune")
    return wq_get_choice(M, K, pw.N, pw.bits, pw.group)


def wq_get_choice(M: int, K: int, N: int, bits: int, group: int):
    v, s = ctypes.c_int(), ctypes.c_int()
    _check(lib.wq_get_choice(M, K, N, bits, group, ctypes.byref(v), ctypes.byref(s)), "wq_get_choice")
    return v.value, s.value


def wq_set_choice(M, K, N, bits, group, variant, split) -> None:
    _check(lib.wq_set_choice(M, K, N, bits, group, variant, split), "wq_set_choice")


def wq_clear_tuning() -> None:
    _check(lib.wq_clear_tuning(), "wq_clear_tuning")


def wq_save_tuning(path: str) -> None:
    _check(lib.wq_save_tuning(path.encode()), "wq_save_tuning")


def wq_load_tuning(path: str) -> int:
    return int(lib.wq_load_tuning(path.encode()))


# ---------------------------------------------------------------------------
# debug views
# ---------------------------------------------------------------------------

def wq_unpack_debug(pw: PackedWeight, stream=None):
    q = torch.empty((pw.N, pw.K), dtype=torch.int8, device=pw.wq.device)
    z = None
    if pw.bits == 4:
        z = torch.empty((pw.N, pw.K // pw.group), dtype=torch.int8, device=pw.wq.device)
    _check(lib.wq_unpack_debug(_p(pw.wq), _p(pw.zeros), pw.bits, pw.K, pw.N, pw.group, _p(q), _p(z), _s(stream)),
           "wq_unpack_debug")
    return q, z


def wq_dequant_debug(pw: PackedWeight, stream=None) -> torch.Tensor:
    w = torch.empty((pw.N, pw.K), dtype=torch.float32, device=pw.wq.device)
    _check(lib.wq_dequant_debug(_p(pw.wq), _p(pw.scales), _p(pw.zeros), pw.bits, pw.K, pw.N, pw.group, _p(w),
                                _s(stream)), "wq_dequant_debug")
    return w


def wq_device_error(stream=None) -> int:
    return int(lib.wq_device_error(_s(stream)))


def wq_wait_selftest(limit_us: int = 50000, stream=None) -> None:
    """Enqueues a kernel whose bounded wait runs out after limit_us (nothing
    completes its mbarrier); it records WQ_ERR_TIMEOUT in the device error
    word, which wq_device_error then reports."""
    _check(lib.wq_wait_selftest(int(limit_us), _s(stream)), "wq_wait_selftest")


def wq_gemv_i8_plan(bits: int, K: int, N: int, G: int, warps: int = 16):
    """The integer GEMV's work split for G CTAs of `warps` warps (host only):
    (meta {CPR, LB, RB0, RL}, runs [G][warps][4] = first row block, its
    first chunk, chunks, shared-warp flag)."""
    meta = (ctypes.c_int * 4)()
    runs = (ctypes.c_int * (G * warps * 4))()
    _check(lib.wq_gemv_i8_plan(bits, K, N, G, warps, meta, runs), "wq_gemv_i8_plan")
    return dict(CPR=meta[0], LB=meta[1], RB0=meta[2], RL=meta[3]), \
        [[tuple(runs[(c * warps + w) * 4:(c * warps + w) * 4 + 4]) for w in range(warps)] for c in range(G)]


def wq_stream_k_plan(U: int, G: int, KB: int):
    """The stream-K cuts of U units over G CTAs (KB k-blocks per panel), host
    only: (start [G + 1], first panel [G + 1], owner of every unit by the
    per-CTA table, the same by the division form)."""
    start = (ctypes.c_int * (G + 1))()
    first = (ctypes.c_int * (G + 1))()
    own_t = (ctypes.c_int * max(U, 1))()
    own_d = (ctypes.c_int * max(U, 1))()
    _check(lib.wq_stream_k_plan(U, G, KB, start, first, own_t, own_d), "wq_stream_k_plan")
    return list(start), list(first), list(own_t)[:U], list(own_d)[:U]


def wq_gemv_i8_contributors(bits: int, K: int, N: int, G: int, warps: int, rb: int, cpr: int):
    """Contributors of shared row block rb, in summation order: a list of
    (global warp index, partial slot)."""
    ids = (ctypes.c_int * max(cpr, 1))()
    slots = (ctypes.c_int * max(cpr, 1))()
    n = ctypes.c_int(0)
    _check(lib.wq_gemv_i8_contributors(bits, K, N, G, warps, rb, ids, slots, ctypes.byref(n)),
           "wq_gemv_i8_contributors")
    return [(ids[i], slots[i]) for i in range(n.value)]
