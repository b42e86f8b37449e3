"""The stream-K cuts shared by the persistent kernels (stream-K GEMV and GEMM,
the role-split W4A16 GEMM, the integer tensor-core GEMMs), checked on the
host through the library's debug view: the kernels' own partition code
compiled for the host, no GPU.

U units (128-row panel x 128-k block, panel-major) are cut into G contiguous
ranges.  Every unit belongs to exactly one CTA, by the per-CTA table's
binary search (the fix-ups' lookup) and by the division form alike; the
contributors of a panel, the CTAs from the owner of its first unit to the
owner of its last, are exactly the CTAs whose ranges meet it; a panel with
one contributor lies whole inside that CTA's range (it writes y and takes
no ticket); and no CTA puts two split panels into one of its two partial
slots.  Shapes: the five workloads' unit counts at the grids their kernels
launch (one or two CTAs per SM, at most the unit count), and edge cases."""
import ctypes

import pytest

import weight_only_quantized_02_b200 as wq

ERR_NULL, ERR_SHAPE = -1, -2  # include/wq.h, wq_status


def _check(U, G, KB):
    start, first, own_t, own_d = wq.wq_stream_k_plan(U, G, KB)
    sizes = [start[c + 1] - start[c] for c in range(G)]
    assert start[0] == 0 and start[G] == U
    assert min(sizes) >= 1 and max(sizes) - min(sizes) <= 1  # equal shares, none empty
    assert first == [s // KB for s in start]
    brute = [c for c in range(G) for _ in range(sizes[c])]
    assert own_t == brute
    assert own_d == brute
    slots = {}
    for p in range(U // KB):
        lo, hi = p * KB, (p + 1) * KB
        cf, cl = own_t[lo], own_t[hi - 1]
        meets = [c for c in range(G) if start[c] < hi and start[c + 1] > lo]
        assert meets == list(range(cf, cl + 1)), p
        if cf == cl:
            assert start[cf] <= lo and start[cf + 1] >= hi
            continue
        for c in meets:
            slot = 0 if p == first[c] else 1
            assert (c, slot) not in slots, (c, slot, p, slots.get((c, slot)))
            slots[(c, slot)] = p


def _grid(U, ctas):
    return min(ctas, U)


@pytest.mark.parametrize("name,N,K", [
    ("w8_gemv_1024", 1024, 1024),
    ("w8_decode_5120x17408", 17408, 5120),
    ("w4g128_decode_5120x25600", 25600, 5120),
    ("w4g128_splitk_17408x5120", 5120, 17408),
    ("w8_vocab_5120x152064", 152064, 5120),
])
@pytest.mark.parametrize("ctas", [148, 296, 444, 512])
def test_workload_cuts(name, N, K, ctas):
    panels, KB = -(-N // 128), -(-K // 128)
    U = panels * KB
    _check(U, _grid(U, ctas), KB)


@pytest.mark.parametrize("U,G,KB", [
    (1, 1, 1),        # one unit
    (7, 7, 7),        # one panel, a CTA per unit
    (40, 40, 40),     # one panel of 40 k-blocks over 40 CTAs
    (64, 64, 8),      # G capped at U
    (136 * 3, 148, 136),  # fewer units per CTA than k-blocks per panel: ranges inside one panel
    (5440, 147, 136),
    (5440, 149, 40),
    (9973, 1, 9973),  # one CTA takes everything
    (8 * 13, 13, 13),
    (1000 * 3, 997, 3),  # prime grid, short panels
])
def test_edge_cuts(U, G, KB):
    _check(U, G, KB)


def test_plan_rejects_out_of_range_without_touching_buffers():
    buf = (ctypes.c_int * 4)()
    for U, G, KB in ((4, 5, 1), (4, 0, 1), (0, 1, 1), (4, 1, 0), (2 ** 31, 1, 1)):
        assert wq.lib.wq_stream_k_plan(U, G, KB, buf, buf, buf, buf) == ERR_SHAPE
    assert wq.lib.wq_stream_k_plan(4, 1, 1, None, buf, buf, buf) == ERR_NULL
