"""The integer GEMV's work split, checked on the host through the library's
debug views (the same partition code the kernel runs, compiled for the
host; no GPU): every chunk of every 16-row block is taken by exactly one
warp, a warp's partial slots never clash, and the contributors listed for
a shared row block are exactly the warps whose chunks meet it, in warp
order.  Shapes span the five decode workloads, ragged k-blocks, fewer row
blocks than CTAs and both launch shapes."""
import random

import pytest

import weight_only_quantized_02_b200 as wq


def _check(bits, K, N, G, warps):
    meta, runs = wq.wq_gemv_i8_plan(bits, K, N, G, warps)
    CPR, LB, RB0, RL = meta["CPR"], meta["LB"], meta["RB0"], meta["RL"]
    NRB = N // 16
    assert LB == NRB // G and RB0 == G * LB and RL == (NRB - RB0) * CPR
    owner = {}
    shared_parts = {}  # rb -> [(global warp, slot)] in warp order
    own_parts = {}  # (cta, rb) -> number of partial contributors
    for c in range(G):
        for w in range(warps):
            rb0, q0, n, shared = runs[c][w]
            rb, q, start = rb0, q0, q0
            segs = 0
            for i in range(n):
                assert (rb, q) not in owner, ("chunk taken twice", rb, q)
                owner[(rb, q)] = (c, w)
                if shared:
                    assert RB0 <= rb < NRB
                else:
                    assert c * LB <= rb < (c + 1) * LB
                if q == CPR - 1 or i == n - 1:  # end of a segment
                    whole = start == 0 and q == CPR - 1
                    if not whole:
                        segs += 1
                        slot = 0 if rb == rb0 else 1
                        if shared:
                            shared_parts.setdefault(rb, []).append((c * warps + w, slot))
                        else:
                            own_parts[(c, rb)] = own_parts.get((c, rb), 0) + 1
                    rb, q, start = rb + 1, 0, 0
                else:
                    q += 1
            assert segs <= 2  # two partial slots per warp
    assert len(owner) == NRB * CPR  # every chunk once
    for rb in range(RB0, NRB):
        got = wq.wq_gemv_i8_contributors(bits, K, N, G, warps, rb, CPR)
        assert got == shared_parts.get(rb, [(owner[(rb, 0)][0] * warps + owner[(rb, 0)][1], 0)])
        assert len(set(got)) == len(got)
    seen = set()
    for parts in shared_parts.values():
        for p in parts:
            assert p not in seen  # no warp writes two row blocks into one slot
            seen.add(p)
    for n in own_parts.values():
        assert n >= 2  # a CTA's split row block has at least two contributors


def _grid(bits, K, N, warps, sms=148):
    D = 4 if bits == 8 else 6
    I = (N // 16) * -(-(-(-K // 128)) // D)
    G = min((16 // warps) * sms, 448 * 8 // warps, -(-I // (2 * warps)))
    return max(1, G)


WORKLOADS = [(8, 1024, 1024), (8, 5120, 17408), (4, 5120, 25600), (4, 17408, 5120), (8, 5120, 152064)]


@pytest.mark.parametrize("bits,K,N", WORKLOADS)
@pytest.mark.parametrize("warps", [16, 8])
def test_partition_of_the_workloads(bits, K, N, warps):
    _check(bits, K, N, _grid(bits, K, N, warps), warps)


def test_partition_edge_shapes():
    for bits, K, N in [(8, 16, 16), (4, 128, 16), (8, 1120, 400), (4, 1152, 400), (8, 65536, 48), (4, 65536, 4096)]:
        for warps in (16, 8):
            for G in (1, 2, 3, 7, _grid(bits, K, N, warps)):
                _check(bits, K, N, G, warps)


def test_partition_random_shapes():
    rng = random.Random(7)
    for _ in range(60):
        bits = rng.choice([4, 8])
        K = rng.choice([128, 256, 1024, 1152, 5120, 8192]) if bits == 4 else rng.choice([16, 496, 1120, 5120, 8192])
        N = 16 * rng.randint(1, 4000)
        warps = rng.choice([16, 8])
        G = rng.choice([_grid(bits, K, N, warps), rng.randint(1, 448), rng.randint(1, 20)])
        _check(bits, K, N, G, warps)


def test_plan_rejects_bad_arguments():
    with pytest.raises(RuntimeError):
        wq.wq_gemv_i8_plan(6, 1024, 1024, 4, 16)
    with pytest.raises(RuntimeError):
        wq.wq_gemv_i8_plan(8, 1024, 1000, 4, 16)  # N not a multiple of 16
    with pytest.raises(RuntimeError):
        wq.wq_gemv_i8_plan(8, 1024, 1024, 4, 12)  # warps
    with pytest.raises(RuntimeError):
        wq.wq_gemv_i8_contributors(8, 1024, 1024, 4, 16, 0, 8)  # not a shared row block (LB covers all)
