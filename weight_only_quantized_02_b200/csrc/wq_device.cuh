// wq_device.cuh -- sm_100a device helpers for the weight-only quantized
// linear layer: inline-PTX wrappers (mbarrier, bulk/tensor copies, tcgen05,
// mma.sync) plus the packed-layout addressing shared by every kernel.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "wq_layout.h"

namespace wq {

enum : int { kErrNone = 0, kErrTimeout = 1 };

// ---------------------------------------------------------------------------
// Shared-memory addresses, mbarriers
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void *p)
{
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void fence_mbar_init()
{
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
                 "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

__device__ __forceinline__ uint64_t globaltimer_ns()
{
    uint64_t t;
    asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
    return t;
}

// Waits for the phase with the given parity to complete.  Gives up after
// kWaitLimitNs of wall time and returns false; the caller records the
// failure in its device error word and winds down without further waits.
constexpr uint64_t kWaitLimitNs = 2000000000ull; // 2 s

// One try_wait that may suspend the thread in hardware until the phase
// completes or about `ns` nanoseconds pass, so a waiting thread takes no
// issue slots from the warps doing the work.
__device__ __forceinline__ bool mbar_try_wait_suspend(uint64_t *bar, uint32_t parity, uint32_t ns)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity), "r"(ns)
        : "memory");
    return ok != 0;
}

__device__ __forceinline__ bool mbar_wait_for(uint64_t *bar, uint32_t parity, uint64_t limit_ns)
{
    if (mbar_try_wait(bar, parity))
        return true;
    const uint64_t t0 = globaltimer_ns();
    for (;;) {
        if (mbar_try_wait_suspend(bar, parity, 1000000u)) // suspended for up to 1 ms per try
            return true;
        if (globaltimer_ns() - t0 > limit_ns)
            return false;
    }
}

__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity)
{
    return mbar_wait_for(bar, parity, kWaitLimitNs);
}

// Warp-uniform form for warps that go on to execute .sync.aligned
// instructions: every lane polls, the warp agrees on the outcome.
__device__ __forceinline__ bool mbar_wait_warp(uint64_t *bar, uint32_t parity)
{
    return __all_sync(0xffffffffu, mbar_wait(bar, parity)) != 0;
}

// ---------------------------------------------------------------------------
// Bulk (TMA engine) copies, global -> shared, completing on an mbarrier.
// No multicast anywhere in this library.
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint64_t policy_evict_first()
{
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
    return p;
}

__device__ __forceinline__ uint64_t policy_evict_last()
{
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
    return p;
}

// 1-D bulk copy; dst, src 16-byte aligned, bytes a multiple of 16.
__device__ __forceinline__ void bulk_g2s(void *dst, const void *src, uint32_t bytes, uint64_t *bar,
                                         uint64_t policy)
{
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
                 " [%0], [%1], %2, [%3], %4;" ::"r"(smem_u32(dst)),
                 "l"(src), "r"(bytes), "r"(smem_u32(bar)), "l"(policy)
                 : "memory");
}

// 2-D tiled tensor load: coordinates (c0 = innermost, c1).
__device__ __forceinline__ void tma_load_2d(void *dst, const CUtensorMap *map, int c0, int c1,
                                            uint64_t *bar, uint64_t policy)
{
    asm volatile("cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
                 ".L2::cache_hint [%0], [%1, {%2, %3}], [%4], %5;" ::"r"(smem_u32(dst)),
                 "l"(map), "r"(c0), "r"(c1), "r"(smem_u32(bar)), "l"(policy)
                 : "memory");
}

__device__ __forceinline__ void prefetch_tensormap(const CUtensorMap *map)
{
    asm volatile("prefetch.tensormap [%0];" ::"l"(map) : "memory");
}

// ---------------------------------------------------------------------------
// Programmatic dependent launch (the kernel is launched with the
// programmatic-stream-serialization attribute).  wait: block until the
// preceding kernel in the stream has completed and its writes are visible;
// a no-op without such a predecessor.  launch_dependents: allow the next
// kernel to begin launching once every CTA of this grid has signalled.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// ---------------------------------------------------------------------------
// Global loads
// ---------------------------------------------------------------------------
// Streaming 128-bit load: read once, keep out of L1.
__device__ __forceinline__ uint4 ldg_stream(const void *p)
{
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.L2::256B.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

// Read-only 64-bit load that may stay in L1 (activations, reused by every warp).
__device__ __forceinline__ uint2 ldg_keep(const void *p)
{
    uint2 v;
    asm volatile("ld.global.nc.v2.u32 {%0,%1}, [%2];" : "=r"(v.x), "=r"(v.y) : "l"(p));
    return v;
}

__device__ __forceinline__ uint4 ldg_keep4(const void *p)
{
    uint4 v;
    asm volatile("ld.global.nc.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
    return v;
}

// ---------------------------------------------------------------------------
// Tensor cores: mma.sync (registers) and tcgen05 (tensor memory)
// ---------------------------------------------------------------------------
// D[16x8] += A[16x16] * B[16x8], bf16 inputs, fp32 accumulate.
__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                               uint32_t a3, uint32_t b0, uint32_t b1)
{
    asm volatile("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
                 "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
                 : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
                 : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void tmem_alloc(uint32_t *smem_dst, uint32_t ncols)
{
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(smem_dst)),
                 "r"(ncols)
                 : "memory");
}

__device__ __forceinline__ void tmem_relinquish()
{
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols)
{
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
                 : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// D(tmem) (+)= A(tmem) * B(smem descriptor); kind::f16 with bf16 inputs.
__device__ __forceinline__ void umma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                        uint32_t idesc, uint32_t accumulate)
{
    asm volatile("{\n\t.reg .pred p;\n\t"
                 "setp.ne.b32 p, %4, 0;\n\t"
                 "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
                 "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
                 : "memory");
}

// Arrives once on the mbarrier when all previously issued tcgen05.mma of
// this thread have completed.
__device__ __forceinline__ void umma_commit(uint64_t *bar)
{
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     smem_u32(bar))
                 : "memory");
}

// Instruction descriptor, kind::f16: bf16 A and B, fp32 D, both K-major,
// M = 128 (weight rows), N = n (tokens).
__host__ __device__ constexpr uint32_t umma_idesc_bf16(int n)
{
    return (1u << 4)                          // D format fp32
           | (1u << 7)                        // A format bf16
           | (1u << 10)                       // B format bf16
           | ((uint32_t)(n >> 3) << 17)       // N >> 3
           | ((uint32_t)(128 >> 4) << 24);    // M >> 4
}

// Shared-memory matrix descriptor, K-major, 128-byte swizzle: rows of 128 B,
// 8-row groups 1024 B apart.  The tile must start 1024-byte aligned; moving
// along K inside the 128-byte row adds the byte offset to the start address.
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t saddr)
{
    return (uint64_t)((saddr >> 4) & 0x3FFFu)   // start address
           | ((uint64_t)1 << 16)                // leading byte offset (unused with swizzle)
           | ((uint64_t)(1024 >> 4) << 32)      // stride byte offset: 8 rows * 128 B
           | ((uint64_t)1 << 46)                // descriptor version (sm_100)
           | ((uint64_t)2 << 61);               // SWIZZLE_128B
}

// 16 TMEM lanes x 1024 bits (32 columns): thread (g = lane/4, t = lane%4)
// writes lanes g and g+8 at columns 2t, 2t+1 (+8, +16, +24 for each repeat).
__device__ __forceinline__ void tmem_st_16x256b_x4(uint32_t taddr, const uint32_t (&r)[16])
{
    asm volatile("tcgen05.st.sync.aligned.16x256b.x4.b32 [%0], "
                 "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
                 "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]),
                 "r"(r[7]), "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]),
                 "r"(r[14]), "r"(r[15])
                 : "memory");
}

__device__ __forceinline__ void tmem_st_16x256b_x2(uint32_t taddr, const uint32_t (&r)[8])
{
    asm volatile("tcgen05.st.sync.aligned.16x256b.x2.b32 [%0], "
                 "{%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(taddr),
                 "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]),
                 "r"(r[7])
                 : "memory");
}

// 32 TMEM lanes x 16 columns: thread i writes lane (quadrant base + i),
// 16 consecutive 32-bit columns.
__device__ __forceinline__ void tmem_st_32x32b_x16(uint32_t taddr, const uint32_t (&r)[16])
{
    asm volatile("tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
                 "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
                 "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]),
                 "r"(r[7]), "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]),
                 "r"(r[14]), "r"(r[15])
                 : "memory");
}

__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// 32 TMEM lanes x 16 columns: thread i gets lane (quadrant base + i), 16
// consecutive fp32 columns.
__device__ __forceinline__ void tmem_ld_32x32b_x16(uint32_t taddr, float (&v)[16])
{
    uint32_t r[16];
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x16.b32 "
                 "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]),
                   "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]),
                   "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
                 : "r"(taddr)
                 : "memory");
#pragma unroll
    for (int i = 0; i < 16; ++i)
        v[i] = __uint_as_float(r[i]);
}

// 32 TMEM lanes x 8 columns.
__device__ __forceinline__ void tmem_ld_32x32b_x8(uint32_t taddr, float (&v)[8])
{
    uint32_t r[8];
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
                 : "r"(taddr)
                 : "memory");
#pragma unroll
    for (int i = 0; i < 8; ++i)
        v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ void fence_proxy_async_smem()
{
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Barrier over a subset of the CTA's warps.  The non-aligned form, after a
// __syncwarp, so that a branch taken by one lane just before it (the ticket
// atomic) cannot leave the warp diverged at an aligned barrier.
__device__ __forceinline__ void named_barrier_sync(int id, int nthreads)
{
    __syncwarp();
    asm volatile("barrier.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// Ticket for "last CTA to arrive finishes the reduction": a release fence
// (covering the partials this CTA's threads stored before the barrier) and
// an acquire fence after the atomic.
__device__ __forceinline__ uint32_t ticket_take(uint32_t *counter)
{
    __threadfence();
    const uint32_t t = atomicAdd(counter, 1u);
    __threadfence();
    return t;
}

// Ticket with one acquire-release atomic at GPU scope: the release orders the
// partials the warp stored before a __syncwarp (cumulativity through the
// warp barrier), the acquire lets the last arriver read every other
// contributor's partials after a __syncwarp.  Called by one lane.
__device__ __forceinline__ uint32_t ticket_take_acq_rel(uint32_t *counter)
{
    uint32_t t;
    asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], 1;" : "=r"(t) : "l"(counter) : "memory");
    return t;
}

// ---------------------------------------------------------------------------
// Stream-K partition: U units cut into G contiguous ranges [start(c),
// start(c+1)); a panel of consecutive units may span several ranges.
// ---------------------------------------------------------------------------
WQ_HD int sk_start(long long U, int G, int c) { return (int)(U * c / G); }

// CTA that owns unit u (ranges [start(c), start(c+1)); empty ranges skipped)
WQ_HD int sk_owner(long long U, int G, int u)
{
    int c = (int)(((long long)u * G) / U);
    if (c >= G)
        c = G - 1;
    while (c + 1 < G && sk_start(U, G, c + 1) <= u)
        ++c;
    while (c > 0 && sk_start(U, G, c) > u)
        --c;
    return c;
}

// The stream-K cuts of the grid, computed once per CTA (one 64-bit division
// per thread) so that the flushes and fix-ups look them up instead of
// dividing: start[c] is the first unit of CTA c, first[c] its first panel.
struct SkTable {
    const int *start, *first;
    // CTA whose range holds unit u: the largest c with start[c] <= u (ranges
    // may be empty; the largest such c has start[c + 1] > u)
    WQ_HD int owner(int u, int G) const
    {
        int lo = 0, hi = G - 1;
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (start[mid] <= u)
                lo = mid;
            else
                hi = mid - 1;
        }
        return lo;
    }
};

// ---------------------------------------------------------------------------
// Integer -> bf16 conversions (exact; written from the IEEE-754 encodings).
// ---------------------------------------------------------------------------

// Four 4-bit codes taken as nibble pairs: returns bf16x2 {128 + n_i, 128 + n_{i+4}}
// for the nibbles at positions i and i+4 of the word shifted right by 4i.
// 0x4300 is bf16 128.0; its 7 mantissa bits hold any value 0..127 exactly.
__device__ __forceinline__ uint32_t nib_pair_bf16(uint32_t w_shifted)
{
    uint32_t r;
    asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(r) : "r"(w_shifted), "r"(0x000F000Fu), "r"(0x43004300u));
    return r; // (a & b) | c
}

// bf16x2 subtract of two exact small integers: exact.
__device__ __forceinline__ uint32_t bf16x2_sub(uint32_t a, uint32_t b)
{
    uint32_t r;
    asm("sub.rn.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    return r;
}

__device__ __forceinline__ uint32_t bf16x2_mul(uint32_t a, uint32_t b)
{
    uint32_t r;
    asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    return r;
}

// Two int8 values (bytes 2h and 2h+1 of w, already offset to unsigned by
// x ^ 0x80) -> bf16x2 of the signed values.  2^23 + u is built in the binary32
// mantissa, the offset 2^23 + 128 is subtracted exactly, and |q| <= 128 has at
// most 8 significant bits, so the bf16 conversion is exact.
__device__ __forceinline__ uint32_t s8pair_bf16(uint32_t u, int h)
{
    const float f0 = __uint_as_float(__byte_perm(u, 0x4B000000u, h == 0 ? 0x7540u : 0x7542u));
    const float f1 = __uint_as_float(__byte_perm(u, 0x4B000000u, h == 0 ? 0x7541u : 0x7543u));
    const float q0 = f0 - 8388736.0f; // 2^23 + 128
    const float q1 = f1 - 8388736.0f;
    __nv_bfloat162 b = __floats2bfloat162_rn(q0, q1); // exact: integers |q| <= 128
    return *reinterpret_cast<uint32_t *>(&b);
}

__device__ __forceinline__ float bf16_bits_to_float(uint16_t b) { return __uint_as_float((uint32_t)b << 16); }

} // namespace wq
