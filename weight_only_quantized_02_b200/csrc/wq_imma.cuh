// wq_imma.cuh -- pieces shared by the integer tensor-core kernels (W8A16
// and W4A16 on tcgen05.mma kind::i8): instruction descriptor and MMA, the
// activations' base-256 digits, and the in-kernel digit phase with its grid
// counter.
//
// Activations: every token row of x becomes integers X = round(x * 2^e_m),
// ties to even, e_m = min(21 - E, 127) for 2^E <= max|x_m| < 2^(E+1), so
// |X| < 2^22; X = d0 + 256 d1 + 65536 d2 with d0, d1 in [-128, 127] and
// |d2| <= 64.  The digit block of a 128-k block holds NR rows of 128 bytes
// (row 3m + i = digit i of token m; rows 3M .. NR-1 zero) in the same
// tcgen05 K-major 128-byte-swizzled layout as an INT8 weight block.
#pragma once

#include <cstdint>

#include <cuda_bf16.h>

#include "wq_device.cuh"
#include "wq_layout.h"

namespace wq {

// Instruction descriptor, kind::i8: signed 8-bit A and B, int32 D, both
// K-major, M = 128 (weight rows), N = n (digit rows).
__host__ __device__ constexpr uint32_t umma_idesc_s8(int n)
{
    return (2u << 4)                          // D format s32
           | (1u << 7)                        // A format signed 8-bit
           | (1u << 10)                       // B format signed 8-bit
           | ((uint32_t)(n >> 3) << 17)       // N >> 3
           | ((uint32_t)(128 >> 4) << 24);    // M >> 4
}

// D(tmem) (+)= A(smem descriptor) * B(smem descriptor); kind::i8.
__device__ __forceinline__ void umma_ss_i8(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                           uint32_t accumulate)
{
    asm volatile("{\n\t.reg .pred p;\n\t"
                 "setp.ne.b32 p, %4, 0;\n\t"
                 "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
                 "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
                 : "memory");
}

// 2^e as a binary64, built from its exponent field (|e| < 1000 here).
__device__ __forceinline__ double pow2_of(int e) { return __longlong_as_double((long long)(1023 + e) << 52); }

__device__ __forceinline__ uint16_t i8_output(int32_t d0, int32_t d1, int32_t d2, double scale_pow2)
{
    const double v = ((double)d2 * 65536.0 + (double)d1 * 256.0 + (double)d0) * scale_pow2;
    return __bfloat16_as_ushort(__double2bfloat16(v));
}

// Exponent e_m of a token row from the largest magnitude's bf16 bits:
// |x| < 2^(E+1), e = 21 - E gives |X| < 2^22.  Rows whose largest magnitude
// is below 2^-106 use e = 127 (the largest power of two a binary32 holds).
__device__ __forceinline__ int row_exponent(uint32_t amax_bits)
{
    if (amax_bits == 0)
        return 0;
    const int eb = (int)(amax_bits >> 7);
    const int e = 21 - ((eb ? eb : 1) - 127);
    return e > 127 ? 127 : e;
}

// 16 consecutive activations (bf16 bits in w[8]) -> the digit planes of one
// 16-byte chunk: p[i][j] = bytes 4j..4j+3 of digit plane i.  With the fused
// multiply-add F = x * 2^e + 1.5 * 2^23 rounded once (to nearest, ties to
// even), the binary32 bits of F are 0x4B400000 + X for |X| < 2^22, and
// X + 0x808080 holds the three biased digits d_i + 128 in its low three
// bytes (the balanced base-256 expansion is unique, so no byte carries).
__device__ __forceinline__ void digit_planes(const uint32_t (&w)[8], float s, uint32_t (&p)[3][4])
{
    uint32_t Y[16];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const float lo = __uint_as_float(w[i] << 16), hi = __uint_as_float(w[i] & 0xFFFF0000u);
        Y[2 * i] = __float_as_uint(fmaf(lo, s, 12582912.0f)) - 0x4ABF7F80u;     // X + 0x808080
        Y[2 * i + 1] = __float_as_uint(fmaf(hi, s, 12582912.0f)) - 0x4ABF7F80u;
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const uint32_t a01 = __byte_perm(Y[4 * j], Y[4 * j + 1], 0x5140u);     // d0 d0 d1 d1
        const uint32_t a23 = __byte_perm(Y[4 * j + 2], Y[4 * j + 3], 0x5140u);
        const uint32_t b01 = __byte_perm(Y[4 * j], Y[4 * j + 1], 0x0062u);     // d2 d2 . .
        const uint32_t b23 = __byte_perm(Y[4 * j + 2], Y[4 * j + 3], 0x0062u);
        p[0][j] = __byte_perm(a01, a23, 0x5410u) ^ 0x80808080u; // biased -> two's complement
        p[1][j] = __byte_perm(a01, a23, 0x7632u) ^ 0x80808080u;
        p[2][j] = __byte_perm(b01, b23, 0x5410u) ^ 0x80808080u;
    }
}

__device__ __forceinline__ uint32_t ld_acquire_gpu(const uint32_t *p)
{
    uint32_t v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ void red_release_gpu_add(uint32_t *p, uint32_t v)
{
    asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

__device__ __forceinline__ void fence_proxy_async_global()
{
    asm volatile("fence.proxy.async.global;" ::: "memory");
}

// 16-byte asynchronous global -> shared copy (L2 only), outside the bulk-copy
// engine's queue.
__device__ __forceinline__ void cp_async_16(void *dst_smem, const void *src)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst_smem)), "l"(src) : "memory");
}

// The mbarrier receives one arrival when every cp.async this thread issued
// before has completed (its expected count includes these arrivals).
__device__ __forceinline__ void cp_async_mbar_arrive_noinc(uint64_t *bar)
{
    asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// Row maxima of x (bf16 magnitude bits, the order of magnitudes) by NTH
// threads et = 0 .. NTH-1, BATCH 16-byte loads in flight per thread; each
// thread's running maximum per row is folded into s_amax[m] (zeroed by the
// caller) with a shared-memory atomicMax.  The caller synchronizes before reading s_amax.
template <int NTH, int BATCH = 8>
__device__ __forceinline__ void imma_row_maxima(const uint16_t *__restrict__ x, int M, int K, int et,
                                                uint32_t *s_amax)
{
    const int vpr = K / 8; // 16-byte vectors per token row
    const int total = M * vpr; // M <= 128, K <= 65536: 32-bit index arithmetic
    int cur_m = -1;
    uint32_t cur = 0;
    for (int v0 = et; v0 < total; v0 += BATCH * NTH) {
        uint4 q[BATCH];
#pragma unroll
        for (int b = 0; b < BATCH; ++b) {
            const int v = v0 + b * NTH;
            q[b] = v < total ? ldg_keep4(x + (size_t)v * 8) : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int b = 0; b < BATCH; ++b) {
            const int v = v0 + b * NTH;
            if (v >= total)
                break;
            const int m = v / vpr;
            if (m != cur_m) {
                if (cur_m >= 0)
                    atomicMax(&s_amax[cur_m], cur);
                cur_m = m;
                cur = 0;
            }
            const uint32_t wv[4] = {q[b].x, q[b].y, q[b].z, q[b].w};
#pragma unroll
            for (int h = 0; h < 4; ++h)
                cur = max(cur, max(wv[h] & 0x7FFFu, (wv[h] >> 16) & 0x7FFFu));
        }
    }
    if (cur_m >= 0)
        atomicMax(&s_amax[cur_m], cur);
}

// The digit phase, run by 128 threads (et = 0..127) of CTA c of G after the
// programmatic-launch wait: the row maxima of x (every CTA computes all of
// them, into s_amax / s_e), then CTA c's 1/G share of the digit blocks
// (items = token slot, k-block, 16-k chunk; slots M .. ceil(NR/3)-1 write
// the zero padding rows) into xd, then one release increment of grid[0].
// Uses named barrier 1.  Each thread's first item is loaded together with
// the row maxima, so the phase costs one round trip to L2.
//
// PAIRED = false: natural k order (byte k of the block's row = k).
// PAIRED = true: the k order of an A operand stored in tensor memory with
// tcgen05.st 16x256b from the packed INT4 tiles: in each 32-k step, byte
// 8t + 4s + e holds k = 16s + 4t + e (the 4-byte words of the step's two
// 16-k chunks interleaved).  An item is then a whole 32-k step.
template <int NR, bool PAIRED = false>
__device__ __forceinline__ void imma_digit_phase(const uint16_t *__restrict__ x, int M, int K, int KB, int c, int G,
                                                 int et, uint8_t *xd, uint32_t *s_amax, int *s_e, uint32_t *grid)
{
    constexpr int BB = NR * 128;
    constexpr int W = PAIRED ? 32 : 16;  // k per item
    constexpr int IPB = kBlockK / W;     // items per k-block and token slot
    constexpr int NV = W / 8;            // 16-byte activation vectors per item
    // items (token slot m, k-block, W-k step); slots M .. ceil(NR/3)-1 write the zero padding rows
    constexpr int MS = (NR + 2) / 3;
    const int items = MS * KB * IPB; // items * G stays below 2^32: 32-bit index arithmetic
    const int i0 = (int)((unsigned)items * (unsigned)c / (unsigned)G),
              i1 = (int)((unsigned)items * (unsigned)(c + 1) / (unsigned)G);
    auto item_x = [&](int it, uint4 (&v)[NV]) {
        const int m = it / (KB * IPB), rem = it % (KB * IPB);
        const int k0 = (rem / IPB) * kBlockK + W * (rem % IPB);
#pragma unroll
        for (int j = 0; j < NV; ++j) // k past K or a padding slot: zero activations (zero weights there too)
            v[j] = (m < M && k0 + 8 * j < K) ? ldg_keep4(x + (size_t)m * K + k0 + 8 * j) : make_uint4(0, 0, 0, 0);
    };
    // this thread's first item is loaded together with the row maxima (one round trip)
    uint4 first[NV];
#pragma unroll
    for (int j = 0; j < NV; ++j)
        first[j] = make_uint4(0, 0, 0, 0);
    if (i0 + et < i1)
        item_x(i0 + et, first);
    imma_row_maxima<128>(x, M, K, et, s_amax);
    named_barrier_sync(1, 128);
    if (et < M)
        s_e[et] = row_exponent(s_amax[et]);
    named_barrier_sync(1, 128);
    for (int it = i0 + et; it < i1; it += 128) {
        const int m = it / (KB * IPB), rem = it % (KB * IPB);
        const int kb = rem / IPB, st = rem % IPB;
        uint4 v[NV];
#pragma unroll
        for (int j = 0; j < NV; ++j)
            v[j] = first[j];
        if (it != i0 + et)
            item_x(it, v);
        // digit planes of the item's 16-k chunks: pl[h][d][word]
        uint32_t pl[NV / 2][3][4];
#pragma unroll
        for (int h = 0; h < NV / 2; ++h)
#pragma unroll
            for (int d = 0; d < 3; ++d)
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    pl[h][d][q] = 0u;
        if (m < M) {
            const float sc = __uint_as_float((uint32_t)(127 + s_e[m]) << 23); // 2^e, -106 <= e <= 127
#pragma unroll
            for (int h = 0; h < NV / 2; ++h) {
                const uint4 &a = v[2 * h], &b = v[2 * h + 1];
                const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
                digit_planes(w, sc, pl[h]);
            }
        }
        uint8_t *blk = xd + (size_t)kb * BB;
#pragma unroll
        for (int d = 0; d < 3; ++d) {
            const int jr = 3 * m + d;
            if (jr >= NR)
                continue;
            uint8_t *rowp = blk + (jr >> 3) * 1024 + (jr & 7) * 128;
            if constexpr (PAIRED) {
                // 32-k step st = chunks 2st (s = 0) and 2st + 1 (s = 1): word t of chunk s
                // goes to byte 8t + 4s of the step
                const int c0 = 2 * st, c1 = c0 + 1;
                *reinterpret_cast<uint4 *>(rowp + ((c0 ^ (jr & 7)) << 4)) =
                    make_uint4(pl[0][d][0], pl[1][d][0], pl[0][d][1], pl[1][d][1]);
                *reinterpret_cast<uint4 *>(rowp + ((c1 ^ (jr & 7)) << 4)) =
                    make_uint4(pl[0][d][2], pl[1][d][2], pl[0][d][3], pl[1][d][3]);
            } else {
                *reinterpret_cast<uint4 *>(rowp + ((st ^ (jr & 7)) << 4)) =
                    make_uint4(pl[0][d][0], pl[0][d][1], pl[0][d][2], pl[0][d][3]);
            }
        }
    }
    fence_proxy_async_global();
    named_barrier_sync(1, 128);
    if (et == 0)
        red_release_gpu_add(&grid[0], 1u); // cumulative over the 128 threads' stores
}

} // namespace wq
