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

__device__ __forceinline__ double i8_value(int32_t d0, int32_t d1, int32_t d2, double scale_pow2)
{
    return ((double)d2 * 65536.0 + (double)d1 * 256.0 + (double)d0) * scale_pow2;
}

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

// As digit_planes, and adds to `res` the sum over the 16 elements of the
// rounding residual |x * 2^e - X|: x * 2^e is exact in binary32 (a power-of-
// two scale of an 8-bit significand), X = F - 1.5 * 2^23 is exact, and the
// fused multiply-add x * 2^e - X rounds nothing (|r| <= 1/2 and its bits lie
// within those of x * 2^e).
__device__ __forceinline__ void digit_planes(const uint32_t (&w)[8], float s, uint32_t (&p)[3][4], float &res)
{
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const float lo = __uint_as_float(w[i] << 16), hi = __uint_as_float(w[i] & 0xFFFF0000u);
        const float xl = fmaf(lo, s, 12582912.0f) - 12582912.0f, xh = fmaf(hi, s, 12582912.0f) - 12582912.0f;
        res += fabsf(fmaf(lo, s, -xl)) + fabsf(fmaf(hi, s, -xh));
    }
    digit_planes(w, s, p);
}

// ---------------------------------------------------------------------------
// Exactness guard of the integer path.
//
// Rounding x to X = round(x 2^e) changes y[m][n] by
//     |sum_k w[n][k] (x[m][k] - X[m][k] 2^-e_m)| <= max_k |w[n][k]| * 2^-e_m * R_m,
// R_m = sum_k |x[m][k] 2^e_m - X[m][k]| (each term <= 1/2; zero for every
// element within 2^14 of the row's largest).  The digit phases accumulate an
// upper bound of R_m in units of 2^-24 (an integer sum, the same in any
// order, so every CTA takes the same decisions on every run); the epilogues
// compare the bound with the output's tolerance and recompute, in binary64
// straight from x and the packed codes, every output where the bound does not
// show |y - y_exact| <= 2^-9 max(|y|, 1).  With the bf16 rounding of the
// output that keeps every output within 2^-8 max(|y_exact|, 1) of the exact
// sum, inside the 1e-2 relative tolerance of the layer.  A row of ordinary
// dynamic range never takes the binary64 path; a row holding elements far
// below its largest (an outlier 2^12 above the rest) can take it for many
// outputs, which is slow but exact.
// ---------------------------------------------------------------------------
constexpr double kExactTol = 1.0 / 512.0;

// A 16-element residual sum (binary32, each term <= 1/2) as an upper bound in
// units of 2^-24: the float sum's relative error is below 2^-19, and one
// unit more covers the ceiling.
__device__ __forceinline__ uint32_t residual_units(float res)
{
    return res > 0.f ? (uint32_t)ceilf(res * 16777216.0f * 1.00001f) + 1u : 0u;
}

// Adds `units` to counter[m]: one atomic per warp when the whole warp works
// on the same token row m (the usual case), else one per lane.  All 32
// lanes call it together.
__device__ __forceinline__ void residual_add(unsigned long long *counter, int m, uint32_t units)
{
    const int m0 = __shfl_sync(0xffffffffu, m, 0);
    if (__all_sync(0xffffffffu, m == m0)) {
        unsigned long long u = units;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1)
            u += __shfl_xor_sync(0xffffffffu, u, o);
        if ((threadIdx.x & 31) == 0 && u)
            atomicAdd(&counter[m0], u);
    } else if (units) {
        atomicAdd(&counter[m], (unsigned long long)units);
    }
}

// Bound on |y - y_exact| per unit of max|w| for token row m: units * 2^-24 * 2^-e_m.
__device__ __forceinline__ double residual_bound(unsigned long long units, int e_m)
{
    return (double)units * __longlong_as_double((long long)(1023 - 24 - e_m) << 52);
}

__device__ __forceinline__ bool exact_enough(double y, double bound)
{
    return bound <= kExactTol * fmax(fabs(y), 1.0); // false for NaN: recomputed
}

// Binary64 dot product of token row xm (bf16, K elements) with packed weight
// row n, dequantized from the codes (INT8: sum x q, the caller applies s[n];
// INT4: sum_g s[n][g] sum_{k in g} x (q - z[n][g])).  All 32 lanes of the
// warp call it together and all receive the same sum (fixed order: lane
// partial sums, then a butterfly).  The recompute of the exactness guard.
// Kept out of line: it runs only for the outputs the guard rejects, and the
// callers' streaming loops stay as small as without it.
template <int BITS>
__device__ __noinline__ double packed_row_dot(const uint8_t *__restrict__ wq, const uint16_t *__restrict__ scales,
                                 const uint8_t *__restrict__ zeros, int K, int KB, int n,
                                 const uint16_t *__restrict__ xm, int lane)
{
    const int p = n >> 7, r = n & 127;
    double acc = 0.0;
    // 8 items of 16 k per 128-k block
    for (int it = lane; it < KB * 8; it += 32) {
        const int kb = it >> 3;
        const size_t blk = (size_t)p * KB + kb;
        if constexpr (BITS == 8) {
            const int k0 = kb * kBlockK + 16 * (it & 7);
            if (k0 >= K)
                continue; // codes past K are zero
            const uint4 qv = __ldg(reinterpret_cast<const uint4 *>(wq + (blk << 14) + int8_chunk_in_block(r, it & 7)));
            const uint4 xa = __ldg(reinterpret_cast<const uint4 *>(xm + k0));
            const uint4 xb = __ldg(reinterpret_cast<const uint4 *>(xm + k0 + 8));
            const uint32_t qw[4] = {qv.x, qv.y, qv.z, qv.w};
            const uint32_t xw[8] = {xa.x, xa.y, xa.z, xa.w, xb.x, xb.y, xb.z, xb.w};
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const int q = (int)(int8_t)((qw[i >> 2] >> (8 * (i & 3))) & 0xFFu);
                const uint32_t xb16 = (xw[i >> 1] >> (16 * (i & 1))) & 0xFFFFu;
                acc = fma((double)q, (double)bf16_bits_to_float((uint16_t)xb16), acc);
            }
        } else {
            const int tau = (it >> 2) & 1, t = it & 3;
            const int j = r >> 4, rr = r & 15, g = rr & 7, h = rr >> 3;
            const uint4 v = __ldg(reinterpret_cast<const uint4 *>(wq + (blk << 13) + (size_t)j * 1024 + tau * 512 +
                                                                   16 * (4 * g + t)));
            const uint32_t w0 = h ? v.y : v.x, w1 = h ? v.w : v.z; // runs (a, b) and (c, d)
            const int kt = kb * kBlockK + 64 * tau;
            const double sg = (double)bf16_bits_to_float(scales[blk * kPanelRows + r]);
            const int z = (int)((zeros[blk * 64 + (r >> 1)] >> (4 * (r & 1))) & 0xFu);
            const int kr[4] = {kt + 4 * t, kt + 16 + 4 * t, kt + 32 + 4 * t, kt + 48 + 4 * t};
            double part = 0.0;
#pragma unroll
            for (int run = 0; run < 4; ++run) {
                const uint32_t w = run < 2 ? w0 : w1;
                const uint2 xv = __ldg(reinterpret_cast<const uint2 *>(xm + kr[run]));
                const uint32_t xw[2] = {xv.x, xv.y};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int pos = int4_nibble_pos((run & 1) * 4 + e);
                    const int q = (int)((w >> (4 * pos)) & 0xFu);
                    const uint32_t xb16 = (xw[e >> 1] >> (16 * (e & 1))) & 0xFFFFu;
                    part = fma((double)(q - z), (double)bf16_bits_to_float((uint16_t)xb16), part);
                }
            }
            acc = fma(sg, part, acc);
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
        acc += __shfl_xor_sync(0xffffffffu, acc, o);
    return acc;
}

// Writes y[m][n] = v for the warp's 32 consecutive weight rows n = nb + lane
// (token m the same across the warp; rows at or past N write nothing).  An
// output whose bound the exactness guard cannot accept is recomputed by the
// whole warp in binary64 (packed_row_dot; INT8 times s[n]).
template <int BITS>
__device__ __forceinline__ void imma_emit_rows(const uint16_t *__restrict__ x, const uint8_t *__restrict__ wq,
                                               const uint16_t *__restrict__ scales, const uint8_t *__restrict__ zeros,
                                               uint16_t *y, int K, int KB, int N, int nb, int m, double v,
                                               double bound, int lane)
{
    const int n = nb + lane;
    const bool redo = n < N && !exact_enough(v, bound);
    if (n < N && !redo)
        y[(size_t)m * N + n] = __bfloat16_as_ushort(__double2bfloat16(v));
    for (uint32_t mask = __ballot_sync(0xffffffffu, redo); mask; mask &= mask - 1) {
        const int src = __ffs(mask) - 1, nn = nb + src;
        double r = packed_row_dot<BITS>(wq, scales, zeros, K, KB, nn, x + (size_t)m * K, lane);
        if constexpr (BITS == 8)
            r *= (double)bf16_bits_to_float(scales[nn]);
        if (lane == src)
            y[(size_t)m * N + nn] = __bfloat16_as_ushort(__double2bfloat16(r));
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
                                                 int et, uint8_t *xd, uint32_t *s_amax, int *s_e, uint32_t *grid,
                                                 unsigned long long *g_res)
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
            uint32_t units = 0;
#pragma unroll
            for (int h = 0; h < NV / 2; ++h) {
                const uint4 &a = v[2 * h], &b = v[2 * h + 1];
                const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
                float res = 0.f;
                digit_planes(w, sc, pl[h], res);
                units += residual_units(res);
            }
            if (units) // this CTA's share of the row's residual sum (exactness guard)
                atomicAdd(&g_res[m], (unsigned long long)units);
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

// After the digit phase, by the same 128 threads: once every CTA has counted
// itself on grid[0] (acquire, bounded), the residual bound of every token row
// into s_rb (residual_bound of the grid-wide sum).  False if the wait gave up.
__device__ __forceinline__ bool imma_residual_bounds(int M, int G, int et, const uint32_t *grid,
                                                     const unsigned long long *g_res, const int *s_e, double *s_rb)
{
    bool ok = true;
    if (et < M) {
        const uint64_t t0 = globaltimer_ns();
        while (ld_acquire_gpu(grid) < (uint32_t)G) {
            if (globaltimer_ns() - t0 > kWaitLimitNs) {
                ok = false;
                break;
            }
        }
        s_rb[et] = ok ? residual_bound(__ldcg(g_res + et), s_e[et]) : 0.0;
    }
    named_barrier_sync(1, 128);
    return ok;
}

} // namespace wq
