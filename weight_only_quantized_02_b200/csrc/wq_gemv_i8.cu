// wq_gemv_i8.cu -- decode-regime GEMV (M <= 8) on the integer mma.sync
// path: mma.sync m16n8k32 s8 x s8 -> s32 straight on the packed weight
// codes, the activations as exact base-256 digits.
//
// The sum over k of the weight-only linear layer is an integer sum once the
// activations are integers ("Per-channel W8A16 quantization" and
// "Group-wise W4A16 quantization", tileInfer README, Features table):
//     W8A16:  y[m][n] = s[n] 2^-e_m sum_k q[n][k] X[m][k]
//     W4A16:  y[m][n] = 2^-e_m sum_g s[g][n] (sum_{k in g} q[n][k] X[m][k] - z[g][n] sum_{k in g} X[m][k])
// with X = round(x 2^e_m) = d0 + 256 d1 + 65536 d2 (the activations'
// fixed-point form of the integer tensor-core kernels, wq_imma.cuh).  The
// A operand of every MMA is the packed weights exactly as they sit in HBM:
// INT8 codes need no instruction at all, INT4 codes one mask (and one shift)
// per 4 nibbles; the zero point becomes one integer multiply-add per output
// and group with the digit sum of the group.  The bf16-dequantizing GEMV
// spends several instructions per weight and is issue-bound below HBM
// bandwidth at decode sizes; this one issues a fraction of that.
//
// Activations: every CTA first turns all of x into digit rows in its own
// shared memory (row maxima, then the digits; M*K values, a few tens per
// thread at decode sizes), so no CTA waits for another and the B fragments
// come from shared memory.  The digit rows' byte order inside a 128-k block
// matches the weights' k order (INT8: natural; INT4: the nibble order of
// the packed mma tiles, see gi_digits), so a lane's B fragment is one
// contiguous load.
//
// Work split: each CTA owns LB = (N/16) / G whole 16-row blocks, split in
// equal contiguous runs of chunks (D k-blocks of one row block) between
// most of its warps; the remaining row blocks' chunks are cut stream-K
// style between the CTAs, and each CTA's share between its first few warps
// (see gi_cta).  Each warp streams its run through a D-deep ring of
// register prefetches (the first D issued before the programmatic-launch
// wait: weights never depend on the preceding kernel).  A CTA's own row
// block split between its warps is summed from shared memory once all of
// them are done: no round trip to L2 at the end of the stream.  A shared
// row block is finished by the last contributor to take its ticket
// (acquire-release, never waited on), which sums the partials in
// contributor order and writes y (INT8 partials are exact integers).
#include <cstdint>

#include <cuda_bf16.h>

#include "wq.h"
#include "wq_device.cuh"
#include "wq_imma.cuh"
#include "wq_internal.h"

namespace wq {

// Warps of the stream-K partition (every launch shape): at most kGiMaxCtas * 8.
constexpr int kGiMaxWarps = kGiMaxCtas * 8;

struct GiParams {
    const uint16_t *x;
    int M, K, N, KB;
    int CPR;        // chunks (D consecutive k-blocks, the last one ragged) per 16-row block
    int LB;         // 16-row blocks each CTA owns whole: CTA c has c LB .. c LB + LB - 1
    int RB0;        // G LB: row blocks RB0 .. N/16 - 1 are shared between CTAs
    int RL;         // chunks of the shared row blocks, (N/16 - RB0) CPR
    const uint8_t *wq;
    const uint16_t *scales;
    const uint8_t *zeros;
    uint16_t *y;
    uint32_t *part; // [kGiMaxWarps][2 slots][16 rows][NR] partials
    uint32_t *cnt;  // one ticket per 16-row block
    const uint32_t *wmax; // INT4: max |s (q - z)| over the whole weight (binary32 bits, packed trailer)
};

// Prefetch depth (items in flight per warp) by weight format.
template <int BITS>
struct GiCfg {
    static constexpr int D = BITS == 8 ? 4 : 6;
};

__device__ __forceinline__ void imma_16832(int32_t (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                           uint32_t b0, uint32_t b1)
{
    asm volatile("mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 "
                 "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
                 : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
                 : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Shared-memory digit rows: row 3m + i (digit i of token m) of S bytes,
// S = 128 * KB + 64 (INT8) or K + 16 (INT4): the stride puts the two rows a
// quarter-warp reads in different banks.  INT4 adds the digit sums of every
// row and 128-k block.
template <int BITS>
__host__ __device__ constexpr int gi_row_stride(int K)
{
    return BITS == 8 ? (K + 127) / 128 * 128 + 64 : K + 16;
}

// The activations of the whole layer as digit rows in shared memory (all
// NTH threads of the CTA): the row maxima (e_m), then every 16-k chunk of every token
// row, thread ch = chunk % 8 of each group of eight converting k = 16 c ..
// 16 c + 15 (zero past K).  Each CTA converts all of x (M*K values, a few
// tens per thread at decode sizes) and no CTA waits for another.  Digit row
// 3m + i of block kb holds its 128 bytes in the order the B fragments read:
//   INT8: natural, byte kk holds k = kk (a lane's 16-byte weight chunk and
//         its 16 digit bytes cover the same k).
//   INT4: byte 32 t + 8 st + 2 a + s holds k = 32 st + 16 s + 4 t + a: the
//         packed mma tile gives lane t of 32-k step st the nibbles of
//         k = 4t + a (low nibbles) and 16 + 4t + a (high nibbles) interleaved,
//         so a lane's 32 bytes of a block are its four steps' B fragments.
template <int BITS, int NR, int NTH>
__device__ __forceinline__ void gi_digits(const GiParams &p, uint8_t *sd, int32_t *s_dsum, uint32_t *s_amax,
                                          int *s_e, unsigned long long *s_res)
{
    const int et = threadIdx.x, ch = et & 7;
    const int M = p.M, K = p.K, KB = p.KB;
    const int S = gi_row_stride<BITS>(K);
    const int cpr = KB * 8; // 16-k chunks per token row
    const int items = M * cpr;
    // The thread's first HOLD chunks are loaded once, together (one round
    // trip to L2), and kept in registers from the row maxima to the digits;
    // chunks beyond HOLD * NTH (M > 4 at K = 5120 with 512 threads) are
    // loaded in both passes.
    constexpr int HOLD = NR == 8 ? 2 : 3;
    auto load_chunk = [&](int it, uint4 &a, uint4 &b) {
        a = make_uint4(0, 0, 0, 0);
        b = a;
        const int m = it / cpr, c = it % cpr; // chunk c: k = 16c .. 16c + 15
        if (it < items && 16 * c < K) {
            const uint16_t *src = p.x + (size_t)m * K + 16 * c;
            a = ldg_keep4(src);
            b = ldg_keep4(src + 8);
        }
    };
    auto chunk_max = [&](int it, const uint4 &a, const uint4 &b) {
        if (it >= items)
            return;
        const uint32_t wv[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
        uint32_t mx = 0;
#pragma unroll
        for (int h = 0; h < 8; ++h)
            mx = max(mx, max(wv[h] & 0x7FFFu, (wv[h] >> 16) & 0x7FFFu));
        atomicMax(&s_amax[it / cpr], mx);
    };
    uint4 ha[HOLD], hb[HOLD];
#pragma unroll
    for (int h = 0; h < HOLD; ++h)
        load_chunk(h * NTH + et, ha[h], hb[h]);
#pragma unroll
    for (int h = 0; h < HOLD; ++h)
        chunk_max(h * NTH + et, ha[h], hb[h]);
    for (int it = HOLD * NTH + et; it < items; it += NTH) {
        uint4 a, b;
        load_chunk(it, a, b);
        chunk_max(it, a, b);
    }
    __syncthreads();
    if (et < M)
        s_e[et] = row_exponent(s_amax[et]);
    __syncthreads();
    // chunk it (bf16 in a, b) -> its digit rows; all threads of a warp call
    // it together (the INT4 byte order is made with shuffles)
    auto convert = [&](int it, const uint4 &a, const uint4 &b) {
        const bool act = it < items;
        const int m = act ? it / cpr : 0, c = act ? it % cpr : 0;
        uint32_t pl[3][4];
#pragma unroll
        for (int i = 0; i < 3; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j)
                pl[i][j] = 0u;
        uint32_t units = 0;
        if (act) {
            const float sc = __uint_as_float((uint32_t)(127 + s_e[m]) << 23); // 2^e
            const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
            float res = 0.f;
            digit_planes(w, sc, pl, res);
            units = residual_units(res);
        }
        residual_add(s_res, m, units);
        if constexpr (BITS == 8) {
            if (act) {
#pragma unroll
                for (int i = 0; i < 3; ++i)
                    *reinterpret_cast<uint4 *>(sd + (3 * m + i) * S + 16 * c) =
                        make_uint4(pl[i][0], pl[i][1], pl[i][2], pl[i][3]);
            }
        } else {
            const int kb = c >> 3, s = ch & 1, st = ch >> 1;
#pragma unroll
            for (int i = 0; i < 3; ++i) {
                uint32_t o[4];
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    o[j] = __shfl_xor_sync(0xffffffffu, pl[i][j], 1);
                // lo: the chunk of step st with s = 0, hi: with s = 1
                uint32_t lo[4], hi[4];
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    lo[j] = s ? o[j] : pl[i][j];
                    hi[j] = s ? pl[i][j] : o[j];
                }
                int sum = 0;
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    sum = __dp4a((int)pl[i][j], 0x01010101, sum);
                sum += __shfl_xor_sync(0xffffffffu, sum, 1);
                sum += __shfl_xor_sync(0xffffffffu, sum, 2);
                sum += __shfl_xor_sync(0xffffffffu, sum, 4);
                if (act) {
                    uint8_t *row = sd + (3 * m + i) * S + kb * 128 + 8 * st;
#pragma unroll
                    for (int h = 0; h < 2; ++h) { // this thread writes lanes t = 2s, 2s + 1
                        const int t = 2 * s + h;
                        const uint32_t x0 = s ? lo[2 + h] : lo[h], x1 = s ? hi[2 + h] : hi[h];
                        *reinterpret_cast<uint2 *>(row + 32 * t) =
                            make_uint2(__byte_perm(x0, x1, 0x5140u), __byte_perm(x0, x1, 0x7362u));
                    }
                    if (ch == 0)
                        s_dsum[kb * NR + 3 * m + i] = sum;
                }
            }
        }
    };
#pragma unroll
    for (int h = 0; h < HOLD; ++h)
        if (h * NTH < items) // uniform
            convert(h * NTH + et, ha[h], hb[h]);
    for (int base = HOLD * NTH; base < items; base += NTH) { // uniform trip count: shuffles
        uint4 a, b;
        load_chunk(base + et, a, b);
        convert(base + et, a, b);
    }
    __syncthreads();
}

// Stream-K cuts in 32-bit arithmetic (every U * c and u * G here stays far
// below 2^32; the launch checks the bound): range c of G over U units
// starts at U c / G; gi_owner is the range holding unit u.
__host__ __device__ __forceinline__ int gi_start(int U, int G, int c)
{
    return (int)((unsigned)U * (unsigned)c / (unsigned)G);
}

__host__ __device__ __forceinline__ int gi_owner(int U, int G, int u)
{
    int c = (int)((unsigned)u * (unsigned)G / (unsigned)U);
    c = c < G - 1 ? c : G - 1;
    while (c + 1 < G && gi_start(U, G, c + 1) <= u)
        ++c;
    while (c > 0 && gi_start(U, G, c) > u)
        --c;
    return c;
}

// CTA c's work: its stream-K share [lo, lo + L) of the RL chunks of the
// shared row blocks, taken by its first ws warps, and its LB own row blocks
// (own = LB CPR chunks), split between the other WARPS - ws warps.  A shared
// warp gets about 0.8 of an even share: its tickets and fix-ups (round trips
// to L2) take the rest of its time.  With no own row blocks every warp is a
// shared warp.
struct GiCta {
    int lo, L, ws;
};

__host__ __device__ __forceinline__ GiCta gi_cta(const GiParams &p, int G, int c, int warps)
{
    GiCta t;
    t.lo = gi_start(p.RL, G, c);
    t.L = gi_start(p.RL, G, c + 1) - t.lo;
    const int own = p.LB * p.CPR;
    if (t.L == 0) {
        t.ws = 0;
    } else if (own == 0) {
        t.ws = warps;
    } else {
        const int ws = (5 * t.L * warps + 4 * (t.L + own) - 1) / (4 * (t.L + own)); // ceil(1.25 L warps / total)
        t.ws = ws < 1 ? 1 : ws > warps / 2 ? warps / 2 : ws;
    }
    return t;
}

// Warp `warp` of CTA c: n chunks from chunk q0 of row block rb0 (shared
// warps: its cut of the CTA's shared chunks; the others: its cut of the
// CTA's own row blocks).
__host__ __device__ __forceinline__ void gi_warp_run(const GiParams &p, const GiCta &ct, int c, int warp, int warps,
                                                     int &rb0, int &q0, int &n)
{
    if (warp < ct.ws) {
        const int o0 = gi_start(ct.L, ct.ws, warp);
        n = gi_start(ct.L, ct.ws, warp + 1) - o0;
        rb0 = p.RB0 + (ct.lo + o0) / p.CPR;
        q0 = (ct.lo + o0) % p.CPR;
    } else {
        const int own = p.LB * p.CPR, o0 = gi_start(own, warps - ct.ws, warp - ct.ws);
        n = gi_start(own, warps - ct.ws, warp - ct.ws + 1) - o0;
        rb0 = c * p.LB + o0 / p.CPR;
        q0 = o0 % p.CPR;
    }
}

// Chunk i of shared row block rb: whether a contributor's run starts there
// (the row block's first chunk, or the start of a CTA's share or of a
// warp's cut), that warp (global index) and its partial slot (0 if rb is
// its first row block).
__host__ __device__ __forceinline__ bool gi_contrib_at(const GiParams &p, int G, int warps, int rb, int i, int &gw,
                                                       int &slot)
{
    const int u = (rb - p.RB0) * p.CPR + i, cc = gi_owner(p.RL, G, u);
    const GiCta t = gi_cta(p, G, cc, warps);
    const int o = u - t.lo, wi = gi_owner(t.L, t.ws, o), s0 = gi_start(t.L, t.ws, wi);
    gw = cc * warps + wi;
    slot = p.RB0 + (t.lo + s0) / p.CPR == rb ? 0 : 1;
    return i == 0 || o == s0;
}

// The outputs of 16-row block n0 / 16 for every token (q = 16 m + r, row
// n0 + r): value(q) is the integer path's y in binary64.  The exactness
// guard (wq_imma.cuh) vouches for it or the warp recomputes that output in
// binary64 from x and the packed codes.  All 32 lanes call it together.
template <int BITS, class Value>
__device__ __forceinline__ void gi_emit(const GiParams &p, int n0, const int *s_e, const unsigned long long *s_res,
                                        Value value, int lane)
{
    const int M = p.M, N = p.N;
    const float wmax4 = BITS == 4 ? __uint_as_float(__ldg(p.wmax)) : 0.f;
    for (int q0 = 0; q0 < 16 * M; q0 += 32) {
        const int q = q0 + lane, r = q & 15, m = q >> 4;
        bool redo = false;
        if (q < 16 * M) {
            const double v = value(q);
            const double wmax =
                BITS == 8 ? 128.0 * (double)bf16_bits_to_float(p.scales[n0 + r]) : (double)wmax4;
            redo = !exact_enough(v, wmax * residual_bound(s_res[m], s_e[m]));
            if (!redo)
                p.y[(size_t)m * N + n0 + r] = __bfloat16_as_ushort(__double2bfloat16(v));
        }
        for (uint32_t mask = __ballot_sync(0xffffffffu, redo); mask; mask &= mask - 1) {
            const int src = __ffs(mask) - 1, qq = q0 + src, rr = qq & 15, mm = qq >> 4;
            double v = packed_row_dot<BITS>(p.wq, p.scales, p.zeros, p.K, p.KB, n0 + rr, p.x + (size_t)mm * p.K, lane);
            if constexpr (BITS == 8)
                v *= (double)bf16_bits_to_float(p.scales[n0 + rr]);
            if (lane == src)
                p.y[(size_t)mm * N + n0 + rr] = __bfloat16_as_ushort(__double2bfloat16(v));
        }
    }
}

// One segment's output, its accumulators in red ([16 rows][NR]; INT8 int32
// digit sums D_i, INT4 fp32 group-scaled sums A_i): y of the 16 x M outputs.
template <int BITS, int NR>
__device__ __forceinline__ void gi_write_y(const GiParams &p, int rb, const uint32_t *red, const int *s_e,
                                           const unsigned long long *s_res, int lane)
{
    const int n0 = 16 * rb;
    gi_emit<BITS>(
        p, n0, s_e, s_res,
        [&](int q) -> double {
            const int r = q & 15, m = q >> 4;
            if constexpr (BITS == 8) {
                const int32_t *d = reinterpret_cast<const int32_t *>(red) + r * NR + 3 * m;
                return ((double)d[2] * 65536.0 + (double)d[1] * 256.0 + (double)d[0]) *
                       ((double)bf16_bits_to_float(p.scales[n0 + r]) * pow2_of(-s_e[m]));
            } else {
                const float *a = reinterpret_cast<const float *>(red) + r * NR + 3 * m;
                return ((double)a[2] * 65536.0 + (double)a[1] * 256.0 + (double)a[0]) * pow2_of(-s_e[m]);
            }
        },
        lane);
}

// A partial segment of shared row block rb ended: the warp's partial into
// its slot, then its ticket (acquire-release), returned.
template <int BITS, int NR>
__device__ __forceinline__ uint32_t gi_shared_partial(const GiParams &p, int rb, int slot, int w, const uint32_t *red,
                                                      const int *s_e, int lane)
{
    const int M = p.M;
    __syncwarp();
    uint32_t *mine = p.part + ((size_t)w * 2 + slot) * 16 * NR;
    if constexpr (BITS == 8) {
        for (int i = lane; i < 16 * NR; i += 32)
            mine[i] = red[i];
    } else {
        for (int q = lane; q < 16 * M; q += 32) {
            const int r = q & 15, m = q >> 4;
            const float *a = reinterpret_cast<const float *>(red) + r * NR + 3 * m;
            const double v = ((double)a[2] * 65536.0 + (double)a[1] * 256.0 + (double)a[0]) * pow2_of(-s_e[m]);
            mine[r * NR + m] = __float_as_uint((float)v);
        }
    }
    __syncwarp();
    uint32_t ticket = 0;
    if (lane == 0)
        ticket = ticket_take_acq_rel(&p.cnt[rb]);
    return __shfl_sync(0xffffffffu, ticket, 0);
}

// After the warp's last chunk, for each shared row block it took a ticket
// of: the contributors are listed (one lane per chunk of the row block
// marks where a contributor's run starts: the row block's first chunk, a
// CTA's share or a warp's run), and the last contributor sums their
// partials in order (up to four loaded per round trip to L2) and writes y.
// Its ticket's acquire (taken earlier in program order) orders the reads.
// list: this warp's scratch of at least CPR words (partial offsets).
template <int BITS, int NT, int WARPS>
__device__ __forceinline__ void gi_shared_fixup(const GiParams &p, int rb, uint32_t ticket, int G, const int *s_e,
                                                const unsigned long long *s_res, uint32_t *list, int lane)
{
    constexpr int NR = 8 * NT;
    const int n0 = 16 * rb, CPR = p.CPR;
    int nc = 0;
    for (int base = 0; base < CPR; base += 32) {
        const int i = base + lane;
        bool start = false;
        uint32_t off = 0;
        if (i < CPR) {
            int gw, sl;
            start = gi_contrib_at(p, G, WARPS, rb, i, gw, sl);
            off = ((uint32_t)gw * 2 + sl) * 16 * NR;
        }
        const uint32_t mask = __ballot_sync(0xffffffffu, start);
        if (start)
            list[nc + __popc(mask & ((1u << lane) - 1u))] = off;
        nc += __popc(mask);
    }
    __syncwarp();
    if (ticket != (uint32_t)(nc - 1))
        return;
    gi_emit<BITS>(
        p, n0, s_e, s_res,
        [&](int q) -> double {
            const int r = q & 15, m = q >> 4;
            if constexpr (BITS == 8) {
                int32_t t0 = 0, t1 = 0, t2 = 0;
                for (int k0 = 0; k0 < nc; k0 += 4) {
                    int32_t v[4][3];
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        v[u][0] = v[u][1] = v[u][2] = 0;
                        if (k0 + u < nc) {
                            const int32_t *src =
                                reinterpret_cast<const int32_t *>(p.part + list[k0 + u]) + r * NR + 3 * m;
                            v[u][0] = __ldcg(src);
                            v[u][1] = __ldcg(src + 1);
                            v[u][2] = __ldcg(src + 2);
                        }
                    }
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        t0 += v[u][0];
                        t1 += v[u][1];
                        t2 += v[u][2];
                    }
                }
                return ((double)t2 * 65536.0 + (double)t1 * 256.0 + (double)t0) *
                       ((double)bf16_bits_to_float(p.scales[n0 + r]) * pow2_of(-s_e[m]));
            } else {
                float tot = 0.f;
                for (int k0 = 0; k0 < nc; k0 += 4) {
                    float v[4];
#pragma unroll
                    for (int u = 0; u < 4; ++u)
                        v[u] = k0 + u < nc
                                   ? __ldcg(reinterpret_cast<const float *>(p.part + list[k0 + u]) + r * NR + m)
                                   : 0.f;
#pragma unroll
                    for (int u = 0; u < 4; ++u)
                        if (k0 + u < nc)
                            tot += v[u];
                }
                return (double)tot;
            }
        },
        lane);
    __syncwarp();
    if (lane == 0)
        atomicExch(&p.cnt[rb], 0u); // ready for the next call
}

// After every warp of the CTA has streamed its share: the CTA's own row
// blocks that were split between its warps, summed from the stash in warp
// order (INT8: exact integers; INT4: each contributor's value in binary64,
// summed in binary64) and written to y.
template <int BITS, int NT, int WARPS>
__device__ __forceinline__ void gi_local_out(const GiParams &p, const GiCta &ct, int c, const uint32_t *stash,
                                             const int *s_e, const unsigned long long *s_res, int warp, int lane)
{
    constexpr int NR = 8 * NT;
    const int CPR = p.CPR;
    const int own = p.LB * CPR, wo = WARPS - ct.ws; // own chunks and the warps that take them
    for (int j = warp; j < p.LB; j += WARPS) {
        const int wf = ct.ws + gi_owner(own, wo, j * CPR), wl = ct.ws + gi_owner(own, wo, j * CPR + CPR - 1);
        if (wf == wl)
            continue; // one warp had it whole and wrote y
        const int n0 = 16 * (c * p.LB + j);
        gi_emit<BITS>(
            p, n0, s_e, s_res,
            [&](int q) -> double {
                const int r = q & 15, m = q >> 4;
                int32_t t0 = 0, t1 = 0, t2 = 0;
                double v = 0.0;
                for (int wi = wf; wi <= wl; ++wi) {
                    const int sl = gi_start(own, wo, wi - ct.ws) / CPR == j ? 0 : 1; // j: the warp's first row block?
                    const uint32_t *a = stash + ((size_t)wi * 2 + sl) * 16 * NR + r * NR + 3 * m;
                    if constexpr (BITS == 8) {
                        t0 += (int32_t)a[0];
                        t1 += (int32_t)a[1];
                        t2 += (int32_t)a[2];
                    } else {
                        v += (double)__uint_as_float(a[2]) * 65536.0 + (double)__uint_as_float(a[1]) * 256.0 +
                             (double)__uint_as_float(a[0]);
                    }
                }
                if constexpr (BITS == 8)
                    return ((double)t2 * 65536.0 + (double)t1 * 256.0 + (double)t0) *
                           ((double)bf16_bits_to_float(p.scales[n0 + r]) * pow2_of(-s_e[m]));
                else
                    return v * pow2_of(-s_e[m]);
            },
            lane);
    }
}

// WARPS = 16: one CTA per SM (the digit rows made once per SM); WARPS = 8:
// two per SM.  Either way 128 registers per thread and 16 warps per SM.
template <int BITS, int NT, int WARPS>
__global__ void __launch_bounds__(WARPS * 32, 16 / WARPS) gemv_i8_kernel(const GiParams p)
{
    constexpr int NR = 8 * NT;
    constexpr int D = GiCfg<BITS>::D;
    constexpr int WV = BITS == 8 ? 4 : 2; // 16-byte weight loads per lane and item
    // dynamic: digit rows [3M][S], (INT4) digit sums [KB][NR], then the
    // stash [WARPS][2][16 rows][NR] of partial sums of the CTA's own row blocks
    extern __shared__ __align__(16) uint8_t sd[];
    __shared__ uint32_t s_amax[kGiMaxM];
    __shared__ int s_e[kGiMaxM];
    __shared__ unsigned long long s_res[kGiMaxM]; // residual bound per token row (units of 2^-24)

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
    const int G = gridDim.x, c = blockIdx.x;
    const int w = c * WARPS + warp;
    const int KB = p.KB, M = p.M;
    const int S = gi_row_stride<BITS>(p.K);
    int32_t *s_dsum = reinterpret_cast<int32_t *>(sd + 3 * M * S);
    uint32_t *stash = reinterpret_cast<uint32_t *>(sd + 3 * M * S + (BITS == 4 ? KB * NR * 4 : 0));
    uint32_t *st0 = stash + (size_t)warp * 2 * 16 * NR, *st1 = st0 + 16 * NR;
    const GiCta ct = gi_cta(p, G, c, WARPS);
    const bool shared_warp = warp < ct.ws;
    int rb0, q0, n; // the warp's run: n chunks from chunk q0 of row block rb0
    gi_warp_run(p, ct, c, warp, WARPS, rb0, q0, n);

    // ---------------- weights of the first chunk (before the launch wait) ----------------
    // The warp's work is n consecutive chunks from (rb0, q0): chunk (rb, q) =
    // k-blocks D q .. D q + D - 1 (those below KB) of 16-row block rb.  Ring slot s holds
    // k-block D q + s of a chunk: consuming a slot is followed by loading
    // the same slot of the next chunk, so D k-blocks stay in flight.
    // Loader state: the next chunk to load is (lrb, lq); lw points at its
    // first k-block (INT8: the 16-row block's 2 KB; INT4: this lane's 16
    // bytes of the first tile), ls / lz at its INT4 scales and zero points.
    // Consecutive k-blocks of one 16-row block are 16 KB (INT8) / 8 KB
    // (INT4) apart.
    constexpr int kWStep = BITS == 8 ? 16384 : 8192;
    const int CPR = p.CPR;
    uint4 wb[D][WV];
    uint32_t sz[D][2]; // INT4: bf16 scales of rows g, g+8 | their zero-point bytes
    const int oa = (g << 7) + ((t ^ g) << 4), ob = (g << 7) + (((t + 4) ^ g) << 4); // INT8 chunks t, t+4
    int lrb = rb0, lq = q0;
    const uint8_t *lw = nullptr;
    const uint16_t *ls = nullptr;
    const uint8_t *lz = nullptr;
    auto seek = [&]() { // pointers of chunk (lrb, lq)
        const size_t blk = (size_t)(lrb >> 3) * KB + D * lq;
        const int j = lrb & 7;
        if constexpr (BITS == 8) {
            lw = p.wq + (blk << 14) + (j << 11);
        } else {
            lw = p.wq + ((blk * 8 + j) << 10) + 16 * lane;
            ls = p.scales + blk * kPanelRows + 16 * j + g;
            lz = p.zeros + blk * 64 + 8 * j + (g >> 1);
        }
    };
    auto load_slot = [&](int s, uint4 (&v)[WV], uint32_t (&e)[2]) {
        const uint8_t *b = lw + s * kWStep;
        if constexpr (BITS == 8) {
            v[0] = ldg_stream(b + oa);        // row g,     chunk t
            v[1] = ldg_stream(b + 1024 + oa); // row g + 8, chunk t
            v[2] = ldg_stream(b + ob);        // row g,     chunk t + 4
            v[3] = ldg_stream(b + 1024 + ob); // row g + 8, chunk t + 4
        } else {
            v[0] = ldg_stream(b);
            v[1] = ldg_stream(b + 512);
            const uint16_t *sp = ls + s * kPanelRows;
            const uint8_t *zp = lz + s * 64;
            e[0] = (uint32_t)__ldg(sp) | ((uint32_t)__ldg(sp + 8) << 16);
            e[1] = (uint32_t)__ldg(zp) | ((uint32_t)__ldg(zp + 4) << 8);
        }
    };
    auto next_chunk = [&]() {
        if (++lq == CPR) {
            lq = 0;
            ++lrb;
        }
        seek();
    };
    seek();
    const int rb_first = lrb;
    if (n > 0) {
#pragma unroll
        for (int s = 0; s < D; ++s)
            if (D * lq + s < KB)
                load_slot(s, wb[s], sz[s]);
        next_chunk();
    }

    // ---------------- activations: this CTA's digit rows ----------------
    if (threadIdx.x < kGiMaxM) {
        s_amax[threadIdx.x] = 0u;
        s_res[threadIdx.x] = 0ull;
    }
    __syncthreads();
    // The next kernel on the stream may launch now: its CTAs take the SMs
    // this grid leaves and prefetch their weights while its last CTAs
    // finish; whatever it shares with this grid waits behind its own launch
    // wait.  (Every CTA of this grid is resident by then: one wave.)
    pdl_launch_dependents();
    pdl_wait(); // x, y and the workspace may come from / be in use by the preceding kernel
    gi_digits<BITS, NR, WARPS * 32>(p, sd, s_dsum, s_amax, s_e, s_res);

    // ---------------- stream the warp's chunks ----------------
    int32_t acc_i[NT][4];
    float acc_f[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int r = 0; r < 4; ++r) {
            acc_i[nt][r] = 0;
            acc_f[nt][r] = 0.f;
        }
    // this lane's digit rows: INT8 bytes 16t and 16(t+4) of a block, INT4 bytes 32t .. 32t+31
    const uint8_t *xrow[NT];
    bool xon[NT];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
        xon[nt] = 8 * nt + g < 3 * M;
        xrow[nt] = sd + (xon[nt] ? (8 * nt + g) * S : 0) + (BITS == 8 ? 16 * t : 32 * t);
    }
    const int zsh = 4 * (g & 1);

    // k-block xo (byte offset 128 * kb in a digit row) of ring slot s
    auto consume = [&](int s, int xo) {
        if constexpr (BITS == 8) {
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                uint4 d0 = make_uint4(0, 0, 0, 0), d1 = d0;
                if (xon[nt]) {
                    d0 = *reinterpret_cast<const uint4 *>(xrow[nt] + xo);
                    d1 = *reinterpret_cast<const uint4 *>(xrow[nt] + xo + 64);
                }
                const uint4 *v = wb[s];
                imma_16832(acc_i[nt], v[0].x, v[1].x, v[0].y, v[1].y, d0.x, d0.y);
                imma_16832(acc_i[nt], v[0].z, v[1].z, v[0].w, v[1].w, d0.z, d0.w);
                imma_16832(acc_i[nt], v[2].x, v[3].x, v[2].y, v[3].y, d1.x, d1.y);
                imma_16832(acc_i[nt], v[2].z, v[3].z, v[2].w, v[3].w, d1.z, d1.w);
            }
        } else {
            constexpr uint32_t lo4 = 0x0F0F0F0Fu;
            uint32_t a[2][8]; // per tile: lo/hi of words x, y, z, w
#pragma unroll
            for (int tau = 0; tau < 2; ++tau) {
                const uint4 &v = wb[s][tau];
                a[tau][0] = v.x & lo4;
                a[tau][1] = (v.x >> 4) & lo4;
                a[tau][2] = v.y & lo4;
                a[tau][3] = (v.y >> 4) & lo4;
                a[tau][4] = v.z & lo4;
                a[tau][5] = (v.z >> 4) & lo4;
                a[tau][6] = v.w & lo4;
                a[tau][7] = (v.w >> 4) & lo4;
            }
            const float s_lo = __uint_as_float(sz[s][0] << 16), s_hi = __uint_as_float(sz[s][0] & 0xFFFF0000u);
            const int z_lo = (int)((sz[s][1] >> zsh) & 0xFu), z_hi = (int)((sz[s][1] >> (8 + zsh)) & 0xFu);
            const int32_t *dsum = s_dsum + (xo >> 7) * NR + 2 * t;
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                uint4 d0 = make_uint4(0, 0, 0, 0), d1 = d0;
                if (xon[nt]) {
                    d0 = *reinterpret_cast<const uint4 *>(xrow[nt] + xo);
                    d1 = *reinterpret_cast<const uint4 *>(xrow[nt] + xo + 16);
                }
                int32_t ci[4] = {0, 0, 0, 0};
                imma_16832(ci, a[0][0], a[0][2], a[0][1], a[0][3], d0.x, d0.y);
                imma_16832(ci, a[0][4], a[0][6], a[0][5], a[0][7], d0.z, d0.w);
                imma_16832(ci, a[1][0], a[1][2], a[1][1], a[1][3], d1.x, d1.y);
                imma_16832(ci, a[1][4], a[1][6], a[1][5], a[1][7], d1.z, d1.w);
                int2 ds = make_int2(0, 0);
                if (8 * nt + 2 * t < 3 * M)
                    ds = *reinterpret_cast<const int2 *>(dsum + 8 * nt);
                acc_f[nt][0] = fmaf(s_lo, (float)(ci[0] - z_lo * ds.x), acc_f[nt][0]);
                acc_f[nt][1] = fmaf(s_lo, (float)(ci[1] - z_lo * ds.y), acc_f[nt][1]);
                acc_f[nt][2] = fmaf(s_hi, (float)(ci[2] - z_hi * ds.x), acc_f[nt][2]);
                acc_f[nt][3] = fmaf(s_hi, (float)(ci[3] - z_hi * ds.y), acc_f[nt][3]);
            }
        }
    };

    int crb = rb0, cq = q0; // the chunk being consumed
    int npend = 0, pend_rb0 = 0, pend_rb1 = 0; // shared row blocks with a ticket taken
    uint32_t pend_t0 = 0, pend_t1 = 0;
    bool seg_whole = cq == 0; // the current segment started at the row block's first chunk
    for (int ch = 0; ch < n; ++ch) {
        const int kb0 = D * cq, xo = kb0 * 128;
        const bool more = ch + 1 < n; // the loader points at chunk ch + 1
        if (kb0 + D <= KB && more && D * lq + D <= KB) {
#pragma unroll
            for (int s = 0; s < D; ++s) { // common case: one straight block
                consume(s, xo + 128 * s);
                load_slot(s, wb[s], sz[s]);
            }
        } else {
#pragma unroll
            for (int s = 0; s < D; ++s) {
                if (kb0 + s < KB)
                    consume(s, xo + 128 * s);
                if (more && D * lq + s < KB)
                    load_slot(s, wb[s], sz[s]);
            }
        }
        if (more)
            next_chunk();
        if (cq == CPR - 1 || !more) { // end of a segment: the row block's last chunk or the warp's last
            const bool whole = seg_whole && cq == CPR - 1;
            // an own row block's partial stays in the stash (slot 0: the
            // warp's first row block, 1: its last); everything else passes
            // through slot 1, free until the warp's last segment
            uint32_t *red = (!shared_warp && !whole && crb == rb_first) ? st0 : st1;
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                const int col = 8 * nt + 2 * t;
                if constexpr (BITS == 8) {
                    red[g * NR + col] = (uint32_t)acc_i[nt][0];
                    red[g * NR + col + 1] = (uint32_t)acc_i[nt][1];
                    red[(g + 8) * NR + col] = (uint32_t)acc_i[nt][2];
                    red[(g + 8) * NR + col + 1] = (uint32_t)acc_i[nt][3];
                } else {
                    red[g * NR + col] = __float_as_uint(acc_f[nt][0]);
                    red[g * NR + col + 1] = __float_as_uint(acc_f[nt][1]);
                    red[(g + 8) * NR + col] = __float_as_uint(acc_f[nt][2]);
                    red[(g + 8) * NR + col + 1] = __float_as_uint(acc_f[nt][3]);
                }
#pragma unroll
                for (int r = 0; r < 4; ++r) {
                    acc_i[nt][r] = 0;
                    acc_f[nt][r] = 0.f;
                }
            }
            if (shared_warp && !whole) { // at most two: the first and the last row block of the run
                const uint32_t tk = gi_shared_partial<BITS, NR>(p, crb, crb == rb_first ? 0 : 1, w, red, s_e, lane);
                if (npend == 0) {
                    pend_rb0 = crb;
                    pend_t0 = tk;
                } else {
                    pend_rb1 = crb;
                    pend_t1 = tk;
                }
                ++npend;
            } else if (whole) {
                __syncwarp();
                gi_write_y<BITS, NR>(p, crb, red, s_e, s_res, lane);
                __syncwarp(); // red is rewritten by the next segment
            }
            ++crb;
            cq = 0;
            seg_whole = true;
        } else {
            ++cq;
        }
    }
    if (npend > 0)
        gi_shared_fixup<BITS, NT, WARPS>(p, pend_rb0, pend_t0, G, s_e, s_res, st0, lane);
    if (npend > 1)
        gi_shared_fixup<BITS, NT, WARPS>(p, pend_rb1, pend_t1, G, s_e, s_res, st0, lane);
    __syncthreads(); // every warp's stash is complete
    gi_local_out<BITS, NT, WARPS>(p, ct, c, stash, s_e, s_res, warp, lane);
}

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------
int gi_ntiles(int M) { return M <= 2 ? 1 : M <= 5 ? 2 : 3; }

// Dynamic shared memory of a CTA of `warps` warps: digit rows, INT4 digit
// sums, the stash of partial sums (2 x 16 x NR words per warp).
static size_t gi_smem_bytes_w(int bits, int M, int K, int warps)
{
    const size_t KB = (size_t)(K + kBlockK - 1) / kBlockK;
    const size_t NR = (size_t)8 * gi_ntiles(M);
    const size_t rows = (size_t)3 * M * (bits == 8 ? gi_row_stride<8>(K) : gi_row_stride<4>(K));
    return rows + (bits == 4 ? KB * NR * sizeof(int32_t) : 0) + (size_t)warps * 2 * 16 * NR * sizeof(uint32_t);
}

size_t gi_smem_bytes(int bits, int M, int K) { return gi_smem_bytes_w(bits, M, K, 16); }

bool gi_fits(int bits, int M, int K)
{
    return M >= 1 && M <= kGiMaxM && K >= 1 && K <= kI8MaxK && gi_smem_bytes(bits, M, K) <= kGiMaxSmem;
}

size_t ws_bytes_gemv_i8(int M, int K, int N)
{
    if (M < 1 || M > kGiMaxM || K < 1 || K > kI8MaxK)
        return 0;
    const size_t NR = 8 * gi_ntiles(M);
    return ws_counter_bytes() + (size_t)kGiMaxWarps * 2 * 16 * NR * 4;
}

// The work split of a grid of G CTAs of `warps` warps: chunks per row block,
// own row blocks per CTA, the first shared row block, shared chunks.  False
// when the cuts would leave 32-bit arithmetic.
static bool gi_plan(GiParams &p, int bits, int K, int N, int G, int warps)
{
    const int D = bits == 8 ? GiCfg<8>::D : GiCfg<4>::D;
    const int NRB = N / 16;
    p.KB = (K + kBlockK - 1) / kBlockK;
    p.CPR = (p.KB + D - 1) / D;
    p.LB = NRB / G;
    p.RB0 = G * p.LB;
    p.RL = (NRB - p.RB0) * p.CPR;
    return (long long)NRB * p.CPR * warps < (1LL << 31) && (long long)p.RL * G < (1LL << 31);
}

template <int BITS, int NT, int WARPS>
static cudaError_t launch_gi_t(const LinearArgs &a, void *ws, int sm_count, cudaStream_t st)
{
    const int smem = (int)gi_smem_bytes_w(BITS, a.M, a.K, WARPS);
    int occ = 1;
    {
        const cudaError_t e =
            kernel_setup((const void *)gemv_i8_kernel<BITS, NT, WARPS>, kGiMaxSmem, WARPS * 32, smem, &occ);
        if (e != cudaSuccess)
            return e;
    }
    const int per_sm = occ < 16 / WARPS ? occ : 16 / WARPS;
    const Shape sh{a.bits, a.K, a.N, a.group};
    GiParams p;
    p.x = a.x;
    p.M = a.M;
    p.K = a.K;
    p.N = a.N;
    p.KB = sh.kblocks();
    p.CPR = (p.KB + GiCfg<BITS>::D - 1) / GiCfg<BITS>::D;
    const int I = (a.N / 16) * p.CPR;
    p.wq = (const uint8_t *)a.wq;
    p.scales = (const uint16_t *)a.scales;
    p.zeros = (const uint8_t *)a.zeros;
    p.y = a.y;
    p.cnt = (uint32_t *)ws;
    p.part = (uint32_t *)((uint8_t *)ws + ws_counter_bytes());
    p.wmax = trailer_wmax(a.wq, sh);
    int G = per_sm * sm_count;
    if (G * WARPS > kGiMaxWarps)
        G = kGiMaxWarps / WARPS;
    const int want = (I + 2 * WARPS - 1) / (2 * WARPS); // at least ~2 chunks per warp
    if (G > want)
        G = want;
    if (G < 1)
        G = 1;
    if (!gi_plan(p, BITS, a.K, a.N, G, WARPS))
        return cudaErrorInvalidValue; // beyond the kernel's 32-bit stream-K cuts
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cfg.stream = st;
    cfg.gridDim = dim3(G);
    cfg.blockDim = dim3(WARPS * 32);
    cfg.dynamicSmemBytes = smem;
    return cudaLaunchKernelEx(&cfg, gemv_i8_kernel<BITS, NT, WARPS>, p);
}

template <int BITS, int NT>
static cudaError_t launch_gi_w(const LinearArgs &a, int split, void *ws, int sm_count, cudaStream_t st)
{
    return split == 2 ? launch_gi_t<BITS, NT, 8>(a, ws, sm_count, st) : launch_gi_t<BITS, NT, 16>(a, ws, sm_count, st);
}

cudaError_t launch_gemv_i8(const LinearArgs &a, int split, void *ws, int sm_count, cudaStream_t st)
{
    const int nt = gi_ntiles(a.M);
    if (a.bits == 8) {
        switch (nt) {
        case 1: return launch_gi_w<8, 1>(a, split, ws, sm_count, st);
        case 2: return launch_gi_w<8, 2>(a, split, ws, sm_count, st);
        default: return launch_gi_w<8, 3>(a, split, ws, sm_count, st);
        }
    }
    switch (nt) {
    case 1: return launch_gi_w<4, 1>(a, split, ws, sm_count, st);
    case 2: return launch_gi_w<4, 2>(a, split, ws, sm_count, st);
    default: return launch_gi_w<4, 3>(a, split, ws, sm_count, st);
    }
}

} // namespace wq

// ---------------------------------------------------------------------------
// Debug views of the integer GEMV's work split (host only; no GPU)
// ---------------------------------------------------------------------------
static int gi_debug_args(int bits, int K, int N, int G, int warps)
{
    if ((bits != 4 && bits != 8) || K < 1 || K > wq::kI8MaxK || N < 16 || N % 16 != 0 || G < 1 ||
        G > wq::kGiMaxCtas || (warps != 8 && warps != 16))
        return WQ_ERR_SHAPE;
    return WQ_OK;
}

extern "C" int wq_gemv_i8_plan(int bits, int K, int N, int G, int warps, int *meta, int *runs)
{
    if (meta == nullptr || runs == nullptr)
        return WQ_ERR_NULL;
    const int st = gi_debug_args(bits, K, N, G, warps);
    if (st != WQ_OK)
        return st;
    wq::GiParams p{};
    if (!wq::gi_plan(p, bits, K, N, G, warps))
        return WQ_ERR_SHAPE;
    meta[0] = p.CPR;
    meta[1] = p.LB;
    meta[2] = p.RB0;
    meta[3] = p.RL;
    for (int c = 0; c < G; ++c) {
        const wq::GiCta ct = wq::gi_cta(p, G, c, warps);
        for (int w = 0; w < warps; ++w) {
            int *r = runs + ((size_t)c * warps + w) * 4;
            wq::gi_warp_run(p, ct, c, w, warps, r[0], r[1], r[2]);
            r[3] = w < ct.ws ? 1 : 0;
        }
    }
    return WQ_OK;
}

extern "C" int wq_gemv_i8_contributors(int bits, int K, int N, int G, int warps, int rb, int *warp_ids, int *slots,
                                       int *count)
{
    if (warp_ids == nullptr || slots == nullptr || count == nullptr)
        return WQ_ERR_NULL;
    const int st = gi_debug_args(bits, K, N, G, warps);
    if (st != WQ_OK)
        return st;
    wq::GiParams p{};
    if (!wq::gi_plan(p, bits, K, N, G, warps) || rb < p.RB0 || rb >= N / 16)
        return WQ_ERR_SHAPE;
    int n = 0;
    for (int i = 0; i < p.CPR; ++i) {
        int gw, sl;
        if (wq::gi_contrib_at(p, G, warps, rb, i, gw, sl)) {
            warp_ids[n] = gw;
            slots[n] = sl;
            ++n;
        }
    }
    *count = n;
    return WQ_OK;
}
