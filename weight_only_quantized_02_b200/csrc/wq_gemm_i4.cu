// wq_gemm_i4.cu -- W4A16 (group 128, scale and zero point per group) on the
// integer tensor cores: tcgen05.mma kind::i8 on the exact integers q - z.
//
// y[m][n] = sum_g s[n][g] * sum_{k in g} (q[n][k] - z[n][g]) * x[m][k]
// (the WnA16 grouping of "Toward a Cleaner Quantization Stack in SGLang",
// Figure 4).  The activations become base-256 digits exactly as for W8A16
// (wq_imma.cuh: X = round(x * 2^e_m), |X| < 2^22, three digit rows per
// token).  A group is one 128-k block, so every unit (panel, k-block) is one
// MMA accumulation
//     D_g[n][3m + i] = sum_{k in g} (q - z)[n][k] d_i[m][k]     exact int32
// and the epilogue folds s[n][g] * (D0 + 256 D1 + 65536 D2) into fp32 totals
// per token, one group behind the MMA, then y = 2^-e_m * total in bf16.
//
// Warp roles (448 threads, one CTA per SM), stream-K over the units as in
// wq_gemm_i8.cu:
//   warp 0     producer: per unit bulk copies of the packed 8 KB block and
//              the group's 64 bytes of zero points into a deep ring (the
//              first stages before the programmatic-launch wait).  A stage
//              is released as soon as the expansion warps have read it, so
//              the ring turns over at the memory latency, not the MMA's.
//   warps 6-13 expansion, one 16-row block each: the packed tiles
//              (wq_layout.h) to signed bytes q - z in [-15, 15] (mask, byte
//              permute, SIMD byte subtract), stored into tensor memory with
//              tcgen05.st 16x256b, whose register layout the packed tile
//              already has; the MMA takes A from tensor memory (an M = 128
//              instruction then costs about a third of the shared-memory
//              form).  Within each 32-k step the columns hold k in a fixed
//              word order, which the digit blocks follow (wq_imma.cuh).
//   warp 1     allocates tensor memory; one thread issues four
//              tcgen05.mma kind::i8 (K = 32 each) per unit into one of kTB
//              per-unit accumulators.
//   warps 2-5  first the digit phase (wq_imma.cuh), then per unit: fold
//              s * D into fp32 totals (one thread per output channel), and
//              copy the digit block of unit i + SD into the slot unit i just
//              freed with 16-byte cp.async (outside the bulk-copy queue,
//              where it would wait behind weight blocks issued earlier),
//              counted on an mbarrier as each copy completes.  At a panel's
//              end write y, or store fp32 partials and take a ticket; the
//              last arriver sums every contributor's partial in CTA order
//              (deterministic) and writes y.
// Every wait is bounded (2 s); on a timeout the device error word is set and
// the CTA winds down.
#include <cstdint>

#include <cuda_bf16.h>

#include "wq_device.cuh"
#include "wq_imma.cuh"
#include "wq_internal.h"

namespace wq {

static __device__ int g_i4_error = 0;

struct I4Params {
    const uint16_t *x;
    int M, K, N, KB, U;
    const uint8_t *wq;      // packed blocks, 8 KB per unit
    const uint16_t *scales; // [P][KB][128] bf16
    const uint8_t *zeros;   // [P][KB][64]: row i at nibble i
    uint16_t *y;
    uint8_t *xd;            // [KB][NR][128] digit blocks
    float *part;            // [G][2 slots][NR/3 tokens][128 rows] fp32
    uint32_t *cnt;          // [panels][4] tickets
    uint32_t *grid;         // [2]: digit blocks written, CTAs exited
    unsigned long long *res; // [M] residual sums of the exactness guard
    const uint32_t *wmax;   // max |s (q - z)| over the weight (binary32 bits, packed trailer)
};

template <int NR>
struct I4Cfg {
    static constexpr int kBB = NR * 128;                // digit block
    static constexpr int kPB = 8192;                    // packed block
    static constexpr int kPStage = kPB + 64 + 256;      // packed block, zero points, scales
    static constexpr int kMaxM = NR / 3;
    static constexpr int kPStages = NR == 96 ? 8 : 10;
    static constexpr int kDStages = NR == 96 ? 10 : 12; // digit blocks, issued with the packed ones
    static constexpr int kAStages = 3;                  // expanded A tiles in tensor memory, 32 columns each
    static constexpr int kTB = 4;                       // per-unit accumulators in tensor memory
    static constexpr int kSQ = 8;                       // group scales handed from expansion to epilogue
    static constexpr int kA0 = kTB * NR;                // first A column
    static constexpr int kTmemCols = kA0 + 32 * kAStages <= 256 ? 256 : 512;
    static constexpr int kColGroup = NR < 48 ? NR : 48; // epilogue columns per pass (whole tokens)
    // [digit ring] (1024-byte aligned), the packed ring, the scale ring
    static constexpr int kRingBytes = kDStages * kBB + kPStages * kPStage + kSQ * 256;
    static_assert(NR % 16 == 0 && NR <= 96, "M <= 32 on this path");
    static_assert(kA0 % 32 == 0 && kA0 + 32 * kAStages <= kTmemCols, "tensor memory plan");
    static_assert(kSQ >= kTB + kAStages + 1, "scale slot reuse follows the accumulator ring");
};

constexpr int kI4Threads = 448;

template <int NR>
constexpr size_t i4_smem_bytes()
{
    using C = I4Cfg<NR>;
    // rings + barriers (pfull, pempty per packed stage; xfull, xempty per
    // digit stage; afull, aempty per A tile; accfull, accempty per
    // accumulator) + tensor-memory slot + row maxima / exponents + residual
    // bounds + the stream-K table
    return 1024 + (size_t)C::kRingBytes +
           (2 * C::kPStages + 2 * C::kDStages + 2 * C::kAStages + 2 * C::kTB) * 8 + 16 + 2 * kI8MaxM * 4 +
           kI8MaxM * 8 + (size_t)2 * (kI8MaxCtas + 1) * 4;
}

// Eight nibbles of one packed word (runs a, b of one row; positions
// [a0, a2, b0, b2, a1, a3, b1, b3]) -> runs a and b as bytes q - z.
__device__ __forceinline__ void expand_word(uint32_t v, uint32_t z4, uint32_t &ra, uint32_t &rb)
{
    const uint32_t lo = v & 0x0F0F0F0Fu, hi = (v >> 4) & 0x0F0F0F0Fu; // [a0 b0 a1 b1], [a2 b2 a3 b3]
    ra = __vsub4(__byte_perm(lo, hi, 0x6420u), z4);
    rb = __vsub4(__byte_perm(lo, hi, 0x7531u), z4);
}

// D(tmem) (+)= A(tmem) * B(smem descriptor); kind::i8.  With A in tensor
// memory an M = 128 instruction costs about a third of the shared-memory form.
__device__ __forceinline__ void umma_ts_i8(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                           uint32_t accumulate)
{
    asm volatile("{\n\t.reg .pred p;\n\t"
                 "setp.ne.b32 p, %4, 0;\n\t"
                 "tcgen05.mma.cta_group::1.kind::i8 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
                 "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
                 : "memory");
}

template <int NR>
// 14 warps: at most 4 per SM sub-partition, whose register file holds 16K
// registers, so at most 128 per thread.
__global__ void __maxnreg__(128) gemm_i4_kernel(const I4Params p)
{
    using C = I4Cfg<NR>;
    constexpr int SP = C::kPStages, SD = C::kDStages, SA = C::kAStages, TB = C::kTB;
    constexpr int TCOLS = C::kTmemCols;
    constexpr int CG = C::kColGroup;
    constexpr int MM = C::kMaxM;

    extern __shared__ uint8_t smem_raw[];
    uint8_t *ring = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *dring = ring;                       // [SD][NR x 128] digit blocks
    uint8_t *pring = dring + SD * C::kBB;        // [SP][packed 8 KB | zero points 64 B | scales 256 B]
    uint16_t *sring = reinterpret_cast<uint16_t *>(pring + SP * C::kPStage); // [kSQ][128] group scales
    uint64_t *pfull = reinterpret_cast<uint64_t *>(ring + C::kRingBytes);
    uint64_t *pempty = pfull + SP;
    uint64_t *xfull = pempty + SP;
    uint64_t *xempty = xfull + SD;
    uint64_t *afull = xempty + SD;
    uint64_t *aempty = afull + SA;
    uint64_t *accfull = aempty + SA;
    uint64_t *accempty = accfull + TB;
    uint32_t *s_tmem = reinterpret_cast<uint32_t *>(accempty + TB);
    uint32_t *s_amax = s_tmem + 4;                        // [kI8MaxM]
    int *s_e = reinterpret_cast<int *>(s_amax + kI8MaxM); // [kI8MaxM]
    double *s_rb = reinterpret_cast<double *>(s_e + kI8MaxM); // [kI8MaxM] residual bounds (8-byte aligned)
    int *s_start = reinterpret_cast<int *>(s_rb + kI8MaxM);    // [G + 1] stream-K cuts
    int *s_first = s_start + kI8MaxCtas + 1;                  // [G + 1] first panel of each range

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int G = gridDim.x, c = blockIdx.x;
    const long long U = p.U;
    const int KB = p.KB, M = p.M;
    const int u0 = sk_start(U, G, c), u1 = sk_start(U, G, c + 1);
    const int n = u1 - u0;

    if (threadIdx.x == 0) {
        for (int s = 0; s < SP; ++s) {
            mbar_init(&pfull[s], 1);
            mbar_init(&pempty[s], 8);
        }
        for (int s = 0; s < SD; ++s) {
            mbar_init(&xfull[s], 1);
            mbar_init(&xempty[s], 1);
        }
        for (int s = 0; s < SA; ++s) {
            mbar_init(&afull[s], 8);
            mbar_init(&aempty[s], 1);
        }
        for (int b = 0; b < TB; ++b) {
            mbar_init(&accfull[b], 1);
            mbar_init(&accempty[b], 4);
        }
        fence_mbar_init();
    }
    if (threadIdx.x < kI8MaxM)
        s_amax[threadIdx.x] = 0u;
    for (int i = threadIdx.x; i <= G; i += blockDim.x) {
        const int st = sk_start(U, G, i);
        s_start[i] = st;
        s_first[i] = st / KB;
    }
    if (warp == 1) {
        tmem_alloc(s_tmem, TCOLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *s_tmem;
    const SkTable sk{s_start, s_first};
    bool ok = true;

    if (warp == 0) {
        // ---------------- producer ----------------
        // per unit: the digit block (L2) just ahead of the packed block, zero
        // points and scales (HBM), so both arrive together; packed stages are
        // released by the expansion warps, digit stages by the MMA
        if (lane == 0) {
            const uint64_t pol_w = policy_evict_first(), pol_x = policy_evict_last();
            auto issue_p = [&](int i) {
                const int st = i % SP;
                const size_t u = (size_t)(u0 + i);
                uint8_t *dst = pring + st * C::kPStage;
                mbar_arrive_expect_tx(&pfull[st], C::kPStage);
                bulk_g2s(dst, p.wq + u * C::kPB, C::kPB, &pfull[st], pol_w);
                bulk_g2s(dst + C::kPB, p.zeros + u * 64, 64, &pfull[st], pol_w);
                bulk_g2s(dst + C::kPB + 64, p.scales + u * kPanelRows, 256, &pfull[st], pol_w);
            };
            int xkb = u0 % KB; // k-block of the next digit block issued (units in order), kept without dividing
            auto issue_x = [&](int i) {
                const int sd = i % SD;
                mbar_arrive_expect_tx(&xfull[sd], C::kBB);
                bulk_g2s(dring + sd * C::kBB, p.xd + (size_t)xkb * C::kBB, C::kBB, &xfull[sd], pol_x);
                xkb = xkb + 1 == KB ? 0 : xkb + 1;
            };
            const int pre = n < SP ? n : SP;
            for (int i = 0; i < pre; ++i) // weights never depend on the preceding kernel
                issue_p(i);
            // the preceding call (same workspace) has finished and reset the grid
            // counters; then wait until every CTA's share of the digit blocks is written
            pdl_wait();
            const uint64_t t0 = globaltimer_ns();
            while (ld_acquire_gpu(&p.grid[0]) < (uint32_t)G) {
                if (globaltimer_ns() - t0 > kWaitLimitNs) {
                    ok = false;
                    break;
                }
            }
            fence_proxy_async_global(); // the digit blocks are read by the bulk-copy (async) proxy
            for (int i = 0; i < pre && ok; ++i)
                issue_x(i);
            for (int i = pre; i < n && ok; ++i) {
                if (!mbar_wait(&pempty[i % SP], ((i / SP) - 1) & 1) ||
                    (i >= SD && !mbar_wait(&xempty[i % SD], ((i / SD) - 1) & 1))) {
                    ok = false;
                    break;
                }
                issue_x(i);
                issue_p(i);
            }
        }
        __syncwarp();
        pdl_wait();
        pdl_launch_dependents();
    } else if (warp == 1) {
        // ---------------- MMA issue ----------------
        if (lane == 0) {
            constexpr uint32_t idesc = umma_idesc_s8(NR);
            for (int i = 0; i < n; ++i) {
                const int sd = i % SD, sa = i % SA, b = i % TB;
                if (i >= TB && !mbar_wait(&accempty[b], ((i / TB) - 1) & 1)) {
                    ok = false;
                    break;
                }
                if (!mbar_wait(&afull[sa], (i / SA) & 1) || !mbar_wait(&xfull[sd], (i / SD) & 1)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t sb = smem_u32(dring + sd * C::kBB);
                const uint32_t d = tmem + (uint32_t)(b * NR);
                const uint32_t ta = tmem + (uint32_t)(C::kA0 + 32 * sa);
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) // A from tensor memory: 8 columns (32 k) per step
                    umma_ts_i8(d, ta + 8 * kk, smem_desc_sw128(sb + 32 * kk), idesc, kk > 0 ? 1u : 0u);
                umma_commit(&aempty[sa]);
                umma_commit(&xempty[sd]);
                umma_commit(&accfull[b]);
            }
        }
        __syncwarp();
        pdl_wait();
        pdl_launch_dependents();
    } else if (warp >= 6) {
        // ---------------- expansion: packed tiles -> q - z bytes in tensor memory ----------------
        // warp w may access tensor-memory lanes 32 (w % 4) .. +31: it expands
        // 16-row block j = 2 (w % 4) + h (h = 0 for warps 6-9, 1 for 10-13)
        const int q = warp & 3, h = warp >= 10 ? 1 : 0;
        const int j = 2 * q + h;
        const int g = lane >> 2;
        const int r0 = 16 * j + g, r1 = r0 + 8;
        const uint32_t tl = (uint32_t)(32 * q + 16 * h) << 16;
        for (int i = 0; i < n && ok; ++i) {
            const int st = i % SP, sa = i % SA;
            if (!mbar_wait_warp(&pfull[st], (i / SP) & 1)) {
                ok = false;
                break;
            }
            const uint8_t *pk = pring + st * C::kPStage;
            const uint8_t *z8 = pk + C::kPB;
            const uint4 w0 = *reinterpret_cast<const uint4 *>(pk + j * 1024 + lane * 16);
            const uint4 w1 = *reinterpret_cast<const uint4 *>(pk + j * 1024 + 512 + lane * 16);
            const uint32_t z0 = (z8[r0 >> 1] >> (4 * (r0 & 1))) & 0xFu;
            const uint32_t z1 = (z8[r1 >> 1] >> (4 * (r1 & 1))) & 0xFu;
            if ((lane & 3) == 0) { // the rows' group scales, for the epilogue of unit i
                const uint16_t *sc = reinterpret_cast<const uint16_t *>(z8 + 64);
                sring[(i % C::kSQ) * 128 + r0] = sc[r0];
                sring[(i % C::kSQ) * 128 + r1] = sc[r1];
            }
            // Expand before releasing the stage: the producer refills a
            // released stage at once, and a load still in flight could
            // otherwise return the next block's bytes.
            const uint32_t z40 = z0 * 0x01010101u, z41 = z1 * 0x01010101u;
            // tcgen05.st 16x256b.x4: column group 2 tt + half holds runs (a, b)
            // (half 0) or (c, d) (half 1) of tile tt: lane g / g+8, columns
            // 2t (first run) and 2t + 1 (second run), 4 k per column
            uint32_t r[16];
#pragma unroll
            for (int tt = 0; tt < 2; ++tt) {
                const uint4 &w = tt == 0 ? w0 : w1;
                expand_word(w.x, z40, r[8 * tt + 0], r[8 * tt + 1]); // row g,   runs a, b
                expand_word(w.y, z41, r[8 * tt + 2], r[8 * tt + 3]); // row g+8, runs a, b
                expand_word(w.z, z40, r[8 * tt + 4], r[8 * tt + 5]); // row g,   runs c, d
                expand_word(w.w, z41, r[8 * tt + 6], r[8 * tt + 7]); // row g+8, runs c, d
            }
            __syncwarp();
            if (lane == 0)
                mbar_arrive(&pempty[st]); // the packed stage is free for the next load
            if (i >= SA && !mbar_wait_warp(&aempty[sa], ((i / SA) - 1) & 1)) {
                ok = false;
                break;
            }
            tc_fence_after();
            tmem_st_16x256b_x4(tmem + tl + (uint32_t)(C::kA0 + 32 * sa), r);
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0)
                mbar_arrive(&afull[sa]);
        }
        pdl_launch_dependents();
    } else {
        pdl_wait(); // x, y and the workspace may come from / be in use by the preceding kernel
        const int et = threadIdx.x - 64; // 0..127
        const int quad = warp & 3;
        imma_digit_phase<NR, true>(p.x, M, p.K, KB, c, G, et, p.xd, s_amax, s_e, p.grid, p.res);
        ok = imma_residual_bounds(M, G, et, p.grid, p.res, s_e, s_rb) && ok;
        const double wmax = (double)__uint_as_float(__ldg(p.wmax));

        // ---------------- epilogue: one thread per output channel ----------------
        const int row = 32 * quad + lane;
        const uint32_t tq = (uint32_t)(32 * quad) << 16;
        float acc[MM];
#pragma unroll
        for (int m = 0; m < MM; ++m)
            acc[m] = 0.f;
        int pnl = u0 / KB, kb = u0 - pnl * KB; // panel and k-block of unit i, kept without dividing
        for (int i = 0; i < n && ok; ++i) {
            const int b = i % TB;
            if (!mbar_wait_warp(&accfull[b], (i / TB) & 1)) {
                ok = false;
                break;
            }
            tc_fence_after();
            // written by the expansion warps before this unit's MMA
            const float s = bf16_bits_to_float(sring[(i % C::kSQ) * 128 + row]);
#pragma unroll
            for (int c0 = 0; c0 < NR; c0 += CG) {
                if (c0 < 3 * M) {
                    int32_t v[CG];
#pragma unroll
                    for (int cc = 0; cc < CG; cc += 8) {
                        float f[8];
                        tmem_ld_32x32b_x8(tmem + tq + (uint32_t)(b * NR + c0 + cc), f);
#pragma unroll
                        for (int e2 = 0; e2 < 8; ++e2)
                            v[cc + e2] = __float_as_int(f[e2]);
                    }
                    tmem_wait_ld();
#pragma unroll
                    for (int tk = 0; tk < CG / 3; ++tk) {
                        const int m = c0 / 3 + tk;
                        const float dvl =
                            fmaf((float)v[3 * tk + 2], 65536.f, fmaf((float)v[3 * tk + 1], 256.f, (float)v[3 * tk]));
                        if (m < MM)
                            acc[m] = fmaf(s, dvl, acc[m]);
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0)
                mbar_arrive(&accempty[b]);
            if (i == n - 1 || kb == KB - 1) {
                // panel pnl done: y when this CTA covered it whole, else partial + ticket
                do {
                    const int lo = max(u0, pnl * KB), hi = min(u1, (pnl + 1) * KB);
                    if (lo == pnl * KB && hi == (pnl + 1) * KB) {
#pragma unroll
                        for (int m = 0; m < MM; ++m)
                            if (m < M) // the same across the warp
                                imma_emit_rows<4>(p.x, p.wq, p.scales, p.zeros, p.y, p.K, KB, p.N,
                                                  pnl * kPanelRows + 32 * quad, m, (double)acc[m] * pow2_of(-s_e[m]),
                                                  wmax * s_rb[m], lane);
                        break;
                    }
                    const int slot = (pnl == sk.first[c]) ? 0 : 1;
                    float *mine = p.part + (size_t)(c * 2 + slot) * MM * 128 + row;
#pragma unroll
                    for (int m = 0; m < MM; ++m)
                        if (m < M)
                            mine[(size_t)m * 128] = acc[m];
                    __syncwarp();
                    uint32_t ticket = 0;
                    if (lane == 0)
                        ticket = ticket_take_acq_rel(&p.cnt[pnl * 4 + quad]);
                    ticket = __shfl_sync(0xffffffffu, ticket, 0);
                    const int cf = sk.owner(pnl * KB, G), cl = sk.owner((pnl + 1) * KB - 1, G);
                    if (ticket != (uint32_t)(cl - cf))
                        break;
                    __syncwarp(); // lane 0's acquire orders every lane's reads below
                    float tot[MM];
#pragma unroll
                    for (int m = 0; m < MM; ++m)
                        tot[m] = 0.f;
                    for (int cc = cf; cc <= cl; ++cc) { // contributors in CTA order: deterministic
                        const int sl = (pnl == sk.first[cc]) ? 0 : 1;
                        const float *src = p.part + (size_t)(cc * 2 + sl) * MM * 128 + row;
                        float v[MM];
#pragma unroll
                        for (int m = 0; m < MM; ++m)
                            v[m] = (m < M) ? __ldcg(src + (size_t)m * 128) : 0.f;
#pragma unroll
                        for (int m = 0; m < MM; ++m)
                            tot[m] += v[m];
                    }
#pragma unroll
                    for (int m = 0; m < MM; ++m)
                        if (m < M) // the same across the warp
                            imma_emit_rows<4>(p.x, p.wq, p.scales, p.zeros, p.y, p.K, KB, p.N,
                                              pnl * kPanelRows + 32 * quad, m, (double)tot[m] * pow2_of(-s_e[m]),
                                              wmax * s_rb[m], lane);
                    if (lane == 0)
                        atomicExch(&p.cnt[pnl * 4 + quad], 0u);
                } while (false);
#pragma unroll
                for (int m = 0; m < MM; ++m)
                    acc[m] = 0.f;
            }
            if (++kb == KB) {
                kb = 0;
                ++pnl;
            }
        }
        pdl_launch_dependents();
    }

    if (!ok)
        atomicExch(&g_i4_error, kErrTimeout);
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, TCOLS);
    }
    // the last CTA out resets the grid counters and the residual sums for the
    // next call (every CTA has read them before counting itself out)
    if (threadIdx.x == 0) {
        __threadfence();
        if (atomicAdd(&p.grid[1], 1u) == (uint32_t)(G - 1)) {
            for (int m = 0; m < M; ++m)
                p.res[m] = 0ull;
            atomicExch(&p.grid[0], 0u);
            atomicExch(&p.grid[1], 0u);
        }
    }
}

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------
size_t ws_bytes_gemm_i4(int M, int K, int N)
{
    if (M < 1 || M > kI4MaxM || K < 1)
        return 0;
    const int NR = i8_digit_rows(M);
    const size_t KB = (size_t)(K + kBlockK - 1) / kBlockK;
    return ws_counter_bytes() + KB * NR * 128 + (size_t)kI8MaxCtas * 2 * (NR / 3) * 128 * sizeof(float);
}

template <int NR>
static cudaError_t launch_i4_t(const LinearArgs &a, void *ws, int sm_count, cudaStream_t st)
{
    constexpr size_t smem = i4_smem_bytes<NR>();
    static_assert(smem <= 227 * 1024, "shared memory per CTA");
    {
        const cudaError_t e = kernel_setup((const void *)gemm_i4_kernel<NR>, smem, 0, 0, nullptr);
        if (e != cudaSuccess)
            return e;
    }
    const Shape sh{4, a.K, a.N, 128};
    I4Params p;
    p.x = a.x;
    p.M = a.M;
    p.K = a.K;
    p.N = a.N;
    p.KB = sh.kblocks();
    p.U = sh.panels() * p.KB;
    p.wq = (const uint8_t *)a.wq;
    p.scales = (const uint16_t *)a.scales;
    p.zeros = (const uint8_t *)a.zeros;
    p.y = a.y;
    p.cnt = (uint32_t *)ws;
    p.grid = p.cnt + ws_grid_counter();
    p.res = reinterpret_cast<unsigned long long *>(p.cnt + ws_res_counter());
    p.wmax = trailer_wmax(a.wq, sh);
    p.xd = (uint8_t *)ws + ws_counter_bytes();
    p.part = (float *)(p.xd + (size_t)p.KB * NR * 128);
    int G = sm_count < kI8MaxCtas ? sm_count : kI8MaxCtas;
    if (G > p.U)
        G = p.U;
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cfg.stream = st;
    cfg.gridDim = dim3(G);
    cfg.blockDim = dim3(kI4Threads);
    cfg.dynamicSmemBytes = smem;
    return cudaLaunchKernelEx(&cfg, gemm_i4_kernel<NR>, p);
}

cudaError_t launch_gemm_i4(const LinearArgs &a, void *ws, int sm_count, cudaStream_t st)
{
    switch (i8_digit_rows(a.M)) {
    case 16: return launch_i4_t<16>(a, ws, sm_count, st);
    case 32: return launch_i4_t<32>(a, ws, sm_count, st);
    case 48: return launch_i4_t<48>(a, ws, sm_count, st);
    case 96: return launch_i4_t<96>(a, ws, sm_count, st);
    default: return cudaErrorInvalidValue; // M <= kI4MaxM
    }
}

cudaError_t read_gemm_i4_error(int *code, cudaStream_t st)
{
    int host = 0, zero = 0;
    cudaError_t e = cudaMemcpyFromSymbolAsync(&host, g_i4_error, sizeof(int), 0, cudaMemcpyDeviceToHost, st);
    if (e != cudaSuccess)
        return e;
    e = cudaMemcpyToSymbolAsync(g_i4_error, &zero, sizeof(int), 0, cudaMemcpyHostToDevice, st);
    if (e != cudaSuccess)
        return e;
    e = cudaStreamSynchronize(st);
    *code = host;
    return e;
}

} // namespace wq
