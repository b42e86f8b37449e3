// wq_gemv_sk.cu -- stream-K GEMV for decode-sized M (<= 32), W8A16 / W4A16.
//
// The packed weights are one contiguous stream of (128-row panel, 128-k
// block) units.  Each persistent CTA takes an equal contiguous share of that
// stream (units [U*c/G, U*(c+1)/G)), so every SM moves the same number of
// bytes whatever N and K are; a producer warp pulls the share through a
// STAGES-deep ring of 1-D bulk copies (the TMA engine, no multicast), which
// keeps tens of KB in flight per SM without registers.  Eight consumer warps
// own the eight 16-row blocks of a panel: each reads its 512-byte tiles from
// shared memory -- already m16n8k16 A fragments (wq_layout.h) -- unpacks them
// in registers and runs mma.sync with the activations as the B operand (the
// GEMV row of the tileInfer README, Features table: dequantization in
// registers and 16-byte loads, here each lane's 16-byte shared-memory
// reads).  INT4 groups are scaled in fp32 after their 8 MMAs and
// INT8 rows once at the end, so weights are never rounded.
//
// A panel whose k-blocks are split between two or more CTAs is finished,
// 16 rows at a time, by the last warp to arrive for those rows (atomic
// ticket per (panel, 16-row block), never waited on): it sums the fp32
// partials of all contributors in CTA order, so the result is deterministic,
// and resets the ticket to zero.  Partials live in the workspace:
// [G CTAs][2 slots (first/last panel of the range)][128 rows][8*MT tokens].
#include <cstdint>
#include <mutex>

#include "wq_device.cuh"
#include "wq_internal.h"

namespace wq {

static __device__ int g_gemv_sk_error = 0;

struct GemvSkParams {
    const uint16_t *x;
    int M, K, N;
    const uint8_t *wq;
    const uint16_t *scales;
    const uint8_t *zeros;
    uint16_t *y;
    int KB, U; // k-blocks per panel, units = panels * KB
    float *part;
    uint32_t *cnt;
};

// Ring stage: packed weights of the unit, INT4 scales/zeros, and the unit's
// activation slice x[0..M)[128 k] (one 256-byte bulk copy per token row).
// The row stride makes a warp's activation reads conflict-free: INT4 lanes
// read 8 bytes at row g, column 4t (288 = 72 words: rows 8 banks apart);
// INT8 lanes read 16 bytes at row g, column 16t (272 = 68 words: the two
// rows of a quarter-warp 4 banks apart).
template <int BITS, int MT, int OCC>
struct SkCfg {
    static constexpr int kTPB = BITS == 4 ? 2 : 4;   // tiles per 16-row block per unit
    static constexpr int kRBB = kTPB * kTileBytes;   // bytes of one 16-row block per unit
    static constexpr int kPBB = 8 * kRBB;            // packed bytes per unit
    static constexpr int kSZB = BITS == 4 ? 512 : 0; // scales 256 + zeros 64, padded
    static constexpr int kSZTx = BITS == 4 ? 320 : 0;
    static constexpr int kXRow = BITS == 8 ? 272 : 288; // smem stride of one token row (256 B + pad)
    static constexpr int kXB = 8 * MT * kXRow;
    static constexpr int kStageBytes = kPBB + kSZB + kXB;
    // ring sized so OCC CTAs fit in an SM's 228 KB of shared memory
    static constexpr int kBudget = (220 * 1024) / OCC - 1024;
    static constexpr int kStagesRaw = kBudget / kStageBytes;
    static constexpr int kStages = kStagesRaw > 8 ? 8 : (kStagesRaw < 2 ? 2 : kStagesRaw);
};

constexpr int kSkConsumers = 8;
constexpr int kSkThreads = 32 * (1 + kSkConsumers);

// B fragments of mma.m16n8k16 from the staged activation slice: lane
// (g, t) takes x[8*mt + g][k .. k+4) (k relative to the unit's 128-k block);
// xs already points at row g, column 4t of the stage's x area.
template <int MT, int XROW>
__device__ __forceinline__ void x_frags(const uint8_t *xs, int k, uint2 (&xf)[MT])
{
#pragma unroll
    for (int mt = 0; mt < MT; ++mt)
        xf[mt] = *reinterpret_cast<const uint2 *>(xs + mt * 8 * XROW + 2 * k);
}

// bytes 0..3 of w (int8) -> two bf16x2: {q0, q1}, {q2, q3}; exact.
__device__ __forceinline__ void s8quad_bf16(uint32_t w, uint32_t &lo, uint32_t &hi)
{
    const uint32_t u = w ^ 0x80808080u;
    const uint32_t f0 = __byte_perm(u, 0x4B000000u, 0x7540u), f1 = __byte_perm(u, 0x4B000000u, 0x7541u);
    const uint32_t f2 = __byte_perm(u, 0x4B000000u, 0x7542u), f3 = __byte_perm(u, 0x4B000000u, 0x7543u);
    const uint64_t c = 0x4B0000804B000080ull; // {2^23 + 128, 2^23 + 128}
    uint64_t d01, d23;
    asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d01) : "l"(((uint64_t)f1 << 32) | f0), "l"(c));
    asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d23) : "l"(((uint64_t)f3 << 32) | f2), "l"(c));
    // |q| <= 128 has at most 8 significant bits: the fp32 value's upper half is its bf16
    lo = __byte_perm((uint32_t)d01, (uint32_t)(d01 >> 32), 0x7632u);
    hi = __byte_perm((uint32_t)d23, (uint32_t)(d23 >> 32), 0x7632u);
}

// One INT8 chunk pair of the stage: lane (g, t) holds k = kc .. kc+15 of
// rows g (wa) and g+8 (wb); step i = 0..3 is an m16n8k16 MMA whose k-slots
// 2t, 2t+1, 2t+8, 2t+9 take k = kc+4i .. kc+4i+3.  xv / xw: the same k of
// token row 8*mt + g (kc .. kc+7 and kc+8 .. kc+15).
template <int MT>
__device__ __forceinline__ void sk_int8_chunk(const uint4 &wa, const uint4 &wb, const uint4 (&xv)[MT],
                                              const uint4 (&xw)[MT], float (&acc)[MT][4])
{
    const uint32_t ra[4] = {wa.x, wa.y, wa.z, wa.w}, rb[4] = {wb.x, wb.y, wb.z, wb.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        uint32_t a0, a2, a1, a3;
        s8quad_bf16(ra[i], a0, a2);
        s8quad_bf16(rb[i], a1, a3);
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) {
            const uint4 &xx = i < 2 ? xv[mt] : xw[mt];
            const uint32_t b0 = (i & 1) ? xx.z : xx.x, b1 = (i & 1) ? xx.w : xx.y;
            mma_bf16_16816(acc[mt], a0, a1, a2, a3, b0, b1);
        }
    }
}

template <int MT, int XROW>
__device__ __forceinline__ void sk_int4_tile(const uint4 &w, const uint8_t *xs, int kt, uint32_t zlo, uint32_t zhi,
                                             float (&cg)[MT][4])
{
    uint32_t xr_[4], yr[4], zr[4], wr[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        xr_[i] = bf16x2_sub(nib_pair_bf16(w.x >> (4 * i)), zlo);
        yr[i] = bf16x2_sub(nib_pair_bf16(w.y >> (4 * i)), zhi);
        zr[i] = bf16x2_sub(nib_pair_bf16(w.z >> (4 * i)), zlo);
        wr[i] = bf16x2_sub(nib_pair_bf16(w.w >> (4 * i)), zhi);
    }
    uint2 xa[MT], xb[MT], xc[MT], xd[MT];
    x_frags<MT, XROW>(xs, kt, xa);
    x_frags<MT, XROW>(xs, kt + 16, xb);
    x_frags<MT, XROW>(xs, kt + 32, xc);
    x_frags<MT, XROW>(xs, kt + 48, xd);
#pragma unroll
    for (int mt = 0; mt < MT; ++mt) {
        mma_bf16_16816(cg[mt], xr_[0], yr[0], xr_[1], yr[1], xa[mt].x, xa[mt].y);
        mma_bf16_16816(cg[mt], xr_[2], yr[2], xr_[3], yr[3], xb[mt].x, xb[mt].y);
        mma_bf16_16816(cg[mt], zr[0], wr[0], zr[1], wr[1], xc[mt].x, xc[mt].y);
        mma_bf16_16816(cg[mt], zr[2], wr[2], zr[3], wr[3], xd[mt].x, xd[mt].y);
    }
}

// OCC = CTAs per SM the instance is built for (register bound and ring depth).
template <int BITS, int MT, int OCC>
__global__ void __launch_bounds__(kSkThreads, OCC) gemv_sk_kernel(const GemvSkParams p)
{
    using C = SkCfg<BITS, MT, OCC>;
    constexpr int STAGES = C::kStages;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *ring = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
    uint64_t *full = reinterpret_cast<uint64_t *>(ring + STAGES * C::kStageBytes);
    uint64_t *empty = full + STAGES;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int G = gridDim.x, c = blockIdx.x;
    const long long U = p.U;
    const int u0 = sk_start(U, G, c), u1 = sk_start(U, G, c + 1);
    const int n = u1 - u0;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kSkConsumers);
        }
        fence_mbar_init();
    }
    // token rows M..8*MT of every stage's x area stay zero (the B operand's padding)
    {
        const int pad_rows = 8 * MT - p.M;
        const int words = pad_rows * (C::kXRow / 4);
        for (int s = 0; s < STAGES; ++s) {
            uint32_t *xz = reinterpret_cast<uint32_t *>(ring + s * C::kStageBytes + C::kPBB + C::kSZB + p.M * C::kXRow);
            for (int i = threadIdx.x; i < words; i += blockDim.x)
                xz[i] = 0u;
        }
    }
    fence_proxy_async_smem();
    __syncthreads();
    bool ok = true;

    if (warp == 0) {
        if (lane == 0) {
            const uint64_t pol = policy_evict_first(), pol_x = policy_evict_last();
            auto xbytes_of = [&](int kb) { return min(2 * kBlockK, 2 * (p.K - kb * kBlockK)); };
            auto issue_weights = [&](int i, int st) {
                const size_t u = (size_t)(u0 + i);
                uint8_t *dst = ring + st * C::kStageBytes;
                mbar_arrive_expect_tx(&full[st], C::kPBB + C::kSZTx + p.M * xbytes_of((int)(u % p.KB)));
                bulk_g2s(dst, p.wq + u * C::kPBB, C::kPBB, &full[st], pol);
                if constexpr (BITS == 4) {
                    bulk_g2s(dst + C::kPBB, p.scales + u * kPanelRows, 256, &full[st], pol);
                    bulk_g2s(dst + C::kPBB + 256, p.zeros + u * 64, 64, &full[st], pol);
                }
            };
            auto issue_x = [&](int i, int st) {
                const int kb = (u0 + i) % p.KB;
                uint8_t *dst = ring + st * C::kStageBytes + C::kPBB + C::kSZB;
                for (int m = 0; m < p.M; ++m)
                    bulk_g2s(dst + m * C::kXRow, p.x + (size_t)m * p.K + (size_t)kb * kBlockK, xbytes_of(kb),
                             &full[st], pol_x);
            };
            // weights do not depend on the preceding kernel: start streaming them
            // before waiting for it; activations only after
            const int pre = n < STAGES ? n : STAGES;
            for (int i = 0; i < pre; ++i)
                issue_weights(i, i);
            pdl_wait();
            for (int i = 0; i < pre; ++i)
                issue_x(i, i);
            for (int i = pre; i < n; ++i) {
                const int st = i % STAGES, use = i / STAGES;
                if (!mbar_wait(&empty[st], (use - 1) & 1)) {
                    ok = false;
                    break;
                }
                issue_weights(i, st);
                issue_x(i, st);
            }
        } else {
            pdl_wait();
        }
        pdl_launch_dependents();
    } else {
        pdl_wait(); // the workspace and y may still be in use by the preceding kernel
        const int j = warp - 1; // 16-row block of the panel
        const int g = lane >> 2, t = lane & 3;
        const int KB = p.KB;
        float acc[MT][4];
#pragma unroll
        for (int mt = 0; mt < MT; ++mt)
            acc[mt][0] = acc[mt][1] = acc[mt][2] = acc[mt][3] = 0.f;
        // activations of this lane: row g, column 4t (INT4) or 16t (INT8)
        const int xoff = C::kPBB + C::kSZB + g * C::kXRow + (BITS == 8 ? 32 : 8) * t;

        // write this warp's rows of panel pnl: to y if this CTA covered the
        // whole panel, else as a partial + ticket (last arriver reduces).
        auto flush = [&](int pnl) {
            const int lo = max(u0, pnl * KB), hi = min(u1, (pnl + 1) * KB);
            const int n_lo = pnl * kPanelRows + 16 * j + g, n_hi = n_lo + 8;
            float s_lo = 1.f, s_hi = 1.f;
            if constexpr (BITS == 8) {
                s_lo = n_lo < p.N ? bf16_bits_to_float(p.scales[n_lo]) : 0.f;
                s_hi = n_hi < p.N ? bf16_bits_to_float(p.scales[n_hi]) : 0.f;
            }
            auto store_y = [&](const float (&v)[MT][4]) {
#pragma unroll
                for (int mt = 0; mt < MT; ++mt) {
                    const int m0 = 8 * mt + 2 * t;
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        if (m0 + e < p.M) {
                            if (n_lo < p.N)
                                p.y[(size_t)(m0 + e) * p.N + n_lo] =
                                    __bfloat16_as_ushort(__float2bfloat16_rn(v[mt][e] * s_lo));
                            if (n_hi < p.N)
                                p.y[(size_t)(m0 + e) * p.N + n_hi] =
                                    __bfloat16_as_ushort(__float2bfloat16_rn(v[mt][2 + e] * s_hi));
                        }
                    }
                }
            };
            if (lo == pnl * KB && hi == (pnl + 1) * KB) {
                store_y(acc);
                return;
            }
            constexpr int TOK = 8 * MT;
            const int slot = (pnl == u0 / KB) ? 0 : 1;
            float *mine = p.part + ((size_t)(c * 2 + slot) * kPanelRows) * TOK;
#pragma unroll
            for (int mt = 0; mt < MT; ++mt) {
                const int m0 = 8 * mt + 2 * t;
                *reinterpret_cast<float2 *>(mine + (size_t)(16 * j + g) * TOK + m0) = make_float2(acc[mt][0], acc[mt][1]);
                *reinterpret_cast<float2 *>(mine + (size_t)(16 * j + g + 8) * TOK + m0) =
                    make_float2(acc[mt][2], acc[mt][3]);
            }
            // Each warp takes its own ticket for its 16 rows of the panel, so the
            // fix-up never stalls the CTA's other warps.
            __threadfence();
            __syncwarp();
            uint32_t ticket = 0;
            if (lane == 0)
                ticket = ticket_take(&p.cnt[pnl * 8 + j]);
            ticket = __shfl_sync(0xffffffffu, ticket, 0);
            const int cf = sk_owner(U, G, pnl * KB), cl = sk_owner(U, G, (pnl + 1) * KB - 1);
            if (ticket != (uint32_t)(cl - cf))
                return;
            __threadfence();
            float tot[MT][4];
#pragma unroll
            for (int mt = 0; mt < MT; ++mt)
                tot[mt][0] = tot[mt][1] = tot[mt][2] = tot[mt][3] = 0.f;
            // contributors in CTA order, QC at a time with their loads in flight together
            constexpr int QC = MT == 1 ? 4 : (MT == 2 ? 2 : 1);
            for (int c0 = cf; c0 <= cl; c0 += QC) {
                float2 a[QC][MT], b[QC][MT];
#pragma unroll
                for (int q = 0; q < QC; ++q) {
                    const int cc = c0 + q;
                    if (cc <= cl) {
                        const int sl = (pnl == sk_start(U, G, cc) / KB) ? 0 : 1;
                        const float *src = p.part + ((size_t)(cc * 2 + sl) * kPanelRows) * TOK;
#pragma unroll
                        for (int mt = 0; mt < MT; ++mt) {
                            const int m0 = 8 * mt + 2 * t;
                            a[q][mt] = __ldcg(reinterpret_cast<const float2 *>(src + (size_t)(16 * j + g) * TOK + m0));
                            b[q][mt] = __ldcg(reinterpret_cast<const float2 *>(src + (size_t)(16 * j + g + 8) * TOK + m0));
                        }
                    }
                }
#pragma unroll
                for (int q = 0; q < QC; ++q) {
                    if (c0 + q <= cl) {
#pragma unroll
                        for (int mt = 0; mt < MT; ++mt) {
                            tot[mt][0] += a[q][mt].x;
                            tot[mt][1] += a[q][mt].y;
                            tot[mt][2] += b[q][mt].x;
                            tot[mt][3] += b[q][mt].y;
                        }
                    }
                }
            }
            store_y(tot);
            if (lane == 0)
                atomicExch(&p.cnt[pnl * 8 + j], 0u);
        };

        int cur = n > 0 ? u0 / KB : -1;
        for (int i = 0; i < n; ++i) {
            const int u = u0 + i, pnl = u / KB, kb = u - pnl * KB;
            if (pnl != cur) {
                flush(cur);
#pragma unroll
                for (int mt = 0; mt < MT; ++mt)
                    acc[mt][0] = acc[mt][1] = acc[mt][2] = acc[mt][3] = 0.f;
                cur = pnl;
            }
            const int st = i % STAGES, use = i / STAGES;
            if (ok && !mbar_wait(&full[st], use & 1))
                ok = false;
            const uint8_t *stage = ring + st * C::kStageBytes;
            if (ok) {
                const uint8_t *xs = stage + xoff;
                if constexpr (BITS == 8) {
                    // rows 16j + g and 16j + 8 + g: 8-row groups 2j and 2j + 1, row g of each
                    const uint8_t *wr = stage + (2 * j) * 1024 + g * 128;
                    const int kleft = p.K - kb * kBlockK;
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        const int cc = t + 4 * h;
                        const uint4 wa = *reinterpret_cast<const uint4 *>(wr + ((cc ^ g) << 4));
                        const uint4 wb = *reinterpret_cast<const uint4 *>(wr + 1024 + ((cc ^ g) << 4));
                        const bool kin = 16 * cc < kleft; // chunks past K: zero weights, activations not staged
                        uint4 xv[MT], xw[MT];
#pragma unroll
                        for (int mt = 0; mt < MT; ++mt) {
                            const uint8_t *xp = xs + mt * 8 * C::kXRow + 128 * h;
                            xv[mt] = kin ? *reinterpret_cast<const uint4 *>(xp) : make_uint4(0, 0, 0, 0);
                            xw[mt] = kin ? *reinterpret_cast<const uint4 *>(xp + 16) : make_uint4(0, 0, 0, 0);
                        }
                        sk_int8_chunk<MT>(wa, wb, xv, xw, acc);
                    }
                } else {
                    uint4 w[C::kTPB];
#pragma unroll
                    for (int tt = 0; tt < C::kTPB; ++tt)
                        w[tt] = *reinterpret_cast<const uint4 *>(stage + j * C::kRBB + tt * kTileBytes + lane * 16);
                    const uint16_t *s16 = reinterpret_cast<const uint16_t *>(stage + C::kPBB);
                    const uint8_t *z8 = stage + C::kPBB + 256;
                    const int r = 16 * j + g;
                    const uint32_t zl = (z8[r >> 1] >> (4 * (r & 1))) & 0xFu;
                    const uint32_t zh = (z8[(r + 8) >> 1] >> (4 * (r & 1))) & 0xFu;
                    const uint32_t zlo = 0x43004300u | zl | (zl << 16);
                    const uint32_t zhi = 0x43004300u | zh | (zh << 16);
                    const float slo = bf16_bits_to_float(s16[r]);
                    const float shi = bf16_bits_to_float(s16[r + 8]);
                    float cg[MT][4];
#pragma unroll
                    for (int mt = 0; mt < MT; ++mt)
                        cg[mt][0] = cg[mt][1] = cg[mt][2] = cg[mt][3] = 0.f;
                    sk_int4_tile<MT, C::kXRow>(w[0], xs, 0, zlo, zhi, cg);
                    sk_int4_tile<MT, C::kXRow>(w[1], xs, 64, zlo, zhi, cg);
#pragma unroll
                    for (int mt = 0; mt < MT; ++mt) {
                        acc[mt][0] = fmaf(slo, cg[mt][0], acc[mt][0]);
                        acc[mt][1] = fmaf(slo, cg[mt][1], acc[mt][1]);
                        acc[mt][2] = fmaf(shi, cg[mt][2], acc[mt][2]);
                        acc[mt][3] = fmaf(shi, cg[mt][3], acc[mt][3]);
                    }
                }
            }
            // every read of this stage (weights, scales, activations) is done
            __syncwarp();
            if (lane == 0)
                mbar_arrive(&empty[st]);
        }
        pdl_launch_dependents();
        if (cur >= 0)
            flush(cur);
    }
    if (!ok)
        atomicExch(&g_gemv_sk_error, kErrTimeout);
}

template <int BITS, int MT, int OCC>
static cudaError_t launch_sk_t(const LinearArgs &a, void *ws, int sm_count, cudaStream_t st)
{
    using C = SkCfg<BITS, MT, OCC>;
    constexpr size_t smem = 128 + (size_t)C::kStages * C::kStageBytes + 2 * C::kStages * 8 + 16;
    int occ = 1;
    {
        const cudaError_t e = kernel_setup((const void *)gemv_sk_kernel<BITS, MT, OCC>, smem, kSkThreads, smem, &occ);
        if (e != cudaSuccess)
            return e;
    }
    const int per_sm = OCC < occ ? OCC : occ; // every CTA resident at once
    const Shape sh{a.bits, a.K, a.N, a.group};
    GemvSkParams p;
    p.x = a.x;
    p.M = a.M;
    p.K = a.K;
    p.N = a.N;
    p.wq = (const uint8_t *)a.wq;
    p.scales = (const uint16_t *)a.scales;
    p.zeros = (const uint8_t *)a.zeros;
    p.y = a.y;
    p.KB = sh.kblocks();
    p.U = sh.panels() * sh.kblocks();
    p.cnt = (uint32_t *)ws;
    p.part = (float *)((uint8_t *)ws + ws_counter_bytes());
    int G = per_sm * sm_count;
    if (G > kSkMaxCtas)
        G = kSkMaxCtas;
    if (G > p.U)
        G = p.U;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(G);
    cfg.blockDim = dim3(kSkThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, gemv_sk_kernel<BITS, MT, OCC>, p);
}

template <int BITS, int MT>
static cudaError_t launch_sk_occ(const LinearArgs &a, int occ, void *ws, int sm_count, cudaStream_t st)
{
    switch (occ) {
    case 1: return launch_sk_t<BITS, MT, 1>(a, ws, sm_count, st);
    case 2: return launch_sk_t<BITS, MT, 2>(a, ws, sm_count, st);
    case 4: return launch_sk_t<BITS, MT, 4>(a, ws, sm_count, st);
    default: return launch_sk_t<BITS, MT, 3>(a, ws, sm_count, st);
    }
}

cudaError_t launch_gemv_sk(const LinearArgs &a, int ctas_per_sm, void *ws, int sm_count, cudaStream_t st)
{
    const int mt = (a.M + 7) / 8;
    if (a.bits == 8) {
        if (mt == 1) return launch_sk_occ<8, 1>(a, ctas_per_sm, ws, sm_count, st);
        if (mt == 2) return launch_sk_occ<8, 2>(a, ctas_per_sm, ws, sm_count, st);
        return launch_sk_occ<8, 4>(a, ctas_per_sm, ws, sm_count, st);
    }
    if (mt == 1) return launch_sk_occ<4, 1>(a, ctas_per_sm, ws, sm_count, st);
    if (mt == 2) return launch_sk_occ<4, 2>(a, ctas_per_sm, ws, sm_count, st);
    return launch_sk_occ<4, 4>(a, ctas_per_sm, ws, sm_count, st);
}

cudaError_t read_gemv_sk_error(int *code, cudaStream_t st)
{
    int host = 0, zero = 0;
    cudaError_t e = cudaMemcpyFromSymbolAsync(&host, g_gemv_sk_error, sizeof(int), 0, cudaMemcpyDeviceToHost, st);
    if (e != cudaSuccess)
        return e;
    e = cudaMemcpyToSymbolAsync(g_gemv_sk_error, &zero, sizeof(int), 0, cudaMemcpyHostToDevice, st);
    if (e != cudaSuccess)
        return e;
    e = cudaStreamSynchronize(st);
    *code = host;
    return e;
}

// ===========================================================================
// Allocation-free entry: the stream-K GEMV with its tickets and partial sums
// in a fixed array that lives in the library's own device memory.
//
// For callers that cannot call cudaMalloc when they run the layer: code
// inside a CUDA-graph-captured region or a custom allocator's critical
// section, embedded runtimes whose device memory is fully pre-partitioned, or
// plugin hosts that hand out only input and output buffers.  The array is
// part of the loaded module, so every GPU that loads the library holds it
// (about 4 MiB) until the process exits.
//
// Limits: M <= kNoAllocMaxM tokens and N <= kNoAllocMaxN output channels;
// larger calls are rejected before anything is enqueued.  Every call shares
// the array, so calls that overlap on the GPU (different streams, or
// different host threads without ordering) race; keep them on one stream.
// ===========================================================================
namespace {
constexpr int kNoAllocMaxM = 8;
constexpr int kNoAllocMaxN = 262144;
constexpr size_t kNoAllocTicketBytes = (size_t)(kNoAllocMaxN / kPanelRows) * 8 * sizeof(uint32_t); // 64 KiB
constexpr size_t kNoAllocPartBytes = (size_t)kSkMaxCtas * 2 * kPanelRows * 8 * sizeof(float);       // 4 MiB
constexpr int kNoAllocMaxDevices = 64;
} // namespace

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocTicketBytes + kNoAllocPartBytes];

// Device address of g_noalloc_scratch per device.  In host code the array's
// name is only a host-side stand-in for the device symbol, so the address
// is looked up once per device (with that device current) on the first call.
static void *g_noalloc_addr[kNoAllocMaxDevices] = {};
static std::mutex g_noalloc_mu;

template <int BITS, int OCC>
static cudaError_t launch_sk_noalloc_t(const LinearArgs &a, uint32_t *cnt, float *part, int sm_count,
                                       cudaStream_t st)
{
    using C = SkCfg<BITS, 1, OCC>;
    constexpr size_t smem = 128 + (size_t)C::kStages * C::kStageBytes + 2 * C::kStages * 8 + 16;
    int occ = 1;
    {
        const cudaError_t e = kernel_setup((const void *)gemv_sk_kernel<BITS, 1, OCC>, smem, kSkThreads, smem, &occ);
        if (e != cudaSuccess)
            return e;
    }
    const int per_sm = OCC < occ ? OCC : occ;
    const Shape sh{a.bits, a.K, a.N, a.group};
    GemvSkParams p;
    p.x = a.x;
    p.M = a.M;
    p.K = a.K;
    p.N = a.N;
    p.wq = (const uint8_t *)a.wq;
    p.scales = (const uint16_t *)a.scales;
    p.zeros = (const uint8_t *)a.zeros;
    p.y = a.y;
    p.KB = sh.kblocks();
    p.U = sh.panels() * sh.kblocks();
    p.cnt = cnt;
    p.part = part;
    int G = per_sm * sm_count;
    if (G > kSkMaxCtas)
        G = kSkMaxCtas;
    if (G > p.U)
        G = p.U;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(G);
    cfg.blockDim = dim3(kSkThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    return cudaLaunchKernelEx(&cfg, gemv_sk_kernel<BITS, 1, OCC>, p);
}

int noalloc_max_m() { return kNoAllocMaxM; }
int noalloc_max_n() { return kNoAllocMaxN; }

cudaError_t launch_gemv_sk_noalloc(const LinearArgs &a, int sm_count, cudaStream_t st)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess)
        return e;
    if (dev < 0 || dev >= kNoAllocMaxDevices)
        return cudaErrorInvalidDevice;
    void *base = nullptr;
    {
        std::lock_guard<std::mutex> lk(g_noalloc_mu);
        if (!g_noalloc_addr[dev]) {
            void *ptr = nullptr;
            e = cudaGetSymbolAddress(&ptr, g_noalloc_scratch);
            if (e != cudaSuccess)
                return e;
            g_noalloc_addr[dev] = ptr;
        }
        base = g_noalloc_addr[dev];
    }
    uint32_t *cnt = static_cast<uint32_t *>(base);
    float *part = reinterpret_cast<float *>(static_cast<unsigned char *>(base) + kNoAllocTicketBytes);
    // the tickets this call uses must start at zero (the array keeps the last
    // call's contents); the partial sums are always written before they are read
    const size_t ticket_bytes = (size_t)((a.N + kPanelRows - 1) / kPanelRows) * 8 * sizeof(uint32_t);
    e = cudaMemsetAsync(cnt, 0, ticket_bytes, st);
    if (e != cudaSuccess)
        return e;
    return a.bits == 8 ? launch_sk_noalloc_t<8, 3>(a, cnt, part, sm_count, st)
                       : launch_sk_noalloc_t<4, 3>(a, cnt, part, sm_count, st);
}

} // namespace wq
