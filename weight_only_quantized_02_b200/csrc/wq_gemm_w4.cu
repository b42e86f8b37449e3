// wq_gemm_w4.cu -- W4A16 (group 128, scale and zero point per group) small-M
// GEMM on tcgen05: persistent stream-K, one CTA per SM, every role on its
// own warps with its own ring, so no role waits for another role's round
// trip on every unit.
//
//     y[m][n] = sum_g s[n][g] * D_g[n][m],
//     D_g[n][m] = sum_{k in g} (q[n][k] - z[n][g]) * x[m][k]
//
// (the WnA16 grouping of "Toward a Cleaner Quantization Stack in SGLang",
// Figure 4).  The tensor cores take the exact integers q - z as bf16, so the
// only rounding is the fp32 accumulation; the group scale is applied in fp32
// to each group's accumulator.  Weights are the MMA's M side (128 rows of a
// panel) and tokens its N side (NT = 16 .. 128), so every M <= 128 uses the
// same instruction shape.
//
// Units are (128-row panel, 128-k block) pairs, one group each, laid out
// contiguously in HBM by the packer (wq_layout.h); each CTA takes an equal
// contiguous range of them (the stream-K partitioning that the Marlin
// register and launch scheduling benchmark names as the alternative to a
// fixed split-K).
//
// Warp roles (512 threads):
//   warp 0     scale producer: per unit the group's 256 bytes of scales into
//              a scale ring (bulk copies).
//   warps 1, 3 warp 1 allocates all 512 tensor-memory columns; one thread of
//              each issues eight tcgen05.mma kind::f16 (K = 16 each) per
//              unit, even units and odd units: A (the dequantized tile)
//              from tensor memory, B (x) from shared memory, D into one of
//              kACC per-unit group accumulators.
//   warp 2     x producer: the unit's x tile (NT tokens x 128 k, 2-D tensor
//              map, 128-byte swizzle, rows past M read as zero) into its own
//              ring (kXS stages), released by the MMA's commit.
//   warps 4..  retire warps, one per tensor-memory lane quadrant and column
//              slice: per unit, s[n][g] * D_g into fp32 register totals;
//              at the end of a panel, y (or a partial and a ticket; the last
//              contributor sums every partial in CTA order: deterministic).
//   rest       dequant warps: each fetches its own 16-row blocks of every
//              unit (and their zero points) with 16-byte cp.async into a
//              private shared-memory ring kDepth units deep (the load path,
//              many requests per SM in flight: one thread's bulk copies
//              stream too slowly for the layer), then writes the exact bf16
//              integers q - z into tensor memory (tcgen05.st 16x256b, the
//              register layout the packed tile already has), into one of kAS
//              A stages.  Weights never depend on the preceding kernel.
// Every mbarrier wait is bounded (2 s); on a timeout the device error word
// is set and every role winds down.
#include <cstdint>

#include <cuda_bf16.h>

#include "wq_device.cuh"
#include "wq_gemm_common.cuh"
#include "wq_internal.h"

namespace wq {

static __device__ int g_gemm_w4_error = 0;

struct GemmW4Params {
    int M, K, N, KB, U;
    const uint8_t *wq;
    const uint16_t *scales;
    const uint8_t *zeros;
    uint16_t *y;
    float *part;   // [CTAs][2 slots][NT tokens][128 rows]
    uint32_t *cnt; // [panels][8] tickets
};


template <int NT>
struct W4Cfg {
    static constexpr int kXB = NT * 256;                 // x tile: NT rows x 128 k bf16
    static constexpr int kSS = 32;                       // scale stages (256 B each)
    static constexpr int kXS = NT == 16 ? 8 : NT == 32 ? 6 : 4;
    static constexpr int kDepth = NT <= 32 ? 16 : NT == 64 ? 14 : 10; // units in each dequant warp's ring
    static constexpr int kACC = NT <= 32 ? 128 / NT : 256 / NT; // group accumulators
    static constexpr int kA0 = kACC * NT;                // first A column
    static constexpr int kAS = (512 - kA0) / 64;         // A stages, 64 columns each
    // 16 warps, except 20 at 64 tokens: eight retire warps (their totals fill
    // the registers) then leave eight dequant warps, one per 16-row block;
    // with four, dequantization paced the whole pipeline
    static constexpr int kWarps = NT == 64 ? 20 : 16;
    static constexpr int kThreads = 32 * kWarps;
    static constexpr int kRW = NT >= 64 ? 8 : 4;         // retire warps
    static constexpr int kCW = NT * 4 / kRW;             // token columns per retire warp
    static constexpr int kDW = kWarps - 4 - kRW;         // dequant warps
    static constexpr int kRetireCols = kWarps == 20 ? 16 : 32; // accumulator columns per tensor-memory wait
    static constexpr int kBPW = 8 / kDW;                 // 16-row blocks per dequant warp
    static constexpr int kSlot = kBPW * 1024 + 16;       // a unit's blocks + its 16-byte zero-point segment
    static_assert(kA0 + 64 * kAS == 512, "tensor memory plan");
    static_assert(kAS >= 2 && kACC >= 2, "double buffering");
    static_assert(kDW == 4 || kDW == 8, "dequant warps cover the four lane quadrants evenly");
    static_assert(kCW % 16 == 0, "retire loads 16 columns at a time");
    // The two MMA issuers take alternate units, so a stage of every ring they
    // wait on must come back to the same issuer: with an odd ring an issuer
    // could test a barrier two phases ahead, where the parity wait passes.
    static_assert(kXS % 2 == 0 && kAS % 2 == 0 && kACC % 2 == 0, "rings the MMA issuers wait on are even");
};

// d0 += a b0, d1 += a b1: one packed fp32 FMA (each half rounded as fmaf).
__device__ __forceinline__ void ffma2(float &d0, float &d1, float a, float b0, float b1)
{
    unsigned long long d, aa, bb;
    asm("mov.b64 %0, {%1, %2};" : "=l"(d) : "f"(d0), "f"(d1));
    asm("mov.b64 %0, {%1, %1};" : "=l"(aa) : "f"(a));
    asm("mov.b64 %0, {%1, %2};" : "=l"(bb) : "f"(b0), "f"(b1));
    asm("fma.rn.f32x2 %0, %1, %2, %0;" : "+l"(d) : "l"(aa), "l"(bb));
    asm("mov.b64 {%0, %1}, %2;" : "=f"(d0), "=f"(d1) : "l"(d));
}

// 16-byte asynchronous global -> shared copy (L2 only) and its groups.
__device__ __forceinline__ void cp_async_cg16(uint32_t dst, const void *src)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait_group()
{
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

template <int NT>
constexpr size_t gemm_w4_smem_bytes()
{
    using C = W4Cfg<NT>;
    return 1024 + (size_t)C::kXS * C::kXB + (size_t)C::kSS * 256 + (size_t)C::kDW * C::kDepth * C::kSlot +
           (size_t)(2 * C::kXS + 2 * C::kSS + 2 * C::kAS + 2 * C::kACC) * 8 + 16 +
           (size_t)2 * (kSkMaxCtas + 1) * sizeof(int);
}

// The last contributor to a split panel: sums the fp32 partials of CTAs
// cf .. cl for its row r and tokens t0 .. t0 + CW - 1 in CTA order and
// writes y.  The partials are token-major, so every load is one coalesced
// 128-byte row segment per warp; CG contributors x 16 tokens are in flight
// together (this runs at the very end of the call, on its critical path).
// Called after the retire loop, whose register totals are dead by then.
template <int NT, int CW>
__device__ __forceinline__ void w4_fixup(const GemmW4Params &p, const SkTable &sk, int pnl, int cf, int cl, int r,
                                         int t0)
{
    const int nrow = pnl * kPanelRows + r;
    constexpr int CG = 4;
    for (int j0 = 0; j0 < CW; j0 += 16) {
        float acc[16];
#pragma unroll
        for (int j = 0; j < 16; ++j)
            acc[j] = 0.f;
        for (int c0 = cf; c0 <= cl; c0 += CG) {
            float v[CG][16];
#pragma unroll
            for (int u = 0; u < CG; ++u) {
                const int cc = c0 + u;
                if (cc <= cl) {
                    const int sl = pnl == sk.first[cc] ? 0 : 1;
                    const float *src = p.part + ((size_t)(cc * 2 + sl) * NT + t0 + j0) * kPanelRows + r;
#pragma unroll
                    for (int j = 0; j < 16; ++j)
                        v[u][j] = __ldcg(src + j * kPanelRows);
                }
            }
#pragma unroll
            for (int u = 0; u < CG; ++u) // in CTA order
                if (c0 + u <= cl)
#pragma unroll
                    for (int j = 0; j < 16; ++j)
                        acc[j] += v[u][j];
        }
        if (nrow < p.N) {
            const int jn = min(16, p.M - t0 - j0);
            uint16_t *yp = p.y + (size_t)(t0 + j0) * p.N + nrow;
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                if (j < jn)
                    *yp = __bfloat16_as_ushort(__float2bfloat16_rn(acc[j]));
                yp += p.N;
            }
        }
    }
}

template <int NT>
__global__ void __launch_bounds__(W4Cfg<NT>::kThreads, 1) gemm_w4_kernel(const __grid_constant__ CUtensorMap tmx,
                                                                const GemmW4Params p)
{
    using C = W4Cfg<NT>;
    constexpr int XS = C::kXS, SS = C::kSS, AS = C::kAS, ACC = C::kACC, DEPTH = C::kDepth, SLOT = C::kSlot;
    constexpr int XB = C::kXB, A0 = C::kA0;
    constexpr int RW = C::kRW, CW = C::kCW, DW = C::kDW, BPW = C::kBPW;

    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sX = smem;              // XS x tiles, 1024-byte aligned (swizzled operand)
    uint8_t *sS = sX + XS * XB;      // SS group scales
    uint8_t *sQ = sS + SS * 256;     // DW private rings of DEPTH slots
    uint64_t *bars = reinterpret_cast<uint64_t *>(sQ + (size_t)DW * DEPTH * SLOT);
    uint64_t *xfull = bars, *xempty = xfull + XS;
    uint64_t *sfull = xempty + XS, *sempty = sfull + SS;
    uint64_t *afull = sempty + SS, *aempty = afull + AS;
    uint64_t *accfull = aempty + AS, *accempty = accfull + ACC;
    uint32_t *s_tmem = reinterpret_cast<uint32_t *>(accempty + ACC);
    int *s_start = reinterpret_cast<int *>(s_tmem + 4); // [kSkMaxCtas + 1]
    int *s_first = s_start + kSkMaxCtas + 1;            // [kSkMaxCtas + 1]

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int G = gridDim.x, cta = blockIdx.x;
    const long long U = p.U;
    const int KB = p.KB;
    for (int c = threadIdx.x; c <= G; c += blockDim.x) {
        const int st = sk_start(U, G, c);
        s_start[c] = st;
        s_first[c] = st / KB;
    }
    const SkTable sk{s_start, s_first};
    const int u0 = sk_start(U, G, cta), u1 = sk_start(U, G, cta + 1);
    const int n = u1 - u0;

    if (threadIdx.x == 0) {
        for (int s = 0; s < XS; ++s) {
            mbar_init(&xfull[s], 1);
            mbar_init(&xempty[s], 1);
        }
        for (int s = 0; s < SS; ++s) {
            mbar_init(&sfull[s], 1);
            mbar_init(&sempty[s], RW);
        }
        for (int s = 0; s < AS; ++s) {
            mbar_init(&afull[s], DW);
            mbar_init(&aempty[s], 1);
        }
        for (int s = 0; s < ACC; ++s) {
            mbar_init(&accfull[s], 1);
            mbar_init(&accempty[s], RW);
        }
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(s_tmem, 512);
        tmem_relinquish();
    }
    if (warp == 2 && lane == 0)
        prefetch_tensormap(&tmx);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    // The next kernel on the stream may launch now; whatever it shares with
    // this grid (its x, y, the workspace) waits behind its own launch wait.
    pdl_launch_dependents();
    const uint32_t tmem = *s_tmem;
    bool ok = true;

    auto panel_of = [&](int i) { return (u0 + i) / KB; };

    if (warp == 0) {
        // ---------------- scale producer ----------------
        if (lane == 0) {
            const uint64_t pol = policy_evict_first();
            for (int i = 0; i < n; ++i) {
                const size_t u = (size_t)(u0 + i);
                const int ss = i % SS;
                if (i >= SS && !mbar_wait(&sempty[ss], ((i / SS) - 1) & 1)) {
                    ok = false;
                    break;
                }
                mbar_arrive_expect_tx(&sfull[ss], 256);
                bulk_g2s(sS + ss * 256, p.scales + u * kPanelRows, 256, &sfull[ss], pol);
            }
        }
    } else if (warp == 1 || warp == 3) {
        // ---------------- MMA issuers ----------------
        // Two issuing threads, warp 1 for even units and warp 3 for odd ones:
        // one thread's waits, descriptor arithmetic and commits cost more
        // per unit than the eight small MMAs do on the tensor core.  Every
        // unit has its own A stage and accumulator, so the two streams of
        // MMAs are independent.
        if (lane == 0) {
            constexpr uint32_t idesc = umma_idesc_bf16(NT);
            for (int i = warp == 1 ? 0 : 1; i < n; i += 2) {
                const int as = i % AS, xs = i % XS, ac = i % ACC;
                if (!mbar_wait(&afull[as], (i / AS) & 1) || !mbar_wait(&xfull[xs], (i / XS) & 1) ||
                    (i >= ACC && !mbar_wait(&accempty[ac], ((i / ACC) - 1) & 1))) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                // the descriptor's start-address field is addr >> 4: step along
                // K inside the swizzled tile by adding the byte offset >> 4
                const uint64_t bdesc0 = smem_desc_sw128(smem_u32(sX + xs * XB));
                const uint32_t d_t = tmem + ac * NT, a_t = tmem + A0 + as * 64;
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    umma_ts(d_t, a_t + kk * 8, bdesc0 + (uint64_t)((((kk >> 2) * (NT * 128)) + (kk & 3) * 32) >> 4),
                            idesc, kk > 0 ? 1u : 0u);
                umma_commit(&aempty[as]);
                umma_commit(&xempty[xs]);
                umma_commit(&accfull[ac]);
            }
        }
    } else if (warp == 2) {
        // ---------------- x producer ----------------
        if (lane == 0) {
            pdl_wait(); // x may be written by the preceding kernel
            const uint64_t pol = policy_evict_last();
            for (int i = 0; i < n; ++i) {
                const int xs = i % XS, kb = (u0 + i) % KB;
                if (i >= XS && !mbar_wait(&xempty[xs], ((i / XS) - 1) & 1)) {
                    ok = false;
                    break;
                }
                mbar_arrive_expect_tx(&xfull[xs], XB);
                tma_load_2d(sX + xs * XB, &tmx, kb * kBlockK, 0, &xfull[xs], pol);
                tma_load_2d(sX + xs * XB + NT * 128, &tmx, kb * kBlockK + 64, 0, &xfull[xs], pol);
            }
        }
    } else if (warp >= 4 && warp < 4 + RW) {
        // ---------------- retire warps ----------------
        pdl_wait(); // y and the workspace may still be in use by the preceding kernel
        const int q = warp & 3, c = (warp - 4) >> 2; // lane quadrant, column slice
        const int dw = q + 4 * c;                    // ticket owner index within a panel
        const int r = 32 * q + lane;                 // output row (in the panel) of this thread
        const uint32_t tq = (uint32_t)(32 * q) << 16;
        float tot[CW];
#pragma unroll
        for (int j = 0; j < CW; ++j)
            tot[j] = 0.f;
        int fix_pnl[2], fix_cf[2], fix_cl[2], nfix = 0; // split panels this warp finishes (a range touches <= 2 panels)

        // This thread's CW totals of panel pnl: to y when this CTA covered
        // the whole panel, else as a partial + per-warp ticket.
        auto flush = [&](int pnl) {
            const int lo = max(u0, pnl * KB), hi = min(u1, (pnl + 1) * KB);
            const int nrow = pnl * kPanelRows + r;
            const int t0 = c * CW; // first token of this slice
            if (lo == pnl * KB && hi == (pnl + 1) * KB) {
                if (nrow < p.N) {
                    const int jn = min(CW, p.M - t0); // tokens of this slice that exist
                    uint16_t *yp = p.y + (size_t)t0 * p.N + nrow;
#pragma unroll
                    for (int j = 0; j < CW; ++j) {
                        if (j < jn)
                            *yp = __bfloat16_as_ushort(__float2bfloat16_rn(tot[j]));
                        yp += p.N;
                    }
                }
                return;
            }
            const int slot = (pnl == u0 / KB) ? 0 : 1;
            float *mine = p.part + ((size_t)(cta * 2 + slot) * NT + t0) * kPanelRows + r;
#pragma unroll
            for (int j = 0; j < CW; ++j)
                mine[j * kPanelRows] = tot[j]; // token-major: the warp writes 128 contiguous bytes
            __threadfence(); // every lane's partial is visible before lane 0's ticket
            __syncwarp();
            uint32_t ticket = 0;
            if (lane == 0)
                ticket = ticket_take_acq_rel(&p.cnt[pnl * 8 + dw]);
            ticket = __shfl_sync(0xffffffffu, ticket, 0);
            const int cf = sk.owner(pnl * KB, G), cl = sk.owner((pnl + 1) * KB - 1, G);
            if (ticket != (uint32_t)(cl - cf))
                return;
            // the last contributor: sum the partials once the loop is done
            fix_pnl[nfix] = pnl;
            fix_cf[nfix] = cf;
            fix_cl[nfix] = cl;
            ++nfix;
        };

        int kb = u0 % KB; // k-block of unit i, kept without dividing
        for (int i = 0; i < n; ++i) {
            const int ac = i % ACC, ss = i % SS;
            if (!mbar_wait_warp(&accfull[ac], (i / ACC) & 1) || !mbar_wait_warp(&sfull[ss], (i / SS) & 1)) {
                ok = false;
                break;
            }
            tc_fence_after();
            const float s = bf16_bits_to_float(reinterpret_cast<const uint16_t *>(sS + ss * 256)[r]);
            const uint32_t ta = tmem + tq + ac * NT + c * CW;
            constexpr int RC = C::kRetireCols; // columns per wait
#pragma unroll
            for (int j0 = 0; j0 < CW; j0 += RC) {
                float v[RC / 16][16];
#pragma unroll
                for (int h = 0; h < RC / 16; ++h)
                    if (j0 + 16 * h < CW)
                        tmem_ld_32x32b_x16(ta + j0 + 16 * h, v[h]);
                tmem_wait_ld();
#pragma unroll
                for (int h = 0; h < RC / 16; ++h)
                    if (j0 + 16 * h < CW)
#pragma unroll
                        for (int j = 0; j < 16; j += 2)
                            ffma2(tot[j0 + 16 * h + j], tot[j0 + 16 * h + j + 1], s, v[h][j], v[h][j + 1]);
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&accempty[ac]);
                mbar_arrive(&sempty[ss]);
            }
            if (i == n - 1 || kb == KB - 1) { // the last unit of a panel
                flush(panel_of(i));
#pragma unroll
                for (int j = 0; j < CW; ++j)
                    tot[j] = 0.f;
            }
            kb = kb + 1 == KB ? 0 : kb + 1;
        }
        __syncwarp(); // lane 0's acquire (the tickets) orders every lane's reads below
        for (int f = 0; f < nfix && ok; ++f) {
            w4_fixup<NT, CW>(p, sk, fix_pnl[f], fix_cf[f], fix_cl[f], r, c * CW);
            if (lane == 0)
                atomicExch(&p.cnt[fix_pnl[f] * 8 + dw], 0u); // ready for the next call
        }
    } else if (warp >= 4 + RW) {
        // ---------------- dequant warps ----------------
        const int d = warp - 4 - RW;  // 0 .. DW-1
        const int q = warp & 3;       // lane quadrant
        const int g = lane >> 2;
        int jb[BPW];                  // this warp's 16-row blocks (rows 32q .. 32q+31)
#pragma unroll
        for (int b = 0; b < BPW; ++b)
            jb[b] = BPW == 1 ? 2 * q + (d >> 2) : 2 * q + b;
        uint8_t *ring = sQ + (size_t)d * DEPTH * SLOT;
        const int zseg = 16 * (jb[0] >> 1); // the 16-byte segment of a unit's zero points holding these rows
        auto issue = [&](int i) {           // this warp's part of unit i into slot i % DEPTH
            const uint8_t *src = p.wq + (size_t)(u0 + i) * 8192;
            const uint32_t dst = smem_u32(ring + (i % DEPTH) * SLOT);
#pragma unroll
            for (int b = 0; b < BPW; ++b) {
                cp_async_cg16(dst + b * 1024 + lane * 16, src + jb[b] * 1024 + lane * 16);
                cp_async_cg16(dst + b * 1024 + 512 + lane * 16, src + jb[b] * 1024 + 512 + lane * 16);
            }
            if (lane == 0)
                cp_async_cg16(dst + BPW * 1024, p.zeros + (size_t)(u0 + i) * 64 + zseg);
        };
#pragma unroll 1
        for (int i = 0; i < DEPTH - 1; ++i) { // one commit group per unit, DEPTH - 1 ahead
            if (i < n)
                issue(i);
            cp_async_commit();
        }
        for (int i = 0; i < n; ++i) {
            const int as = i % AS;
            __syncwarp(); // every lane has read the slot refilled next (the zero points are shared)
            if (i + DEPTH - 1 < n)
                issue(i + DEPTH - 1);
            cp_async_commit();
            cp_async_wait_group<DEPTH - 1>(); // unit i has landed (this lane's copies)
            __syncwarp();                     // ... and lane 0's zero points
            const uint8_t *blk = ring + (i % DEPTH) * SLOT;
            uint32_t rr[BPW][2][16];
#pragma unroll
            for (int b = 0; b < BPW; ++b) {
                const uint4 w0 = *reinterpret_cast<const uint4 *>(blk + b * 1024 + lane * 16);
                const uint4 w1 = *reinterpret_cast<const uint4 *>(blk + b * 1024 + 512 + lane * 16);
                const int zo = BPW * 1024 + 8 * (jb[b] & 1) + (g >> 1); // rows 16 jb + g and 16 jb + g + 8
                const uint32_t z0 = (blk[zo] >> (4 * (g & 1))) & 0xFu;
                const uint32_t z1 = (blk[zo + 4] >> (4 * (g & 1))) & 0xFu;
                const uint32_t zlo = 0x43004300u | z0 | (z0 << 16); // bf16x2 {128 + z, 128 + z}
                const uint32_t zhi = 0x43004300u | z1 | (z1 << 16);
                int4_tile_regs(w0, zlo, zhi, rr[b][0]);
                int4_tile_regs(w1, zlo, zhi, rr[b][1]);
            }
            if (i >= AS && !mbar_wait_warp(&aempty[as], ((i / AS) - 1) & 1)) {
                ok = false;
                break;
            }
            tc_fence_after();
#pragma unroll
            for (int b = 0; b < BPW; ++b) {
                const uint32_t ta = tmem + ((uint32_t)(32 * q + 16 * (jb[b] & 1)) << 16) + A0 + as * 64;
                tmem_st_16x256b_x4(ta, rr[b][0]);
                tmem_st_16x256b_x4(ta + 32, rr[b][1]);
            }
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0)
                mbar_arrive(&afull[as]);
        }
        cp_async_wait_group<0>(); // no copy outlives the CTA (a timeout leaves the loop early)
    }

    if (!ok)
        atomicExch(&g_gemm_w4_error, kErrTimeout);
    tc_fence_before();
    // Lane 0 of warps 0-2 ran its role alone: reconverge every warp first, so
    // the CTA barrier below (aligned: whole warps) waits for every role to
    // finish before tensor memory is released.
    __syncwarp();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

template <int NT>
static cudaError_t launch_gemm_w4_t(const LinearArgs &a, void *ws, int sm_count, cudaStream_t st)
{
    constexpr size_t smem = gemm_w4_smem_bytes<NT>();
    static_assert(smem <= 227 * 1024, "shared memory per CTA");
    {
        const cudaError_t e = kernel_setup((const void *)gemm_w4_kernel<NT>, smem, 0, 0, nullptr);
        if (e != cudaSuccess)
            return e;
    }
    CUtensorMap map;
    if (!make_x_map<NT>(&map, a.x, a.M, a.K))
        return cudaErrorInvalidValue;
    const Shape sh{a.bits, a.K, a.N, a.group};
    GemmW4Params p;
    p.M = a.M;
    p.K = a.K;
    p.N = a.N;
    p.KB = sh.kblocks();
    p.U = sh.panels() * sh.kblocks();
    p.wq = (const uint8_t *)a.wq;
    p.scales = (const uint16_t *)a.scales;
    p.zeros = (const uint8_t *)a.zeros;
    p.y = a.y;
    p.cnt = (uint32_t *)ws;
    p.part = (float *)((uint8_t *)ws + ws_counter_bytes());
    int G = sm_count;
    if (G > kSkMaxCtas)
        G = kSkMaxCtas;
    if (G > p.U)
        G = p.U;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(G);
    cfg.blockDim = dim3(W4Cfg<NT>::kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, gemm_w4_kernel<NT>, map, p);
}

cudaError_t launch_gemm_w4(const LinearArgs &a, void *ws, int sm_count, cudaStream_t st)
{
    switch (gemm_token_tile(a.M)) {
    case 16: return launch_gemm_w4_t<16>(a, ws, sm_count, st);
    case 32: return launch_gemm_w4_t<32>(a, ws, sm_count, st);
    case 64: return launch_gemm_w4_t<64>(a, ws, sm_count, st);
    default: return launch_gemm_w4_t<128>(a, ws, sm_count, st);
    }
}

cudaError_t read_gemm_w4_error(int *code, cudaStream_t st)
{
    int host = 0, zero = 0;
    cudaError_t e = cudaMemcpyFromSymbolAsync(&host, g_gemm_w4_error, sizeof(int), 0, cudaMemcpyDeviceToHost, st);
    if (e != cudaSuccess)
        return e;
    e = cudaMemcpyToSymbolAsync(g_gemm_w4_error, &zero, sizeof(int), 0, cudaMemcpyHostToDevice, st);
    if (e != cudaSuccess)
        return e;
    e = cudaStreamSynchronize(st);
    *code = host;
    return e;
}

} // namespace wq
