// wq_gemm_sk.cu -- persistent stream-K GEMM on tcgen05, any M <= 128.
//
// The packed weights are one contiguous stream of (128-row panel, 128-k
// block) units; each persistent CTA takes an equal contiguous range of it,
// so the whole GPU stays busy whatever the panel count (a 5120-row layer is
// only 40 panels for 148 SMs).  This is the stream-K partitioning that the
// Marlin register and launch scheduling benchmark names as the alternative
// to a fixed split-K.
//
// Warp roles (320 threads):
//   warp 0     producer: per unit, the x tile (2-D tensor map, 128-byte
//              swizzle) and the packed weight block (+ INT4 scales, zeros)
//              as bulk copies into a STAGES-deep ring.  Weights are
//              prefetched before the programmatic-launch wait, x after.
//   warp 1     allocates tensor memory; one thread issues tcgen05.mma with
//              the dequantized tile as the A operand from tensor memory.
//   warps 2-9  two dequant warps per tensor-memory lane quadrant: exact
//              integers (INT4 q - z, INT8 q) as bf16 into tensor memory.
//              INT4: one 16-row block per warp, tcgen05.st 16x256b; INT8:
//              one row per thread, half of the block's k each, 32x32b.
//              One unit behind the
//              MMA they retire finished work: INT4 folds s[row][g] * D_g of
//              every group into fp32 register totals (two group accumulators
//              in tensor memory, double-buffered); INT8 reads a panel's
//              accumulator (two, double-buffered) when its last unit is done.
//              Each warp owns 32 rows x NT/2 tokens of the output.
// Panels split between CTAs are finished by the last warp to arrive for
// its rows and tokens (ticket per (panel, warp), never waited on), summing
// the partials of all contributors in CTA order: deterministic.
// Every mbarrier wait is bounded (2 s); on a timeout the device error word
// is set and the CTA winds down.
#include <cstdint>

#include "wq_device.cuh"
#include "wq_gemm_common.cuh"
#include "wq_internal.h"

namespace wq {

static __device__ int g_gemm_sk_error = 0;

struct GemmSkParams {
    int M, K, N, KB, U;
    const uint8_t *wq;
    const uint16_t *scales;
    const uint8_t *zeros;
    uint16_t *y;
    float *part;   // [CTAs][2][128 rows][NT]
    uint32_t *cnt; // [panels][8]
};

template <int BITS, int NT>
struct GskCfg {
    static constexpr int kWB = BITS == 4 ? 8192 : 16384;
    static constexpr int kSZB = BITS == 4 ? 512 : 0;
    static constexpr int kSZTx = BITS == 4 ? 320 : 0;
    static constexpr int kTPR = BITS == 4 ? 2 : 4;
    static constexpr int kXB = NT * 256;
    static constexpr int kStageBytes = kXB + kWB + kSZB;
    static constexpr int kTmemCols = NT >= 64 ? 512 : 256;
    static constexpr int kA0 = 2 * NT < 64 ? 64 : 2 * NT; // two accumulators, then the A ring
    static constexpr int kTmemStages = (kTmemCols - kA0) / 64;
    static constexpr int kSmemStages = (kTmemCols == 512 ? 200 * 1024 : 100 * 1024) / kStageBytes;
    static constexpr int kStagesRaw = kTmemStages < kSmemStages ? kTmemStages : kSmemStages;
    static constexpr int kStages = kStagesRaw > 6 ? 6 : kStagesRaw;
    static constexpr int kOcc = kTmemCols == 512 ? 1 : 2;
    // registers per thread: 10 warps put 3 on some SM sub-partition (16K
    // registers each), so one CTA gets at most 168, two CTAs at most 96
    static constexpr int kMaxRegs = kOcc == 1 ? 168 : 96;
    static_assert(kStages >= 2, "pipeline needs two stages");
    static_assert(kA0 + 64 * kStages <= kTmemCols, "tensor memory budget");
};

constexpr int kGskThreads = 320;

template <int BITS, int NT>
constexpr size_t gemm_sk_smem_bytes()
{
    using C = GskCfg<BITS, NT>;
    return 1024 + (size_t)C::kStages * C::kStageBytes + (4 * C::kStages + 4) * 8 + 16;
}

// Load `HALF` accumulator columns of this warp's 32 rows.
template <int HALF>
__device__ __forceinline__ void tmem_load_cols(uint32_t taddr, float (&v)[HALF])
{
    if constexpr (HALF == 8) {
        tmem_ld_32x32b_x8(taddr, v);
    } else {
#pragma unroll
        for (int c0 = 0; c0 < HALF; c0 += 16) {
            float t[16];
            tmem_ld_32x32b_x16(taddr + c0, t);
#pragma unroll
            for (int e = 0; e < 16; ++e)
                v[c0 + e] = t[e];
        }
    }
    tmem_wait_ld();
}

template <int BITS, int NT>
__global__ void __launch_bounds__(kGskThreads) __maxnreg__((GskCfg<BITS, NT>::kMaxRegs))
    gemm_sk_kernel(const __grid_constant__ CUtensorMap tmx, const GemmSkParams p)
{
    using C = GskCfg<BITS, NT>;
    constexpr int STAGES = C::kStages, TCOLS = C::kTmemCols, A0 = C::kA0;
    constexpr int XB = C::kXB, WB = C::kWB, SZB = C::kSZB, TPR = C::kTPR;
    constexpr int HALF = NT / 2;

    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sX = smem;
    uint8_t *sW = sX + STAGES * XB;
    uint8_t *sSZ = sW + STAGES * WB;
    uint64_t *bars = reinterpret_cast<uint64_t *>(sSZ + STAGES * SZB);
    uint64_t *full = bars, *ldempty = bars + STAGES, *afull = bars + 2 * STAGES, *aempty = bars + 3 * STAGES;
    uint64_t *accfull = bars + 4 * STAGES, *accempty = bars + 4 * STAGES + 2;
    uint32_t *s_misc = reinterpret_cast<uint32_t *>(bars + 4 * STAGES + 4);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int G = gridDim.x, cta = blockIdx.x;
    const long long U = p.U;
    const int KB = p.KB;
    const int u0 = sk_start(U, G, cta), u1 = sk_start(U, G, cta + 1);
    const int n = u1 - u0;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&ldempty[s], 1 + 8);
            mbar_init(&afull[s], 8);
            mbar_init(&aempty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&accfull[b], 1);
            mbar_init(&accempty[b], 8);
        }
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(&s_misc[0], TCOLS);
        tmem_relinquish();
    }
    if (warp == 0 && lane == 0)
        prefetch_tensormap(&tmx);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = s_misc[0];
    bool ok = true;

    auto panel_of = [&](int i) { return (u0 + i) / KB; };
    auto last_of_panel = [&](int i) { return i == n - 1 || panel_of(i + 1) != panel_of(i); };

    if (warp == 0) {
        if (lane == 0) {
            const uint64_t pol_w = policy_evict_first(), pol_x = policy_evict_last();
            auto issue_w = [&](int i, int st) {
                const size_t u = (size_t)(u0 + i);
                mbar_arrive_expect_tx(&full[st], XB + WB + C::kSZTx);
                bulk_g2s(sW + st * WB, p.wq + u * WB, WB, &full[st], pol_w);
                if constexpr (BITS == 4) {
                    bulk_g2s(sSZ + st * SZB, p.scales + u * kPanelRows, 256, &full[st], pol_w);
                    bulk_g2s(sSZ + st * SZB + 256, p.zeros + u * 64, 64, &full[st], pol_w);
                }
            };
            auto issue_x = [&](int i, int st) {
                const int kb = (u0 + i) % KB;
                tma_load_2d(sX + st * XB, &tmx, kb * kBlockK, 0, &full[st], pol_x);
                tma_load_2d(sX + st * XB + NT * 128, &tmx, kb * kBlockK + 64, 0, &full[st], pol_x);
            };
            const int pre = n < STAGES ? n : STAGES;
            for (int i = 0; i < pre; ++i)
                issue_w(i, i);
            pdl_wait();
            for (int i = 0; i < pre; ++i)
                issue_x(i, i);
            for (int i = pre; i < n; ++i) {
                const int st = i % STAGES, use = i / STAGES;
                if (!mbar_wait(&ldempty[st], (use - 1) & 1)) {
                    ok = false;
                    break;
                }
                issue_w(i, st);
                issue_x(i, st);
            }
        } else {
            pdl_wait();
        }
        pdl_launch_dependents();
    } else if (warp == 1) {
        pdl_wait();
        if (lane == 0) {
            constexpr uint32_t idesc = umma_idesc_bf16(NT);
            int pi = -1; // INT8: index of the panel being accumulated, within this range
            for (int i = 0; i < n && ok; ++i) {
                const int st = i % STAGES, use = i / STAGES;
                if (!mbar_wait(&afull[st], use & 1) || !mbar_wait(&full[st], use & 1)) {
                    ok = false;
                    break;
                }
                bool fresh;
                uint32_t dcol;
                if constexpr (BITS == 4) {
                    const int b = i & 1;
                    if (i >= 2 && !mbar_wait(&accempty[b], ((i >> 1) - 1) & 1)) {
                        ok = false;
                        break;
                    }
                    fresh = true;
                    dcol = b * NT;
                } else {
                    fresh = (i == 0) || panel_of(i) != panel_of(i - 1);
                    if (fresh) {
                        ++pi;
                        if (pi >= 2 && !mbar_wait(&accempty[pi & 1], ((pi >> 1) - 1) & 1)) {
                            ok = false;
                            break;
                        }
                    }
                    dcol = (pi & 1) * NT;
                }
                tc_fence_after();
                const uint32_t xs = smem_u32(sX + st * XB);
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint64_t bdesc = smem_desc_sw128(xs + (kk >> 2) * (NT * 128) + (kk & 3) * 32);
                    umma_ts(tmem + dcol, tmem + A0 + st * 64 + kk * 8, bdesc, idesc, (fresh && kk == 0) ? 0u : 1u);
                }
                umma_commit(&aempty[st]);
                umma_commit(&ldempty[st]);
                if constexpr (BITS == 4)
                    umma_commit(&accfull[i & 1]);
                else if (last_of_panel(i))
                    umma_commit(&accfull[pi & 1]);
            }
        }
        pdl_launch_dependents();
    } else {
        // ---------------- dequant / retire / epilogue warps ----------------
        pdl_wait(); // y and the workspace may still be in use by the preceding kernel
        const int dw = warp - 2;          // 0..7
        const int q = warp & 3, h = dw >> 2;
        const int j = 2 * q + h;          // INT4: 16-row block this warp dequantizes
        const int g = lane >> 2;
        const int r = 32 * q + lane;      // output row (in the panel) this thread retires
        const uint32_t tq = (uint32_t)(32 * q) << 16;
        float acc[HALF];
#pragma unroll
        for (int c = 0; c < HALF; ++c)
            acc[c] = 0.f;
        float s_prev = 0.f;

        // Stores this thread's HALF values of panel pnl: to y when this CTA
        // covered the whole panel, else as a partial + per-warp ticket.
        auto flush = [&](int pnl, const float (&v)[HALF]) {
            const int lo = max(u0, pnl * KB), hi = min(u1, (pnl + 1) * KB);
            const int nrow = pnl * kPanelRows + r;
            float scale = 1.f;
            if constexpr (BITS == 8)
                scale = nrow < p.N ? bf16_bits_to_float(p.scales[nrow]) : 0.f;
            auto store_y = [&](const float (&t)[HALF]) {
                if (nrow < p.N) {
#pragma unroll
                    for (int c = 0; c < HALF; ++c)
                        if (h * HALF + c < p.M)
                            p.y[(size_t)(h * HALF + c) * p.N + nrow] =
                                __bfloat16_as_ushort(__float2bfloat16_rn(t[c] * scale));
                }
            };
            if (lo == pnl * KB && hi == (pnl + 1) * KB) {
                store_y(v);
                return;
            }
            const int slot = (pnl == u0 / KB) ? 0 : 1;
            float *mine = p.part + ((size_t)(cta * 2 + slot) * kPanelRows + r) * NT + h * HALF;
#pragma unroll
            for (int c = 0; c < HALF; c += 4)
                *reinterpret_cast<float4 *>(mine + c) = make_float4(v[c], v[c + 1], v[c + 2], v[c + 3]);
            __threadfence();
            __syncwarp();
            uint32_t ticket = 0;
            if (lane == 0)
                ticket = ticket_take(&p.cnt[pnl * 8 + dw]);
            ticket = __shfl_sync(0xffffffffu, ticket, 0);
            const int cf = sk_owner(U, G, pnl * KB), cl = sk_owner(U, G, (pnl + 1) * KB - 1);
            if (ticket != (uint32_t)(cl - cf))
                return;
            __threadfence();
            // sum all contributors in CTA order, 8 or 16 tokens at a time
            constexpr int CH = HALF < 16 ? HALF : 16;
#pragma unroll
            for (int c0 = 0; c0 < HALF; c0 += CH) {
                float tot[CH];
#pragma unroll
                for (int c = 0; c < CH; ++c)
                    tot[c] = 0.f;
                // two contributors' partials in flight at once, summed in CTA order
                for (int cc0 = cf; cc0 <= cl; cc0 += 2) {
                    float4 t4[2][CH / 4];
#pragma unroll
                    for (int u = 0; u < 2; ++u) {
                        const int cc = cc0 + u;
                        const int sl = (cc <= cl && pnl == sk_start(U, G, cc) / KB) ? 0 : 1;
                        const float *src = p.part + ((size_t)(cc * 2 + sl) * kPanelRows + r) * NT + h * HALF + c0;
#pragma unroll
                        for (int c = 0; c < CH; c += 4)
                            t4[u][c / 4] = cc <= cl ? __ldcg(reinterpret_cast<const float4 *>(src + c))
                                                    : make_float4(0.f, 0.f, 0.f, 0.f);
                    }
#pragma unroll
                    for (int u = 0; u < 2; ++u) {
                        if (cc0 + u > cl)
                            break;
#pragma unroll
                        for (int c = 0; c < CH; c += 4) {
                            tot[c] += t4[u][c / 4].x;
                            tot[c + 1] += t4[u][c / 4].y;
                            tot[c + 2] += t4[u][c / 4].z;
                            tot[c + 3] += t4[u][c / 4].w;
                        }
                    }
                }
                if (nrow < p.N) {
#pragma unroll
                    for (int c = 0; c < CH; ++c)
                        if (h * HALF + c0 + c < p.M)
                            p.y[(size_t)(h * HALF + c0 + c) * p.N + nrow] =
                                __bfloat16_as_ushort(__float2bfloat16_rn(tot[c] * scale));
                }
            }
            if (lane == 0)
                atomicExch(&p.cnt[pnl * 8 + dw], 0u);
        };

        // retire unit k (its MMAs have been issued)
        auto complete = [&](int k, float s_k) {
            if constexpr (BITS == 4) {
                const int b = k & 1;
                if (!mbar_wait_warp(&accfull[b], (k >> 1) & 1)) {
                    ok = false;
                    return;
                }
                tc_fence_after();
                if constexpr (HALF == 8) {
                    float v[8];
                    tmem_load_cols<8>(tmem + tq + b * NT + h * HALF, v);
#pragma unroll
                    for (int c = 0; c < 8; ++c)
                        acc[c] = fmaf(s_k, v[c], acc[c]);
                } else {
#pragma unroll
                    for (int c0 = 0; c0 < HALF; c0 += 16) {
                        float v[16];
                        tmem_ld_32x32b_x16(tmem + tq + b * NT + h * HALF + c0, v);
                        tmem_wait_ld();
#pragma unroll
                        for (int c = 0; c < 16; ++c)
                            acc[c0 + c] = fmaf(s_k, v[c], acc[c0 + c]);
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0)
                    mbar_arrive(&accempty[b]);
                if (last_of_panel(k)) {
                    flush(panel_of(k), acc);
#pragma unroll
                    for (int c = 0; c < HALF; ++c)
                        acc[c] = 0.f;
                }
            } else {
                if (!last_of_panel(k))
                    return;
                const int pk = panel_of(k) - panel_of(0);
                const int b = pk & 1;
                if (!mbar_wait_warp(&accfull[b], (pk >> 1) & 1)) {
                    ok = false;
                    return;
                }
                tc_fence_after();
                float v[HALF];
                tmem_load_cols<HALF>(tmem + tq + b * NT + h * HALF, v);
                tc_fence_before();
                __syncwarp();
                if (lane == 0)
                    mbar_arrive(&accempty[b]);
                flush(panel_of(k), v);
            }
        };

        for (int i = 0; i < n && ok; ++i) {
            const int st = i % STAGES, use = i / STAGES;
            if (!mbar_wait_warp(&full[st], use & 1)) {
                ok = false;
                break;
            }
            uint4 w[TPR]; // INT4: tiles of row block j; INT8: chunks 4h .. 4h+3 of row r
#pragma unroll
            for (int tt = 0; tt < TPR; ++tt) {
                if constexpr (BITS == 8)
                    w[tt] = *reinterpret_cast<const uint4 *>(sW + st * WB + int8_chunk_in_block(r, 4 * h + tt));
                else
                    w[tt] = *reinterpret_cast<const uint4 *>(sW + st * WB + j * (TPR * kTileBytes) +
                                                             tt * kTileBytes + lane * 16);
            }
            uint32_t zlo = 0, zhi = 0;
            float s_mine = 0.f;
            if constexpr (BITS == 4) {
                const uint8_t *z8 = sSZ + st * SZB + 256;
                const int r0 = 16 * j + g, r1 = r0 + 8;
                const uint32_t z0 = (z8[r0 >> 1] >> (4 * (r0 & 1))) & 0xFu;
                const uint32_t z1 = (z8[r1 >> 1] >> (4 * (r1 & 1))) & 0xFu;
                zlo = 0x43004300u | z0 | (z0 << 16);
                zhi = 0x43004300u | z1 | (z1 << 16);
                s_mine = bf16_bits_to_float(reinterpret_cast<const uint16_t *>(sSZ + st * SZB)[r]);
            }
            __syncwarp();
            if (lane == 0)
                mbar_arrive(&ldempty[st]);
            if (use > 0 && !mbar_wait_warp(&aempty[st], (use - 1) & 1)) {
                ok = false;
                break;
            }
            tc_fence_after();
            if constexpr (BITS == 4) {
                const uint32_t ta = tmem + ((uint32_t)(32 * q + 16 * h) << 16) + A0 + st * 64;
#pragma unroll
                for (int tt = 0; tt < TPR; ++tt) {
                    uint32_t rr[16];
                    int4_tile_regs(w[tt], zlo, zhi, rr);
                    tmem_st_16x256b_x4(ta + tt * 32, rr);
                }
            } else {
                // row r, chunks 4h .. 4h+3 -> columns 32h .. 32h+31 of the stage
                const uint32_t ta = tmem + tq + A0 + st * 64 + 32 * h;
#pragma unroll
                for (int cp = 0; cp < 2; ++cp) {
                    uint32_t rr[16];
                    int8_chunks_regs(w[2 * cp], w[2 * cp + 1], rr);
                    tmem_st_32x32b_x16(ta + 16 * cp, rr);
                }
            }
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0)
                mbar_arrive(&afull[st]);
            if (i >= 1)
                complete(i - 1, s_prev);
            s_prev = s_mine;
        }
        if (ok && n >= 1)
            complete(n - 1, s_prev);
    }

    if (!ok)
        atomicExch(&g_gemm_sk_error, kErrTimeout);
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, TCOLS);
    }
}

template <int BITS, int NT>
static cudaError_t launch_gemm_sk_t(const LinearArgs &a, int ctas_per_sm, void *ws, int sm_count, cudaStream_t st)
{
    using C = GskCfg<BITS, NT>;
    constexpr size_t smem = gemm_sk_smem_bytes<BITS, NT>();
    static_assert(smem <= 227 * 1024, "shared memory per CTA");
    {
        const cudaError_t e = kernel_setup((const void *)gemm_sk_kernel<BITS, NT>, smem, 0, 0, nullptr);
        if (e != cudaSuccess)
            return e;
    }
    CUtensorMap map;
    if (!make_x_map<NT>(&map, a.x, a.M, a.K))
        return cudaErrorInvalidValue;
    const Shape sh{a.bits, a.K, a.N, a.group};
    GemmSkParams p;
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
    const int per_sm = (ctas_per_sm >= 1 && ctas_per_sm < C::kOcc) ? ctas_per_sm : C::kOcc;
    int G = per_sm * sm_count;
    if (G > kSkMaxCtas)
        G = kSkMaxCtas;
    if (G > p.U)
        G = p.U;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(G);
    cfg.blockDim = dim3(kGskThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, gemm_sk_kernel<BITS, NT>, map, p);
}

cudaError_t launch_gemm_sk(const LinearArgs &a, int ctas_per_sm, void *ws, int sm_count, cudaStream_t st)
{
    const int nt = a.M <= 16 ? 16 : a.M <= 32 ? 32 : a.M <= 64 ? 64 : 128;
    if (a.bits == 4) {
        switch (nt) {
        case 16: return launch_gemm_sk_t<4, 16>(a, ctas_per_sm, ws, sm_count, st);
        case 32: return launch_gemm_sk_t<4, 32>(a, ctas_per_sm, ws, sm_count, st);
        case 64: return launch_gemm_sk_t<4, 64>(a, ctas_per_sm, ws, sm_count, st);
        default: return launch_gemm_sk_t<4, 128>(a, ctas_per_sm, ws, sm_count, st);
        }
    }
    switch (nt) {
    case 16: return launch_gemm_sk_t<8, 16>(a, ctas_per_sm, ws, sm_count, st);
    case 32: return launch_gemm_sk_t<8, 32>(a, ctas_per_sm, ws, sm_count, st);
    case 64: return launch_gemm_sk_t<8, 64>(a, ctas_per_sm, ws, sm_count, st);
    default: return launch_gemm_sk_t<8, 128>(a, ctas_per_sm, ws, sm_count, st);
    }
}

cudaError_t read_gemm_sk_error(int *code, cudaStream_t st)
{
    int host = 0, zero = 0;
    cudaError_t e = cudaMemcpyFromSymbolAsync(&host, g_gemm_sk_error, sizeof(int), 0, cudaMemcpyDeviceToHost, st);
    if (e != cudaSuccess)
        return e;
    e = cudaMemcpyToSymbolAsync(g_gemm_sk_error, &zero, sizeof(int), 0, cudaMemcpyHostToDevice, st);
    if (e != cudaSuccess)
        return e;
    e = cudaStreamSynchronize(st);
    *code = host;
    return e;
}

} // namespace wq
