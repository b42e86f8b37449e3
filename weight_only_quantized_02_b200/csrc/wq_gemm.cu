// wq_gemm.cu -- small-M (8..128 tokens) split-K GEMM on tcgen05 tensor cores.
//
// y^T = dequant(W) . x^T: the weight rows are the MMA's M side (128 rows per
// CTA), the tokens its N side (NT = 16/32/64/128), so decode-sized batches
// still fill a 128-row tensor-core tile.  One CTA owns a 128-row panel and a
// K range (split-K over 128-k blocks; the split-factor grid and its
// trade-off are those of the split_k auto-tune in Mit han lab Llm awq Kernel
// Selection Thresholds, The Insight).
//
// Warp roles (192 threads):
//   warp 0     TMA producer: per 128-k block, the x tile (2-D tensor map,
//              128-byte swizzle) and the packed weight block (+ INT4 scales
//              and zeros) as 1-D bulk copies into a STAGES-deep ring.
//   warp 1     allocates tensor memory; one thread issues tcgen05.mma with
//              the dequantized weights as the A operand *from tensor memory*
//              and x as the B operand from shared memory; fp32 accumulators
//              in tensor memory.
//   warps 2-5  dequantize the block to exact integers in bf16 (INT4: q - z,
//              INT8: q) and write it to tensor memory: INT4 with tcgen05.st
//              16x256b (the packed tile is that store's register layout),
//              INT8 one row per thread with 32x32b (the swizzled block gives
//              each thread its row's chunks without bank conflicts).  The weights are never rounded: INT8's per-channel
//              scale is applied in the epilogue; INT4 accumulates each
//              128-k group into one of two tensor-memory buffers and these
//              warps fold s[row][g] * D_g into fp32 register totals one group
//              behind the MMA (the same arithmetic as the GEMV).  Then they
//              run the epilogue.
// Epilogue: split == 1 stores bf16 y.  split > 1 stores fp32 partials; the
// last CTA of a panel to arrive (atomic ticket, no waiting) sums all partials
// in split order 0..S-1, so each (variant, split) is run-to-run deterministic,
// and resets the ticket to zero.
//
// Every mbarrier wait is bounded (2 s); a wait that gives up records
// kErrTimeout in the device error word and the CTA winds down.
#include <cstdint>
#include <cstdio>

#include <cudaTypedefs.h>

#include "wq_device.cuh"
#include "wq_gemm_common.cuh"
#include "wq_internal.h"

namespace wq {

static __device__ int g_gemm_error = 0;

struct GemmParams {
    int M, K, N, KB, S;
    const uint8_t *wq;
    const uint16_t *scales;
    const uint8_t *zeros;
    uint16_t *y;
    float *part;   // [S][M][N] fp32 partials (S > 1)
    uint32_t *cnt; // [panels] tickets (S > 1)
};

template <int BITS>
struct GemmBits {
    static constexpr int kWBytes = BITS == 4 ? 8192 : 16384; // packed block per stage
    static constexpr int kSZBytes = BITS == 4 ? 512 : 0;     // scales (256) + zeros (64), padded
    static constexpr int kSZTx = BITS == 4 ? 320 : 0;
    static constexpr int kTilesPerRb = BITS == 4 ? 2 : 4;
};

// Tensor-memory plan per (bits, token tile).  INT4 keeps two group
// accumulators (double-buffered, NT columns each) so the MMA of group g+1
// overlaps the fp32 rescale of group g; INT8 keeps one accumulator for the
// whole K range.  The A ring (64 columns = 128 k of bf16 per stage) follows.
template <int BITS, int NT>
struct GemmTile {
    static constexpr int kAccBufs = BITS == 4 ? 2 : 1;
    static constexpr int kTmemCols = NT == 128 ? 512 : 256;
    static constexpr int kA0 = (kAccBufs * NT + 63) / 64 * 64 < 64 ? 64 : (kAccBufs * NT + 63) / 64 * 64;
    static constexpr int kTmemStages = (kTmemCols - kA0) / 64;
    static constexpr int kSmemStageBytes = NT * 256 + GemmBits<BITS>::kWBytes + GemmBits<BITS>::kSZBytes;
    static constexpr int kSmemStages = (200 * 1024) / kSmemStageBytes;
    static constexpr int kStagesRaw = kTmemStages < kSmemStages ? kTmemStages : kSmemStages;
    static constexpr int kStages = kStagesRaw > 4 ? 4 : kStagesRaw;
    static constexpr int kMinBlocks = kTmemCols == 512 ? 1 : 2;
    static_assert(kStages >= 2, "pipeline needs two stages");
    static_assert(kA0 + 64 * kStages <= kTmemCols, "tensor memory budget");
};

template <int BITS, int NT>
constexpr size_t gemm_smem_bytes()
{
    return 1024 + (size_t)GemmTile<BITS, NT>::kStages * GemmTile<BITS, NT>::kSmemStageBytes +
           (4 * GemmTile<BITS, NT>::kStages + 5) * 8 + 16;
}

// Stores one output row's NT values (token m = column) as y, or as split-K
// partials followed by the last-arriver reduction.  Runs on the 128
// dequant/epilogue threads (named barrier 1).
template <int NT>
__device__ __forceinline__ void gemm_store(const GemmParams &p, int panel, int split, int n, bool nvalid,
                                           float scale, int warp, int lane, uint32_t *s_ticket,
                                           const float (&v)[NT])
{
    if (p.S == 1) {
        if (nvalid) {
#pragma unroll
            for (int m = 0; m < NT; ++m)
                if (m < p.M)
                    p.y[(size_t)m * p.N + n] = __bfloat16_as_ushort(__float2bfloat16_rn(v[m] * scale));
        }
        return;
    }
    if (nvalid) {
#pragma unroll
        for (int m = 0; m < NT; ++m)
            if (m < p.M)
                p.part[((size_t)split * p.M + m) * p.N + n] = v[m];
    }
    __threadfence();
    named_barrier_sync(1, 128);
    if (warp == 2 && lane == 0)
        *s_ticket = ticket_take(&p.cnt[panel]);
    named_barrier_sync(1, 128);
    if (*s_ticket == (uint32_t)(p.S - 1)) {
        __threadfence();
        if (nvalid) {
            for (int m = 0; m < p.M; ++m) {
                float sum = 0.f;
                for (int s = 0; s < p.S; ++s)
                    sum += __ldcg(&p.part[((size_t)s * p.M + m) * p.N + n]);
                p.y[(size_t)m * p.N + n] = __bfloat16_as_ushort(__float2bfloat16_rn(sum * scale));
            }
        }
        if (warp == 2 && lane == 0)
            atomicExch(&p.cnt[panel], 0u);
    }
}

template <int BITS, int NT>
__global__ void __launch_bounds__(192, GemmTile<BITS, NT>::kMinBlocks)
    gemm_kernel(const __grid_constant__ CUtensorMap tmx, const GemmParams p)
{
    using T = GemmTile<BITS, NT>;
    constexpr int STAGES = T::kStages;
    constexpr int TCOLS = T::kTmemCols;
    constexpr int A0 = T::kA0;
    constexpr int XB = NT * 256;
    constexpr int WB = GemmBits<BITS>::kWBytes;
    constexpr int SZB = GemmBits<BITS>::kSZBytes;
    constexpr int TPR = GemmBits<BITS>::kTilesPerRb;

    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sX = smem;
    uint8_t *sW = sX + STAGES * XB;
    uint8_t *sSZ = sW + STAGES * WB;
    uint64_t *bars = reinterpret_cast<uint64_t *>(sSZ + STAGES * SZB);
    uint64_t *full = bars, *ldempty = bars + STAGES, *afull = bars + 2 * STAGES, *aempty = bars + 3 * STAGES;
    uint64_t *accfull = bars + 4 * STAGES;      // [2]
    uint64_t *accempty = bars + 4 * STAGES + 2; // [2]
    uint32_t *s_misc = reinterpret_cast<uint32_t *>(bars + 4 * STAGES + 4);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int panel = blockIdx.x, split = blockIdx.y;
    const int kb0 = (int)((long long)p.KB * split / p.S);
    const int kb1 = (int)((long long)p.KB * (split + 1) / p.S);
    const int nk = kb1 - kb0;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&ldempty[s], 1 + 4);
            mbar_init(&afull[s], 4);
            mbar_init(&aempty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&accfull[b], 1);
            mbar_init(&accempty[b], 4);
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

    if (warp == 0) {
        if (lane == 0) {
            const uint64_t pol_w = policy_evict_first(), pol_x = policy_evict_last();
            for (int i = 0; i < nk; ++i) {
                const int st = i % STAGES, use = i / STAGES;
                if (use > 0 && !mbar_wait(&ldempty[st], (use - 1) & 1)) {
                    ok = false;
                    break;
                }
                const int kb = kb0 + i;
                const size_t blk = (size_t)panel * p.KB + kb;
                mbar_arrive_expect_tx(&full[st], XB + WB + GemmBits<BITS>::kSZTx);
                tma_load_2d(sX + st * XB, &tmx, kb * kBlockK, 0, &full[st], pol_x);
                tma_load_2d(sX + st * XB + NT * 128, &tmx, kb * kBlockK + 64, 0, &full[st], pol_x);
                bulk_g2s(sW + st * WB, p.wq + blk * WB, WB, &full[st], pol_w);
                if constexpr (BITS == 4) {
                    bulk_g2s(sSZ + st * SZB, p.scales + blk * kPanelRows, 256, &full[st], pol_w);
                    bulk_g2s(sSZ + st * SZB + 256, p.zeros + blk * 64, 64, &full[st], pol_w);
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            constexpr uint32_t idesc = umma_idesc_bf16(NT);
            for (int i = 0; i < nk; ++i) {
                const int st = i % STAGES, use = i / STAGES;
                if (!mbar_wait(&afull[st], use & 1) || !mbar_wait(&full[st], use & 1)) {
                    ok = false;
                    break;
                }
                uint32_t dcol = 0;
                if constexpr (BITS == 4) {
                    const int b = i & 1;
                    if (i >= 2 && !mbar_wait(&accempty[b], ((i >> 1) - 1) & 1)) {
                        ok = false;
                        break;
                    }
                    dcol = b * NT;
                }
                tc_fence_after();
                const uint32_t xs = smem_u32(sX + st * XB);
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint64_t bdesc = smem_desc_sw128(xs + (kk >> 2) * (NT * 128) + (kk & 3) * 32);
                    const uint32_t acc = BITS == 4 ? (kk > 0 ? 1u : 0u) : ((i > 0 || kk > 0) ? 1u : 0u);
                    umma_ts(tmem + dcol, tmem + A0 + st * 64 + kk * 8, bdesc, idesc, acc);
                }
                umma_commit(&aempty[st]);
                umma_commit(&ldempty[st]);
                if constexpr (BITS == 4)
                    umma_commit(&accfull[i & 1]);
            }
            if constexpr (BITS == 8)
                umma_commit(&accfull[0]);
        }
    } else {
        // ---------------- dequant / rescale / epilogue warps ----------------
        const int quad = warp & 3; // tensor-memory lane quadrant this warp may access
        const int g = lane >> 2;
        const int row = 32 * quad + lane; // this thread's output row in the panel
        const uint32_t tlane = (uint32_t)(32 * quad) << 16;
        float acc[NT]; // INT4: fp32 totals of this row, one per token
#pragma unroll
        for (int c = 0; c < NT; ++c)
            acc[c] = 0.f;
        float s_prev = 0.f;

        // fold group j's accumulator into the fp32 totals: acc += s_row * D_j
        auto rescale = [&](int j, float s) {
            const int b = j & 1;
            if (!mbar_wait_warp(&accfull[b], (j >> 1) & 1)) {
                ok = false;
                return;
            }
            tc_fence_after();
#pragma unroll
            for (int c0 = 0; c0 < NT; c0 += 16) {
                float v[16];
                tmem_ld_32x32b_x16(tmem + tlane + b * NT + c0, v);
                tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < 16; ++e)
                    acc[c0 + e] = fmaf(s, v[e], acc[c0 + e]);
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0)
                mbar_arrive(&accempty[b]);
        };

        for (int i = 0; i < nk && ok; ++i) {
            const int st = i % STAGES, use = i / STAGES;
            if (!mbar_wait_warp(&full[st], use & 1)) {
                ok = false;
                break;
            }
            uint4 w[2][TPR]; // INT4: tiles of row blocks 2*quad + jj; INT8: chunk 4*jj + tt of this thread's row
            uint32_t zz[2][2];
            float s_mine = 0.f;
#pragma unroll
            for (int jj = 0; jj < 2; ++jj) {
                const int j = 2 * quad + jj;
#pragma unroll
                for (int tt = 0; tt < TPR; ++tt) {
                    if constexpr (BITS == 8)
                        w[jj][tt] = *reinterpret_cast<const uint4 *>(sW + st * WB + int8_chunk_in_block(row, 4 * jj + tt));
                    else
                        w[jj][tt] = *reinterpret_cast<const uint4 *>(sW + st * WB + j * (TPR * kTileBytes) +
                                                                     tt * kTileBytes + lane * 16);
                }
                if constexpr (BITS == 4) {
                    const uint8_t *z8 = sSZ + st * SZB + 256;
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        const int r = 16 * j + g + 8 * h;
                        const uint32_t z = (z8[r >> 1] >> (4 * (r & 1))) & 0xFu;
                        zz[jj][h] = 0x43004300u | z | (z << 16);
                    }
                }
            }
            if constexpr (BITS == 4)
                s_mine = bf16_bits_to_float(reinterpret_cast<const uint16_t *>(sSZ + st * SZB)[row]);
            __syncwarp();
            if (lane == 0)
                mbar_arrive(&ldempty[st]);
            if (use > 0 && !mbar_wait_warp(&aempty[st], (use - 1) & 1)) {
                ok = false;
                break;
            }
            tc_fence_after();
            if constexpr (BITS == 4) {
#pragma unroll
                for (int jj = 0; jj < 2; ++jj) {
                    const uint32_t ta = tmem + ((uint32_t)(32 * quad + 16 * jj) << 16) + A0 + st * 64;
#pragma unroll
                    for (int tt = 0; tt < TPR; ++tt) {
                        uint32_t r[16];
                        int4_tile_regs(w[jj][tt], zz[jj][0], zz[jj][1], r);
                        tmem_st_16x256b_x4(ta + tt * 32, r);
                    }
                }
            } else {
                // this thread's row, chunks 0..7 -> columns 8c .. 8c+7 of the stage
                const uint32_t ta = tmem + tlane + A0 + st * 64;
#pragma unroll
                for (int cp = 0; cp < 4; ++cp) {
                    uint32_t r[16];
                    int8_chunks_regs(w[cp >> 1][2 * (cp & 1)], w[cp >> 1][2 * (cp & 1) + 1], r);
                    tmem_st_32x32b_x16(ta + 16 * cp, r);
                }
            }
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0)
                mbar_arrive(&afull[st]);
            if constexpr (BITS == 4) {
                if (i >= 1)
                    rescale(i - 1, s_prev);
                s_prev = s_mine;
            }
        }
        if constexpr (BITS == 4) {
            if (ok && nk >= 1)
                rescale(nk - 1, s_prev);
        }

        // ---------------- epilogue ----------------
        const int n = panel * kPanelRows + row;
        const bool nvalid = n < p.N;
        if constexpr (BITS == 4) {
            gemm_store<NT>(p, panel, split, n, nvalid, 1.f, warp, lane, &s_misc[1], acc);
        } else {
            if (!mbar_wait_warp(&accfull[0], 0))
                ok = false;
            tc_fence_after();
            const float scale = nvalid ? bf16_bits_to_float(p.scales[n]) : 0.f;
            // stage this row's NT accumulators through registers 16 columns at a time
            float v[NT];
#pragma unroll
            for (int c0 = 0; c0 < NT; c0 += 16) {
                float t[16];
                tmem_ld_32x32b_x16(tmem + tlane + c0, t);
                tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < 16; ++e)
                    v[c0 + e] = t[e];
            }
            gemm_store<NT>(p, panel, split, n, nvalid, scale, warp, lane, &s_misc[1], v);
        }
    }

    if (!ok)
        atomicExch(&g_gemm_error, kErrTimeout);
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, TCOLS);
    }
}

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------
template <int BITS, int NT>
static cudaError_t launch_gemm_t(const LinearArgs &a, int S, void *ws, cudaStream_t st)
{
    constexpr size_t smem = gemm_smem_bytes<BITS, NT>();
    static_assert(smem <= 227 * 1024, "shared memory per CTA");
    {
        const cudaError_t e = kernel_setup((const void *)gemm_kernel<BITS, NT>, smem, 0, 0, nullptr);
        if (e != cudaSuccess)
            return e;
    }
    CUtensorMap map;
    if (!make_x_map<NT>(&map, a.x, a.M, a.K))
        return cudaErrorInvalidValue;
    const Shape sh{a.bits, a.K, a.N, a.group};
    GemmParams p;
    p.M = a.M;
    p.K = a.K;
    p.N = a.N;
    p.KB = sh.kblocks();
    p.S = S;
    p.wq = (const uint8_t *)a.wq;
    p.scales = (const uint16_t *)a.scales;
    p.zeros = (const uint8_t *)a.zeros;
    p.y = a.y;
    p.cnt = (uint32_t *)ws;
    p.part = ws ? (float *)((uint8_t *)ws + ws_counter_bytes()) : nullptr;
    dim3 grid(sh.panels(), S);
    gemm_kernel<BITS, NT><<<grid, 192, smem, st>>>(map, p);
    return cudaGetLastError();
}

cudaError_t launch_gemm(const LinearArgs &a, int split, void *ws, int sm_count, cudaStream_t st)
{
    (void)sm_count;
    const int nt = a.M <= 16 ? 16 : a.M <= 32 ? 32 : a.M <= 64 ? 64 : 128;
    if (a.bits == 4) {
        switch (nt) {
        case 16: return launch_gemm_t<4, 16>(a, split, ws, st);
        case 32: return launch_gemm_t<4, 32>(a, split, ws, st);
        case 64: return launch_gemm_t<4, 64>(a, split, ws, st);
        default: return launch_gemm_t<4, 128>(a, split, ws, st);
        }
    }
    switch (nt) {
    case 16: return launch_gemm_t<8, 16>(a, split, ws, st);
    case 32: return launch_gemm_t<8, 32>(a, split, ws, st);
    case 64: return launch_gemm_t<8, 64>(a, split, ws, st);
    default: return launch_gemm_t<8, 128>(a, split, ws, st);
    }
}

// One thread waits, through the kernels' bounded wait, on an mbarrier that
// nothing arrives on: the wait gives up after limit_ns, the timeout is
// recorded in the device error word exactly as a kernel records it, and the
// kernel returns.  Failure detection under test, without a fault or a hang.
__global__ void wait_selftest_kernel(uint64_t limit_ns)
{
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0 && !mbar_wait_for(&bar, 0, limit_ns))
        atomicExch(&g_gemm_error, kErrTimeout);
}

cudaError_t launch_wait_selftest(uint64_t limit_ns, cudaStream_t st)
{
    wait_selftest_kernel<<<1, 32, 0, st>>>(limit_ns);
    return cudaGetLastError();
}

cudaError_t read_device_error(int *code, cudaStream_t st)
{
    int host = 0, zero = 0;
    cudaError_t e = cudaMemcpyFromSymbolAsync(&host, g_gemm_error, sizeof(int), 0, cudaMemcpyDeviceToHost, st);
    if (e != cudaSuccess)
        return e;
    e = cudaMemcpyToSymbolAsync(g_gemm_error, &zero, sizeof(int), 0, cudaMemcpyHostToDevice, st);
    if (e != cudaSuccess)
        return e;
    e = cudaStreamSynchronize(st);
    *code = host;
    return e;
}

} // namespace wq
