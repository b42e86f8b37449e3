// wq_gemm_i8.cu -- W8A16 on the integer tensor cores: tcgen05.mma kind::i8
// straight on the packed INT8 codes, no weight dequantization at all.
//
// The per-channel scale of W8A16 factors out of the k sum ("Per-channel
// W8A16 quantization", tileInfer README, Features table):
//     y[m][n] = s[n] * sum_k q[n][k] * x[m][k]
// so the sum over k can run on integers.  Every token row of x becomes
// integers X = round(x * 2^e_m), e_m chosen from the row's largest
// magnitude so that |X| < 2^22 (every element within 2^14 of the row's
// largest is exact; smaller ones are rounded to nearest, ties to even, at
// 2^-e_m), and X is written as three signed base-256 digits
//     X = d0 + 256 d1 + 65536 d2,   d0, d1 in [-128, 127], |d2| <= 64.
// The tensor cores multiply the weight codes (the A operand, 128 output
// channels) by the digit rows (the B operand, row 3m + i = digit i of token
// m) with int32 accumulators in tensor memory:
//     D[n][3m + i] = sum_k q[n][k] d_i[m][k]        exact for K <= 65536
// and the epilogue recombines y = s[n] 2^-e_m (D0 + 256 D1 + 65536 D2) in
// binary64 before the bf16 rounding.
//
// Why: the bf16-dequantizing kernels spend tens of instructions per 16
// bytes of weights, which caps them below HBM bandwidth at decode sizes.
// Here the packed block is already the tensor cores' canonical K-major
// 128-byte-swizzled layout (wq_layout.h): a 1-D bulk copy lands it where the
// MMA reads it, and the SM's threads never touch the weights.
//
// Work split: stream-K.  The (panel, k-block) units form one stream; CTA c of
// G (two per SM where two rings fit, for NR <= 48, else one) takes units
// [U*c/G, U*(c+1)/G).  Warp roles (192 threads):
//   warp 0     producer: per unit one 16 KB bulk copy of the weight block and
//              one of the unit's digit block (L2-resident) into a ring; the
//              first stages' weights are issued before the programmatic-launch
//              wait (weights never depend on the preceding kernel), digit
//              blocks only once the grid has written them.
//   warp 1     allocates tensor memory; one thread issues four
//              tcgen05.mma kind::i8 (K = 32 each) per unit into one of two
//              accumulator buffers (one panel segment per buffer).
//   warps 2-5  first the activations: every CTA computes the row maxima
//              (e_m) and writes 1/G of the digit blocks to the workspace,
//              then counts itself on a grid counter (release); the producer
//              waits for all G (acquire, bounded).  Then the epilogue, one
//              thread per output channel: write y when the CTA covered the
//              whole panel, else store int32 partials and take a ticket; the
//              last arriver for a panel's rows sums every contributor's
//              partial (integer sums: exact in any order) and writes y.
// The grid is one wave (G <= CTAs per SM x SMs), so every CTA becomes
// resident (a dependent kernel launches only after every CTA of this grid
// has started) and the grid counter wait always ends; the last CTA to exit
// resets it.  For small M (NR <= 48) two CTAs share an SM, each with its own
// ring and producer thread: twice the weight copies in flight per SM.
// Every wait is bounded (2 s); on a timeout the device error word is set and
// the CTA winds down.
#include <cstdint>

#include <cuda_bf16.h>

#include "wq_device.cuh"
#include "wq_imma.cuh"
#include "wq_internal.h"

namespace wq {

static __device__ int g_i8_error = 0;

struct I8Params {
    const uint16_t *x;
    int M, K, N, KB, U;
    const uint8_t *wq;
    const uint16_t *scales;
    uint16_t *y;
    uint8_t *xd;    // [KB][NR][128] digit blocks
    int32_t *part;  // [G][2 slots][NR][128 rows] int32
    uint32_t *cnt;  // [panels][4] tickets
    uint32_t *grid; // [2]: digit blocks written, CTAs exited
    unsigned long long *res; // [M] residual sums of the exactness guard
};

// Per digit-row count NR (the MMA's N): ring depth, tensor-memory columns and
// CTAs per SM.  Up to NR = 48 (M <= 16) the ring stays near 100 KB so two
// CTAs fit on an SM.
template <int NR>
struct I8Cfg {
    static constexpr int kAB = 16384;    // weight block
    static constexpr int kBB = NR * 128; // digit block
    static constexpr int kStageBytes = kAB + kBB;
    static constexpr int kOcc = NR <= 48 ? 2 : 1;
    static constexpr int kBudget = kOcc == 2 ? 100 * 1024 : 200 * 1024;
    static constexpr int kStagesRaw = kBudget / kStageBytes;
    static constexpr int kStages = kStagesRaw > 12 ? 12 : kStagesRaw;
    static constexpr int kTmemCols = 2 * NR <= 32 ? 32 : 2 * NR <= 64 ? 64 : 2 * NR <= 128 ? 128 : 2 * NR <= 256 ? 256 : 512;
    // epilogue columns per pass: whole tokens (3 columns each), a multiple of 8
    static constexpr int kColGroup = NR < 48 ? NR : 48;
    static_assert(NR % 16 == 0 && NR <= 256, "MMA N: multiple of 16, at most 256");
    static_assert(kStages >= 4, "ring depth");
};

constexpr int kI8Threads = 192;

template <int NR>
constexpr size_t i8_smem_bytes()
{
    // ring + barriers (full, empty per stage; accfull, accempty x 2) +
    // tensor-memory slot + row maxima / exponents + residual bounds
    return 1024 + (size_t)I8Cfg<NR>::kStages * I8Cfg<NR>::kStageBytes + (2 * I8Cfg<NR>::kStages + 4) * 8 + 16 +
           2 * kI8MaxM * 4 + kI8MaxM * 8 + (size_t)2 * (2 * kI8MaxCtas + 1) * 4;
}

template <int NR>
__global__ void __launch_bounds__(kI8Threads, I8Cfg<NR>::kOcc) gemm_i8_kernel(const I8Params p)
{
    using C = I8Cfg<NR>;
    constexpr int STAGES = C::kStages;
    constexpr int TCOLS = C::kTmemCols;
    constexpr int CG = C::kColGroup;

    extern __shared__ uint8_t smem_raw[];
    uint8_t *ring = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *full = reinterpret_cast<uint64_t *>(ring + STAGES * C::kStageBytes);
    uint64_t *empty = full + STAGES;
    uint64_t *accfull = empty + STAGES; // [2]
    uint64_t *accempty = accfull + 2;   // [2]
    uint32_t *s_tmem = reinterpret_cast<uint32_t *>(accempty + 2);
    uint32_t *s_amax = s_tmem + 4;                        // [kI8MaxM] row maxima (bf16 magnitude bits)
    int *s_e = reinterpret_cast<int *>(s_amax + kI8MaxM); // [kI8MaxM] exponents e_m
    double *s_rb = reinterpret_cast<double *>(s_e + kI8MaxM); // [kI8MaxM] residual bounds (8-byte aligned)
    int *s_start = reinterpret_cast<int *>(s_rb + kI8MaxM);    // [G + 1] stream-K cuts
    int *s_first = s_start + 2 * kI8MaxCtas + 1;              // [G + 1] first panel of each range

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int G = gridDim.x, c = blockIdx.x;
    const long long U = p.U;
    const int KB = p.KB, M = p.M;
    const int u0 = sk_start(U, G, c), u1 = sk_start(U, G, c + 1);
    const int n = u1 - u0;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
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
        if (lane == 0) {
            const uint64_t pol_w = policy_evict_first(), pol_x = policy_evict_last();
            auto issue_w = [&](int i, int st) {
                mbar_arrive_expect_tx(&full[st], C::kStageBytes);
                bulk_g2s(ring + st * C::kStageBytes, p.wq + (size_t)(u0 + i) * C::kAB, C::kAB, &full[st], pol_w);
            };
            int xkb = u0 % KB; // k-block of the next digit block issued, kept without dividing
            auto issue_x = [&](int i, int st) {
                (void)i;
                bulk_g2s(ring + st * C::kStageBytes + C::kAB, p.xd + (size_t)xkb * C::kBB, C::kBB, &full[st], pol_x);
                xkb = xkb + 1 == KB ? 0 : xkb + 1;
            };
            const int pre = n < STAGES ? n : STAGES;
            for (int i = 0; i < pre; ++i) // weights never depend on the preceding kernel
                issue_w(i, i);
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
                issue_x(i, i);
            for (int i = pre; i < n && ok; ++i) {
                const int st = i % STAGES, use = i / STAGES;
                if (!mbar_wait(&empty[st], (use - 1) & 1)) {
                    ok = false;
                    break;
                }
                issue_w(i, st);
                issue_x(i, st);
            }
        }
        __syncwarp();
        pdl_wait();
        pdl_launch_dependents();
    } else if (warp == 1) {
        if (lane == 0) {
            constexpr uint32_t idesc = umma_idesc_s8(NR);
            int seg = -1, kb = u0 % KB; // k-block of unit i, kept without dividing
            for (int i = 0; i < n; ++i, kb = kb + 1 == KB ? 0 : kb + 1) {
                const bool first = (i == 0 || kb == 0), last = (i == n - 1 || kb == KB - 1);
                const int st = i % STAGES, use = i / STAGES;
                if (first) {
                    ++seg;
                    if (seg >= 2 && !mbar_wait(&accempty[seg & 1], ((seg >> 1) - 1) & 1)) {
                        ok = false;
                        break;
                    }
                }
                if (!mbar_wait(&full[st], use & 1)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t sa = smem_u32(ring + st * C::kStageBytes), sb = sa + C::kAB;
                const uint32_t d = tmem + (uint32_t)((seg & 1) * NR);
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    umma_ss_i8(d, smem_desc_sw128(sa + 32 * kk), smem_desc_sw128(sb + 32 * kk), idesc,
                               (first && kk == 0) ? 0u : 1u);
                umma_commit(&empty[st]);
                if (last)
                    umma_commit(&accfull[seg & 1]);
            }
        }
        __syncwarp();
        pdl_wait();
        pdl_launch_dependents();
    } else {
        pdl_wait(); // x, y and the workspace may come from / be in use by the preceding kernel
        const int et = threadIdx.x - 64; // 0..127
        const int quad = warp & 3;
        const int K = p.K;
        // ---------------- activations: row maxima, then 1/G of the digit blocks ----------------
        imma_digit_phase<NR>(p.x, M, K, KB, c, G, et, p.xd, s_amax, s_e, p.grid, p.res);
        ok = imma_residual_bounds(M, G, et, p.grid, p.res, s_e, s_rb) && ok;
        // ---------------- epilogue: one thread per output channel ----------------
        const int row = 32 * quad + lane;
        const uint32_t tq = (uint32_t)(32 * quad) << 16;
        int seg = 0;
        for (int pnl = n > 0 ? u0 / KB : 0; n > 0 && pnl <= (u1 - 1) / KB && ok; ++pnl, ++seg) {
            const int lo = max(u0, pnl * KB), hi = min(u1, (pnl + 1) * KB);
            const bool whole = (lo == pnl * KB && hi == (pnl + 1) * KB);
            const int b = seg & 1;
            const int cf = sk.owner(pnl * KB, G), cl = sk.owner((pnl + 1) * KB - 1, G);
            // A split panel whose other contributors have all taken their tickets
            // (typically the last segment of the range: its partner did its part
            // first): this warp is the last arriver.  It reads their partials now,
            // while its own MMAs are still running, and takes no ticket.
            bool early_last = false;
            int32_t pre[CG];
#pragma unroll
            for (int j = 0; j < CG; ++j)
                pre[j] = 0;
            if (!whole && 3 * M <= CG) {
                uint32_t seen = 0;
                if (lane == 0)
                    seen = ld_acquire_gpu(&p.cnt[pnl * 4 + quad]);
                early_last = __shfl_sync(0xffffffffu, seen, 0) == (uint32_t)(cl - cf);
                if (early_last) {
                    __syncwarp(); // lane 0's acquire orders every lane's reads below
                    for (int cc = cf; cc <= cl; ++cc) {
                        if (cc == c)
                            continue;
                        const int sl = (pnl == sk.first[cc]) ? 0 : 1;
                        const int32_t *src = p.part + (size_t)(cc * 2 + sl) * NR * 128 + row;
                        int32_t v[CG];
#pragma unroll
                        for (int j = 0; j < CG; ++j)
                            v[j] = (j < 3 * M) ? __ldcg(src + (size_t)j * 128) : 0;
#pragma unroll
                        for (int j = 0; j < CG; ++j)
                            pre[j] += v[j];
                    }
                }
            }
            if (!mbar_wait_warp(&accfull[b], (seg >> 1) & 1)) {
                ok = false;
                break;
            }
            tc_fence_after();
            const int nrow = pnl * kPanelRows + row;
            const double s_n = nrow < p.N ? (double)bf16_bits_to_float(p.scales[nrow]) : 0.0;
            const int slot = (pnl == sk.first[c]) ? 0 : 1;
            int32_t *mine = p.part + (size_t)(c * 2 + slot) * NR * 128;
#pragma unroll
            for (int c0 = 0; c0 < NR; c0 += CG) {
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
                if (c0 + CG >= NR) { // the accumulator buffer is free for the MMA again
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0)
                        mbar_arrive(&accempty[b]);
                }
                if (whole || early_last) {
                    if (early_last) { // one pass: 3M <= CG
#pragma unroll
                        for (int j = 0; j < CG; ++j)
                            v[j] += pre[j];
                    }
#pragma unroll
                    for (int t = 0; t < CG / 3; ++t) {
                        const int m = c0 / 3 + t; // the same across the warp
                        if (m < M)
                            imma_emit_rows<8>(p.x, p.wq, p.scales, nullptr, p.y, K, KB, p.N, pnl * kPanelRows + 32 * quad,
                                              m, i8_value(v[3 * t], v[3 * t + 1], v[3 * t + 2], s_n * pow2_of(-s_e[m])),
                                              128.0 * s_n * s_rb[m], lane);
                    }
                } else {
#pragma unroll
                    for (int cc = 0; cc < CG; ++cc)
                        if (c0 + cc < 3 * M)
                            mine[(size_t)(c0 + cc) * 128 + row] = v[cc];
                }
            }
            if (whole)
                continue;
            if (early_last) { // every other contributor is done: reset the ticket for the next call
                if (lane == 0)
                    atomicExch(&p.cnt[pnl * 4 + quad], 0u);
                continue;
            }
            // Split panel: every contributor's warp takes a ticket for its 32
            // rows (one acquire-release atomic after a warp barrier); the last
            // one sums all partials (exact integers) and writes y.
            __syncwarp();
            uint32_t ticket = 0;
            if (lane == 0)
                ticket = ticket_take_acq_rel(&p.cnt[pnl * 4 + quad]);
            ticket = __shfl_sync(0xffffffffu, ticket, 0);
            if (ticket != (uint32_t)(cl - cf))
                continue;
            __syncwarp(); // lane 0's acquire orders every lane's reads below
            for (int c0 = 0; c0 < 3 * M; c0 += CG) {
                int32_t tot[CG];
#pragma unroll
                for (int j = 0; j < CG; ++j)
                    tot[j] = 0;
                for (int cc = cf; cc <= cl; ++cc) { // all CG loads of a contributor in flight together
                    const int sl = (pnl == sk.first[cc]) ? 0 : 1;
                    const int32_t *src = p.part + (size_t)(cc * 2 + sl) * NR * 128 + row;
                    int32_t v[CG];
#pragma unroll
                    for (int j = 0; j < CG; ++j)
                        v[j] = (c0 + j < 3 * M) ? __ldcg(src + (size_t)(c0 + j) * 128) : 0;
#pragma unroll
                    for (int j = 0; j < CG; ++j)
                        tot[j] += v[j];
                }
#pragma unroll
                for (int t = 0; t < CG / 3; ++t) {
                    const int m = c0 / 3 + t; // the same across the warp
                    if (m < M)
                        imma_emit_rows<8>(p.x, p.wq, p.scales, nullptr, p.y, K, KB, p.N, pnl * kPanelRows + 32 * quad, m,
                                          i8_value(tot[3 * t], tot[3 * t + 1], tot[3 * t + 2], s_n * pow2_of(-s_e[m])),
                                          128.0 * s_n * s_rb[m], lane);
                }
            }
            if (lane == 0)
                atomicExch(&p.cnt[pnl * 4 + quad], 0u);
        }
        pdl_launch_dependents();
    }

    if (!ok)
        atomicExch(&g_i8_error, kErrTimeout);
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
int i8_digit_rows(int M) { return M <= 5 ? 16 : M <= 10 ? 32 : M <= 16 ? 48 : M <= 32 ? 96 : 192; }

size_t ws_bytes_gemm_i8(int M, int K, int N)
{
    if (M < 1 || M > kI8MaxM || K < 1)
        return 0;
    const int NR = i8_digit_rows(M);
    const size_t KB = (size_t)(K + kBlockK - 1) / kBlockK;
    const size_t ctas = (size_t)(NR <= 48 ? 2 : 1) * kI8MaxCtas; // the grid: CTAs per SM x at most kI8MaxCtas SMs
    return ws_counter_bytes() + KB * NR * 128 + ctas * 2 * NR * 128 * sizeof(int32_t);
}

template <int NR>
static cudaError_t launch_i8_t(const LinearArgs &a, void *ws, int sm_count, cudaStream_t st)
{
    constexpr size_t smem = i8_smem_bytes<NR>();
    static_assert(smem <= 227 * 1024, "shared memory per CTA");
    static_assert(I8Cfg<NR>::kOcc == 1 || 2 * (smem + 1024) <= 228 * 1024, "two CTAs per SM");
    {
        const cudaError_t e = kernel_setup((const void *)gemm_i8_kernel<NR>, smem, 0, 0, nullptr);
        if (e != cudaSuccess)
            return e;
    }
    const Shape sh{8, a.K, a.N, 0};
    I8Params p;
    p.x = a.x;
    p.M = a.M;
    p.K = a.K;
    p.N = a.N;
    p.KB = sh.kblocks();
    p.U = sh.panels() * p.KB;
    p.wq = (const uint8_t *)a.wq;
    p.scales = (const uint16_t *)a.scales;
    p.y = a.y;
    p.cnt = (uint32_t *)ws;
    p.grid = p.cnt + ws_grid_counter();
    p.res = reinterpret_cast<unsigned long long *>(p.cnt + ws_res_counter());
    p.xd = (uint8_t *)ws + ws_counter_bytes();
    p.part = (int32_t *)(p.xd + (size_t)p.KB * NR * 128);
    // two CTAs per SM where they fit: twice the weight copies in flight per
    // SM (one producer thread and its ring per CTA)
    constexpr int occ = I8Cfg<NR>::kOcc;
    static_assert(occ == (NR <= 48 ? 2 : 1), "workspace sizing (ws_bytes_gemm_i8) follows the occupancy");
    int G = occ * (sm_count < kI8MaxCtas ? sm_count : kI8MaxCtas);
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
    cfg.blockDim = dim3(kI8Threads);
    cfg.dynamicSmemBytes = smem;
    return cudaLaunchKernelEx(&cfg, gemm_i8_kernel<NR>, p);
}

cudaError_t launch_gemm_i8(const LinearArgs &a, void *ws, int sm_count, cudaStream_t st)
{
    switch (i8_digit_rows(a.M)) {
    case 16: return launch_i8_t<16>(a, ws, sm_count, st);
    case 32: return launch_i8_t<32>(a, ws, sm_count, st);
    case 48: return launch_i8_t<48>(a, ws, sm_count, st);
    case 96: return launch_i8_t<96>(a, ws, sm_count, st);
    default: return launch_i8_t<192>(a, ws, sm_count, st);
    }
}

cudaError_t read_gemm_i8_error(int *code, cudaStream_t st)
{
    int host = 0, zero = 0;
    cudaError_t e = cudaMemcpyFromSymbolAsync(&host, g_i8_error, sizeof(int), 0, cudaMemcpyDeviceToHost, st);
    if (e != cudaSuccess)
        return e;
    e = cudaMemcpyToSymbolAsync(g_i8_error, &zero, sizeof(int), 0, cudaMemcpyHostToDevice, st);
    if (e != cudaSuccess)
        return e;
    e = cudaStreamSynchronize(st);
    *code = host;
    return e;
}

} // namespace wq
