// wq_gemm_i8.cu -- W8A16 on the integer tensor cores: tcgen05.mma kind::i8
// straight on the packed INT8 codes, no dequantization instructions at all.
//
// The per-channel scale of W8A16 factors out of the k sum ("Per-channel
// W8A16 quantization", tileInfer README, Features table):
//     y[m][n] = s[n] * sum_k q[n][k] * x[m][k]
// so the sum over k can run on integers.  A small pre-pass turns every
// token row of x into integers X = round(x * 2^e_m), with e_m chosen from
// the row's largest magnitude so that |X| < 2^22 (every element within 2^14
// of the row's largest is exact; smaller ones are rounded to nearest, ties
// to even, at 2^-e_m), and writes X as three signed base-256 digits
//     X = d0 + 256 d1 + 65536 d2,   d0, d1 in [-128, 127], |d2| <= 64.
// The tensor cores multiply the weight codes (the A operand, 128 output
// channels) by the digit rows (the B operand, column 3m + i = digit i of
// token m) with int32 accumulators in tensor memory:
//     D[n][3m + i] = sum_k q[n][k] d_i[m][k]        exact, K <= 65536
// and the epilogue recombines y = s[n] 2^-e_m (D0 + 256 D1 + 65536 D2) in
// binary64 before the bf16 rounding.
//
// Why: on B200 the bf16-dequantizing kernels spend tens of instructions per
// 16 bytes of weights, which caps them well below HBM bandwidth at decode
// sizes.  Here the packed block is already the tensor cores' canonical
// K-major 128-byte-swizzled layout (wq_layout.h), so a 1-D bulk copy lands it
// where the MMA reads it and the SM's threads only issue copies and MMAs.
//
// Work split: stream-K.  The (panel, k-block) units form one stream; CTA c of
// G (one per SM) takes units [U*c/G, U*(c+1)/G).  Warp roles (192 threads):
//   warp 0     producer: per unit one 16 KB bulk copy of the weight block
//              and one of the digit block into a STAGES-deep ring; weights
//              are prefetched before the programmatic-launch wait.
//   warp 1     allocates tensor memory; one thread issues four
//              tcgen05.mma kind::i8 (K = 32 each) per unit into one of two
//              accumulator buffers (a panel segment per buffer).
//   warps 2-5  epilogue, one thread per output channel: read the segment's
//              accumulator, then either write y (the CTA covered the whole
//              panel) or store int32 partials and take a ticket; the last
//              arriver for a panel's rows sums every contributor's partial
//              (integer sums: exact in any order) and writes y.
// Every mbarrier wait is bounded (2 s); on a timeout the device error word
// is set and the CTA winds down.
#include <cstdint>

#include <cuda_bf16.h>

#include "wq_device.cuh"
#include "wq_internal.h"

namespace wq {

static __device__ int g_i8_error = 0;

// ---------------------------------------------------------------------------
// Pre-pass: activations -> exponent e_m and base-256 digit blocks.
// xd: [KB][NR rows][128 bytes], each k-block in the same canonical swizzled
// layout as an INT8 weight block; row 3m + i = digit i of token m; rows
// 3M .. NR-1 and k past K are zero.  xe[m] = e_m.
// ---------------------------------------------------------------------------
__device__ __forceinline__ int bf16_to_scaled_int(uint32_t b, int e)
{
    const uint32_t ex = (b >> 7) & 0xFFu;
    const int mant = (int)(ex ? (0x80u | (b & 0x7Fu)) : (b & 0x7Fu));
    const int sh = (int)(ex ? ex : 1u) - 134 + e; // x = mant * 2^(ex' - 134)
    int X;
    if (sh >= 0) {
        X = mant << sh; // sh <= 14 for every element of the row
    } else if (sh < -15) {
        X = 0; // below half a unit
    } else {
        const int rs = -sh;
        const int q = mant >> rs, rem = mant - (q << rs), half = 1 << (rs - 1);
        X = q + ((rem > half || (rem == half && (q & 1))) ? 1 : 0);
    }
    return (b & 0x8000u) ? -X : X;
}

__global__ void __launch_bounds__(256) xdigits_kernel(const uint16_t *__restrict__ x, int M, int K, int KB, int NR,
                                                      uint8_t *__restrict__ xd, int *__restrict__ xe)
{
    pdl_launch_dependents(); // the GEMM may start streaming weights now
    pdl_wait();              // x may come from the preceding kernel
    const int m = blockIdx.x;
    const size_t kb_bytes = (size_t)NR * 128;
    if (m == M) { // padding rows 3M .. NR-1 of every k-block
        const int rows = NR - 3 * M;
        const int vec = rows * 8; // 16-byte vectors per k-block
        for (int i = threadIdx.x; i < KB * vec; i += blockDim.x) {
            const int kb = i / vec, v = i % vec;
            const int j = 3 * M + v / 8, slot = v % 8;
            *reinterpret_cast<uint4 *>(xd + kb * kb_bytes + (j >> 3) * 1024 + (j & 7) * 128 + slot * 16) =
                make_uint4(0, 0, 0, 0);
        }
        return;
    }
    __shared__ uint32_t s_max[8];
    const uint16_t *row = x + (size_t)m * K;
    uint32_t amax = 0;
    for (int k = 8 * threadIdx.x; k < K; k += 8 * blockDim.x) {
        const uint4 v = *reinterpret_cast<const uint4 *>(row + k);
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int i = 0; i < 4; ++i)
            amax = max(amax, max(w[i] & 0x7FFFu, (w[i] >> 16) & 0x7FFFu));
    }
#pragma unroll
    for (int o = 16; o; o >>= 1)
        amax = max(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    if ((threadIdx.x & 31) == 0)
        s_max[threadIdx.x >> 5] = amax;
    __syncthreads();
    amax = s_max[0];
    for (int i = 1; i < (int)(blockDim.x >> 5); ++i)
        amax = max(amax, s_max[i]);
    // |x| < 2^(E+1) with E the largest element's exponent: e = 21 - E gives |X| < 2^22
    const int ebits = (int)(amax >> 7);
    const int e = amax == 0 ? 0 : 21 - ((ebits ? ebits : 1) - 127);
    if (threadIdx.x == 0)
        xe[m] = e;
    const int chunks = KB * 8;
    for (int ci = threadIdx.x; ci < chunks; ci += blockDim.x) {
        const int kb = ci >> 3, c = ci & 7, k0 = 16 * ci;
        uint32_t d[3][4] = {{0, 0, 0, 0}, {0, 0, 0, 0}, {0, 0, 0, 0}};
        if (k0 < K) {
            const uint4 v0 = *reinterpret_cast<const uint4 *>(row + k0);
            const uint4 v1 = *reinterpret_cast<const uint4 *>(row + k0 + 8);
            const uint32_t w[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const uint32_t b = (w[i >> 1] >> (16 * (i & 1))) & 0xFFFFu;
                const int X = bf16_to_scaled_int(b, e);
                const int d0 = ((X + 128) & 255) - 128;
                const int X1 = (X - d0) >> 8;
                const int d1 = ((X1 + 128) & 255) - 128;
                const int d2 = (X1 - d1) >> 8;
                d[0][i >> 2] |= (uint32_t)(d0 & 255) << (8 * (i & 3));
                d[1][i >> 2] |= (uint32_t)(d1 & 255) << (8 * (i & 3));
                d[2][i >> 2] |= (uint32_t)(d2 & 255) << (8 * (i & 3));
            }
        }
#pragma unroll
        for (int i = 0; i < 3; ++i) {
            const int j = 3 * m + i;
            *reinterpret_cast<uint4 *>(xd + kb * kb_bytes + (j >> 3) * 1024 + (j & 7) * 128 + ((c ^ (j & 7)) << 4)) =
                make_uint4(d[i][0], d[i][1], d[i][2], d[i][3]);
        }
    }
}

// ---------------------------------------------------------------------------
// The GEMM.
// ---------------------------------------------------------------------------
struct I8Params {
    int M, K, N, KB, U;
    const uint8_t *wq;
    const uint16_t *scales;
    uint16_t *y;
    const uint8_t *xd;
    const int *xe;
    int32_t *part;  // [G][2 slots][NR][128 rows] int32
    uint32_t *cnt;  // [panels][4] tickets
};

// Per digit-row count NR (the MMA's N): ring depth and tensor-memory columns.
template <int NR>
struct I8Cfg {
    static constexpr int kAB = 16384;          // weight block
    static constexpr int kBB = NR * 128;       // digit block
    static constexpr int kStageBytes = kAB + kBB;
    static constexpr int kStagesRaw = (200 * 1024) / kStageBytes;
    static constexpr int kStages = kStagesRaw > 12 ? 12 : kStagesRaw;
    static constexpr int kTmemCols = 2 * NR <= 32 ? 32 : 2 * NR <= 64 ? 64 : 2 * NR <= 128 ? 128 : 2 * NR <= 256 ? 256 : 512;
    static constexpr int kColGroup = NR < 48 ? NR : 48; // epilogue columns per pass (16 tokens)
    static_assert(NR % 16 == 0 && NR <= 256, "MMA N: multiple of 16, at most 256");
    static_assert(kStages >= 3, "ring depth");
};

template <int NR>
constexpr size_t i8_smem_bytes()
{
    return 1024 + (size_t)I8Cfg<NR>::kStages * I8Cfg<NR>::kStageBytes + (2 * I8Cfg<NR>::kStages + 4) * 8 + 16;
}

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

template <int NR>
__global__ void __launch_bounds__(192, 1) gemm_i8_kernel(const I8Params p)
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

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int G = gridDim.x, c = blockIdx.x;
    const long long U = p.U;
    const int KB = p.KB;
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
    if (warp == 1) {
        tmem_alloc(s_tmem, TCOLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *s_tmem;
    bool ok = true;

    if (warp == 0) {
        if (lane == 0) {
            const uint64_t pol_w = policy_evict_first(), pol_x = policy_evict_last();
            auto issue_w = [&](int i, int st) {
                uint8_t *dst = ring + st * C::kStageBytes;
                mbar_arrive_expect_tx(&full[st], C::kStageBytes);
                bulk_g2s(dst, p.wq + (size_t)(u0 + i) * C::kAB, C::kAB, &full[st], pol_w);
            };
            auto issue_x = [&](int i, int st) {
                const int kb = (u0 + i) % KB;
                bulk_g2s(ring + st * C::kStageBytes + C::kAB, p.xd + (size_t)kb * C::kBB, C::kBB, &full[st], pol_x);
            };
            // weights do not depend on the preceding kernels: stream them before waiting
            const int pre = n < STAGES ? n : STAGES;
            for (int i = 0; i < pre; ++i)
                issue_w(i, i);
            pdl_wait();
            for (int i = 0; i < pre; ++i)
                issue_x(i, i);
            for (int i = pre; i < n; ++i) {
                const int st = i % STAGES, use = i / STAGES;
                if (!mbar_wait(&empty[st], (use - 1) & 1)) {
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
            constexpr uint32_t idesc = umma_idesc_s8(NR);
            int seg = -1;
            for (int i = 0; i < n; ++i) {
                const int u = u0 + i, kb = u % KB;
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
        pdl_launch_dependents();
    } else {
        // ---------------- epilogue: one thread per output channel ----------------
        pdl_wait(); // xe, y and the workspace may still be in use by the preceding kernels
        const int quad = warp & 3;
        const int row = 32 * quad + lane;
        const uint32_t tq = (uint32_t)(32 * quad) << 16;
        const int M = p.M;
        int seg = 0;
        for (int pnl = n > 0 ? u0 / KB : 0; n > 0 && pnl <= (u1 - 1) / KB && ok; ++pnl, ++seg) {
            const int lo = max(u0, pnl * KB), hi = min(u1, (pnl + 1) * KB);
            const bool whole = (lo == pnl * KB && hi == (pnl + 1) * KB);
            const int b = seg & 1;
            if (!mbar_wait_warp(&accfull[b], (seg >> 1) & 1)) {
                ok = false;
                break;
            }
            tc_fence_after();
            const int nrow = pnl * kPanelRows + row;
            const double s_n = nrow < p.N ? (double)bf16_bits_to_float(p.scales[nrow]) : 0.0;
            const int slot = (pnl == u0 / KB) ? 0 : 1;
            int32_t *mine = p.part + (size_t)(c * 2 + slot) * NR * 128;
#pragma unroll
            for (int c0 = 0; c0 < NR; c0 += CG) {
                int32_t v[CG];
#pragma unroll
                for (int cc = 0; cc < CG; cc += 16) {
                    float f[16];
                    tmem_ld_32x32b_x16(tmem + tq + (uint32_t)(b * NR + c0 + cc), f);
#pragma unroll
                    for (int e2 = 0; e2 < 16; ++e2)
                        v[cc + e2] = __float_as_int(f[e2]);
                }
                tmem_wait_ld();
                if (c0 + CG >= NR) { // the accumulator buffer is free for the MMA again
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0)
                        mbar_arrive(&accempty[b]);
                }
                if (whole) {
                    if (nrow < p.N) {
#pragma unroll
                        for (int t = 0; t < CG / 3; ++t) {
                            const int m = c0 / 3 + t;
                            if (m < M)
                                p.y[(size_t)m * p.N + nrow] =
                                    i8_output(v[3 * t], v[3 * t + 1], v[3 * t + 2], s_n * pow2_of(-__ldg(p.xe + m)));
                        }
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
            // Split panel: every contributor's warp takes a ticket for its 32
            // rows; the last one sums all partials (exact integers) and writes y.
            __threadfence();
            __syncwarp();
            uint32_t ticket = 0;
            if (lane == 0)
                ticket = ticket_take(&p.cnt[pnl * 4 + quad]);
            ticket = __shfl_sync(0xffffffffu, ticket, 0);
            const int cf = sk_owner(U, G, pnl * KB), cl = sk_owner(U, G, (pnl + 1) * KB - 1);
            if (ticket != (uint32_t)(cl - cf))
                continue;
            __threadfence();
            for (int c0 = 0; c0 < 3 * M; c0 += CG) {
                int32_t tot[CG];
#pragma unroll
                for (int j = 0; j < CG; ++j)
                    tot[j] = 0;
                for (int cc = cf; cc <= cl; ++cc) { // all CG loads of a contributor in flight together
                    const int sl = (pnl == sk_start(U, G, cc) / KB) ? 0 : 1;
                    const int32_t *src = p.part + (size_t)(cc * 2 + sl) * NR * 128 + row;
                    int32_t v[CG];
#pragma unroll
                    for (int j = 0; j < CG; ++j)
                        v[j] = (c0 + j < 3 * M) ? __ldcg(src + (size_t)(c0 + j) * 128) : 0;
#pragma unroll
                    for (int j = 0; j < CG; ++j)
                        tot[j] += v[j];
                }
                if (nrow < p.N) {
#pragma unroll
                    for (int t = 0; t < CG / 3; ++t) {
                        const int m = c0 / 3 + t;
                        if (m < M)
                            p.y[(size_t)m * p.N + nrow] =
                                i8_output(tot[3 * t], tot[3 * t + 1], tot[3 * t + 2], s_n * pow2_of(-__ldg(p.xe + m)));
                    }
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
}

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------
int i8_digit_rows(int M) { return M <= 5 ? 16 : M <= 10 ? 32 : M <= 16 ? 48 : M <= 32 ? 96 : 192; }

size_t ws_bytes_gemm_i8(int M, int K, int N)
{
    if (M < 1 || M > kI8MaxM)
        return 0;
    const int NR = i8_digit_rows(M);
    const size_t KB = (size_t)(K + kBlockK - 1) / kBlockK;
    return ws_counter_bytes(N) + 256 + KB * NR * 128 + (size_t)kI8MaxCtas * 2 * NR * 128 * sizeof(int32_t);
}

template <int NR>
static cudaError_t launch_i8_t(const LinearArgs &a, void *ws, int sm_count, cudaStream_t st)
{
    constexpr size_t smem = i8_smem_bytes<NR>();
    static_assert(smem <= 227 * 1024, "shared memory per CTA");
    static bool attr_set = false;
    if (!attr_set) {
        cudaError_t e = cudaFuncSetAttribute(gemm_i8_kernel<NR>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)smem);
        if (e != cudaSuccess)
            return e;
        attr_set = true;
    }
    const Shape sh{8, a.K, a.N, 0};
    const int KB = sh.kblocks();
    uint8_t *base = (uint8_t *)ws + ws_counter_bytes(a.N);
    int *xe = (int *)base;
    uint8_t *xd = base + 256;
    int32_t *part = (int32_t *)(xd + (size_t)KB * NR * 128);

    // the pre-pass: one block per token row plus one for the padding rows
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cfg.stream = st;
    cfg.gridDim = dim3(a.M + 1);
    cfg.blockDim = dim3(256);
    cfg.dynamicSmemBytes = 0;
    cudaError_t e = cudaLaunchKernelEx(&cfg, xdigits_kernel, a.x, a.M, a.K, KB, NR, xd, xe);
    if (e != cudaSuccess)
        return e;

    I8Params p;
    p.M = a.M;
    p.K = a.K;
    p.N = a.N;
    p.KB = KB;
    p.U = sh.panels() * KB;
    p.wq = (const uint8_t *)a.wq;
    p.scales = (const uint16_t *)a.scales;
    p.y = a.y;
    p.xd = xd;
    p.xe = xe;
    p.part = part;
    p.cnt = (uint32_t *)ws;
    int G = sm_count < kI8MaxCtas ? sm_count : kI8MaxCtas;
    if (G > p.U)
        G = p.U;
    cfg.gridDim = dim3(G);
    cfg.blockDim = dim3(192);
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
