// wq_gemv.cu -- decode-regime GEMV (M <= 32) for W8A16 and W4A16.
//
// Register-level dequantization with 128-bit weight loads and no shared
// memory on the weight path (the "BitBLAS-style GEMV" row of the tileInfer
// README, Features table).  Each warp streams one 16-row block over a K
// slice; every lane's 16-byte loads unpack straight into m16n8k16 A
// fragments (see wq_layout.h), which go into mma.sync with the activations
// as the 8-token B operand and fp32 accumulators.  For W4A16 the MMA sees
// exact (q - z) integers and the bf16 group scale is applied in fp32 after
// each group (32, 64 or 128 k), so the weights are never rounded.  For W8A16 the per-channel scale is applied once in the
// epilogue.  K slices of one row block are summed across warps through
// shared memory in a fixed order (deterministic).
#include <cstdint>

#include <cuda_fp16.h>

#include "wq_device.cuh"
#include "wq_internal.h"

namespace wq {

struct GemvParams {
    const uint16_t *x;
    int M, K, N;
    const uint8_t *wq;
    const uint16_t *scales;
    const uint8_t *zeros;
    uint16_t *y;
    Shape sh;
    int ks; // K slices per 16-row block (1, 2, 4, 8); the 8 warps of a CTA
            // cover 8/ks row blocks
};

constexpr int kGemvWarps = 8;

// Activation format of a launch: bf16 (the layer's default) or fp16 (the
// FP16 half of the validation matrix of the Marlin register and launch
// scheduling benchmark, "Validation and limits").  Dequantized weights are
// exact integers in either format (|q - z| <= 15, |q| <= 128), built with
// the format's magic constant: 128 + n in bf16 (0x4300 | n), 1024 + n in
// fp16 (0x6400 | n).  Accumulation is fp32; the output is rounded to the
// activation format, to nearest even.
template <bool F16>
struct Act {
    static constexpr uint32_t kMagic2 = F16 ? 0x64006400u : 0x43004300u;
    __device__ static __forceinline__ uint32_t nib_pair(uint32_t w_shifted)
    {
        uint32_t r;
        asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(r) : "r"(w_shifted), "r"(0x000F000Fu), "r"(kMagic2));
        return r; // (a & b) | c
    }
    __device__ static __forceinline__ uint32_t sub2(uint32_t a, uint32_t b)
    {
        uint32_t r;
        if constexpr (F16)
            asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
        else
            asm("sub.rn.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
        return r;
    }
    __device__ static __forceinline__ void mma(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                               uint32_t b0, uint32_t b1)
    {
        if constexpr (F16)
            asm volatile("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 "
                         "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
                         : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
                         : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
        else
            mma_bf16_16816(d, a0, a1, a2, a3, b0, b1);
    }
    // two int8 codes (bytes 2h, 2h+1 of u = w ^ 0x80808080) as a pair of the format
    __device__ static __forceinline__ uint32_t s8pair(uint32_t u, int h)
    {
        if constexpr (F16) {
            const float f0 = __uint_as_float(__byte_perm(u, 0x4B000000u, h == 0 ? 0x7540u : 0x7542u));
            const float f1 = __uint_as_float(__byte_perm(u, 0x4B000000u, h == 0 ? 0x7541u : 0x7543u));
            __half2 v = __floats2half2_rn(f0 - 8388736.0f, f1 - 8388736.0f); // exact: |q| <= 128
            return *reinterpret_cast<uint32_t *>(&v);
        } else {
            return s8pair_bf16(u, h);
        }
    }
    __device__ static __forceinline__ uint16_t out(float v)
    {
        if constexpr (F16)
            return __half_as_ushort(__float2half_rn(v));
        else
            return __bfloat16_as_ushort(__float2bfloat16_rn(v));
    }
};

template <int MT>
__device__ __forceinline__ void load_x_frag(const GemvParams &p, int g, int k, uint2 (&xf)[MT])
{
#pragma unroll
    for (int mt = 0; mt < MT; ++mt) {
        const int m = 8 * mt + g;
        xf[mt] = (m < p.M) ? ldg_keep(p.x + (size_t)m * p.K + k) : make_uint2(0u, 0u);
    }
}

// One INT8 chunk pair: this lane's 16 consecutive k (kc .. kc+15) of rows g
// (wa) and g+8 (wb).  Step i = 0..3 is an m16n8k16 MMA whose k-slots 2t,
// 2t+1, 2t+8, 2t+9 take k = kc+4i .. kc+4i+3; the activations of the same k
// are xv[mt] (kc .. kc+7) and xw[mt] (kc+8 .. kc+15) of token row 8*mt + g.
template <int MT, bool F16>
__device__ __forceinline__ void int8_chunk(const uint4 &wa, const uint4 &wb, const uint4 (&xv)[MT],
                                           const uint4 (&xw)[MT], float (&acc)[MT][4])
{
    const uint32_t ra[4] = {wa.x, wa.y, wa.z, wa.w}, rb[4] = {wb.x, wb.y, wb.z, wb.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const uint32_t ua = ra[i] ^ 0x80808080u, ub = rb[i] ^ 0x80808080u;
        const uint32_t a0 = Act<F16>::s8pair(ua, 0), a2 = Act<F16>::s8pair(ua, 1);
        const uint32_t a1 = Act<F16>::s8pair(ub, 0), a3 = Act<F16>::s8pair(ub, 1);
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) {
            const uint4 &xx = i < 2 ? xv[mt] : xw[mt];
            const uint32_t b0 = (i & 1) ? xx.z : xx.x, b1 = (i & 1) ? xx.w : xx.y;
            Act<F16>::mma(acc[mt], a0, a1, a2, a3, b0, b1);
        }
    }
}

// One INT4 tile (16 rows x 64 k): four MMAs per 8-token tile on exact
// (q - z) values.  zlo / zhi are bf16x2 {128+z, 128+z} of rows g and g+8.
template <int MT, bool F16>
__device__ __forceinline__ void int4_tile(const GemvParams &p, const uint4 &w, int kt_base, int g, int t,
                                          uint32_t zlo, uint32_t zhi, float (&cg)[MT][4])
{
    using A = Act<F16>;
    uint32_t xr[4], yr[4], zr[4], wr[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        xr[i] = A::sub2(A::nib_pair(w.x >> (4 * i)), zlo);
        yr[i] = A::sub2(A::nib_pair(w.y >> (4 * i)), zhi);
        zr[i] = A::sub2(A::nib_pair(w.z >> (4 * i)), zlo);
        wr[i] = A::sub2(A::nib_pair(w.w >> (4 * i)), zhi);
    }
    uint2 xa[MT], xb[MT], xc[MT], xd[MT];
    load_x_frag<MT>(p, g, kt_base + 4 * t, xa);
    load_x_frag<MT>(p, g, kt_base + 16 + 4 * t, xb);
    load_x_frag<MT>(p, g, kt_base + 32 + 4 * t, xc);
    load_x_frag<MT>(p, g, kt_base + 48 + 4 * t, xd);
#pragma unroll
    for (int mt = 0; mt < MT; ++mt) {
        A::mma(cg[mt], xr[0], yr[0], xr[1], yr[1], xa[mt].x, xa[mt].y);
        A::mma(cg[mt], xr[2], yr[2], xr[3], yr[3], xb[mt].x, xb[mt].y);
        A::mma(cg[mt], zr[0], wr[0], zr[1], wr[1], xc[mt].x, xc[mt].y);
        A::mma(cg[mt], zr[2], wr[2], zr[3], wr[3], xd[mt].x, xd[mt].y);
    }
}

// INT8: the K range of this slice is a run of 64-k half-blocks [h0, h1);
// in half-block hb lane (g, t) takes chunk c = 4*(hb%2) + t of rows g and g+8.
template <int MT, bool F16>
__device__ __forceinline__ void gemv_int8_slice(const GemvParams &p, int rb, int h0, int h1, int lane,
                                                float (&acc)[MT][4])
{
    constexpr int U = 2;
    const int g = lane >> 2, t = lane & 3;
    const int pnl = rb >> 3, r = 16 * (rb & 7) + g; // row of the panel (and r + 8)
    const uint8_t *panel = p.wq + p.sh.block_offset(pnl, 0);
    auto load_w = [&](int hb, uint4 &wa, uint4 &wb) {
        if (hb < h1) {
            const uint8_t *src = panel + (size_t)(hb >> 1) * 16384 + int8_chunk_in_block(r, 4 * (hb & 1) + t);
            wa = ldg_stream(src);
            wb = ldg_stream(src + 1024);
        } else {
            wa = wb = make_uint4(0, 0, 0, 0);
        }
    };
    uint4 ca[U], cb[U], na[U], nb[U];
#pragma unroll
    for (int u = 0; u < U; ++u)
        load_w(h0 + u, ca[u], cb[u]);
    for (int hb = h0; hb < h1; hb += U) {
#pragma unroll
        for (int u = 0; u < U; ++u)
            load_w(hb + U + u, na[u], nb[u]);
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int kc = 64 * (hb + u) + 16 * t;
            if (hb + u < h1) {
                uint4 xv[MT], xw[MT];
#pragma unroll
                for (int mt = 0; mt < MT; ++mt) {
                    const int m = 8 * mt + g;
                    const bool ok = m < p.M && kc < p.K; // k past K: zero weights, keep x finite
                    const uint16_t *xr = p.x + (size_t)m * p.K + kc;
                    xv[mt] = ok ? ldg_keep4(xr) : make_uint4(0, 0, 0, 0);
                    xw[mt] = ok ? ldg_keep4(xr + 8) : make_uint4(0, 0, 0, 0);
                }
                int8_chunk<MT, F16>(ca[u], cb[u], xv, xw, acc);
            }
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            ca[u] = na[u];
            cb[u] = nb[u];
        }
    }
}

// One INT4 tile (16 rows x 64 k) whose two halves (k 0-31: words x, y;
// k 32-63: words z, w) are separate 32-k groups: each half's two MMAs go
// into their own accumulator, scaled into acc by that group's scale.
// zl[h] / zh[h]: the pairs {magic + z} of rows g and g+8 in half h; sl/sh
// the scales (binary32).
template <int MT, bool F16>
__device__ __forceinline__ void int4_tile_g32(const GemvParams &p, const uint4 &w, int kt_base, int g, int t,
                                              const uint32_t (&zl)[2], const uint32_t (&zh)[2], const float (&sl)[2],
                                              const float (&sh)[2], float (&acc)[MT][4])
{
    using A = Act<F16>;
    uint32_t xr[4], yr[4], zr[4], wr[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        xr[i] = A::sub2(A::nib_pair(w.x >> (4 * i)), zl[0]);
        yr[i] = A::sub2(A::nib_pair(w.y >> (4 * i)), zh[0]);
        zr[i] = A::sub2(A::nib_pair(w.z >> (4 * i)), zl[1]);
        wr[i] = A::sub2(A::nib_pair(w.w >> (4 * i)), zh[1]);
    }
    uint2 xa[MT], xb[MT], xc[MT], xd[MT];
    load_x_frag<MT>(p, g, kt_base + 4 * t, xa);
    load_x_frag<MT>(p, g, kt_base + 16 + 4 * t, xb);
    load_x_frag<MT>(p, g, kt_base + 32 + 4 * t, xc);
    load_x_frag<MT>(p, g, kt_base + 48 + 4 * t, xd);
#pragma unroll
    for (int mt = 0; mt < MT; ++mt) {
        float c0[4] = {0.f, 0.f, 0.f, 0.f}, c1[4] = {0.f, 0.f, 0.f, 0.f};
        A::mma(c0, xr[0], yr[0], xr[1], yr[1], xa[mt].x, xa[mt].y);
        A::mma(c0, xr[2], yr[2], xr[3], yr[3], xb[mt].x, xb[mt].y);
        A::mma(c1, zr[0], wr[0], zr[1], wr[1], xc[mt].x, xc[mt].y);
        A::mma(c1, zr[2], wr[2], zr[3], wr[3], xd[mt].x, xd[mt].y);
        acc[mt][0] = fmaf(sl[1], c1[0], fmaf(sl[0], c0[0], acc[mt][0]));
        acc[mt][1] = fmaf(sl[1], c1[1], fmaf(sl[0], c0[1], acc[mt][1]));
        acc[mt][2] = fmaf(sh[1], c1[2], fmaf(sh[0], c0[2], acc[mt][2]));
        acc[mt][3] = fmaf(sh[1], c1[3], fmaf(sh[0], c0[3], acc[mt][3]));
    }
}

// INT4 over the 128-k blocks [b0, b1) of row block rb, groups of LG k
// (32, 64 or 128; NG = 128 / LG groups per block).  Each group's MMAs
// accumulate on their own and are scaled into acc in fp32 at the group's
// end, so the weights the MMA sees are the exact integers q - z.
template <int MT, int LG, bool F16>
__device__ __forceinline__ void gemv_int4_slice(const GemvParams &p, int rb, int b0, int b1, int lane,
                                                float (&acc)[MT][4])
{
    constexpr int UG = 2;        // blocks per prefetch batch (2 tiles each)
    constexpr int NG = 128 / LG; // groups per block
    const int g = lane >> 2, t = lane & 3;
    const int KL = p.K / LG;     // groups per row
    const int pnl = rb >> 3, rowp = 16 * (rb & 7) + g; // row inside the panel
    // this lane's 16 bytes of the row block's tiles: (rb, k-block bi) is 1 KB
    // at ((panel KB + bi) 8 + rb % 8) KB, its two 64-k tiles 512 B apart
    const uint8_t *base = p.wq + ((size_t)pnl * p.sh.kblocks() * 8 + (rb & 7)) * 1024 + 16 * lane;
    uint4 cw[UG][2], nw[UG][2];
    uint16_t cs[UG][NG][2], ns[UG][NG][2];
    uint8_t cz[UG][NG][2], nz[UG][NG][2];
    auto load = [&](int bi, uint4 (&w)[2], uint16_t (&sc)[NG][2], uint8_t (&z)[NG][2]) {
        if (bi < b1) {
            w[0] = ldg_stream(base + (size_t)bi * 8192);
            w[1] = ldg_stream(base + (size_t)bi * 8192 + 512);
#pragma unroll
            for (int j = 0; j < NG; ++j) {
                const size_t grp = (size_t)pnl * KL + (size_t)bi * NG + j;
                sc[j][0] = __ldg(p.scales + grp * kPanelRows + rowp);
                sc[j][1] = __ldg(p.scales + grp * kPanelRows + rowp + 8);
                z[j][0] = __ldg(p.zeros + grp * 64 + rowp / 2);
                z[j][1] = __ldg(p.zeros + grp * 64 + (rowp + 8) / 2);
            }
        } else {
            w[0] = w[1] = make_uint4(0, 0, 0, 0);
#pragma unroll
            for (int j = 0; j < NG; ++j) {
                sc[j][0] = sc[j][1] = 0;
                z[j][0] = z[j][1] = 0;
            }
        }
    };
#pragma unroll
    for (int u = 0; u < UG; ++u)
        load(b0 + u, cw[u], cs[u], cz[u]);
    const int zsh = 4 * (rowp & 1);
    auto zpair = [&](uint8_t zb) {
        const uint32_t zz = (zb >> zsh) & 0xFu;
        return Act<F16>::kMagic2 | zz | (zz << 16); // the pair {magic + z, magic + z}
    };
    for (int bi = b0; bi < b1; bi += UG) {
#pragma unroll
        for (int u = 0; u < UG; ++u)
            load(bi + UG + u, nw[u], ns[u], nz[u]);
#pragma unroll
        for (int u = 0; u < UG; ++u) {
            if (bi + u < b1) {
                const int kt_base = 128 * (bi + u);
                if constexpr (LG == 32) {
#pragma unroll
                    for (int tau = 0; tau < 2; ++tau) { // tile tau: groups 2 tau and 2 tau + 1
                        const uint32_t zl[2] = {zpair(cz[u][2 * tau][0]), zpair(cz[u][2 * tau + 1][0])};
                        const uint32_t zh[2] = {zpair(cz[u][2 * tau][1]), zpair(cz[u][2 * tau + 1][1])};
                        const float sl[2] = {bf16_bits_to_float(cs[u][2 * tau][0]),
                                             bf16_bits_to_float(cs[u][2 * tau + 1][0])};
                        const float sh[2] = {bf16_bits_to_float(cs[u][2 * tau][1]),
                                             bf16_bits_to_float(cs[u][2 * tau + 1][1])};
                        int4_tile_g32<MT, F16>(p, cw[u][tau], kt_base + 64 * tau, g, t, zl, zh, sl, sh, acc);
                    }
                } else {
#pragma unroll
                    for (int j = 0; j < NG; ++j) { // LG = 64: one tile per group; 128: both tiles
                        float cg[MT][4];
#pragma unroll
                        for (int mt = 0; mt < MT; ++mt)
                            cg[mt][0] = cg[mt][1] = cg[mt][2] = cg[mt][3] = 0.f;
                        const uint32_t zlo = zpair(cz[u][j][0]), zhi = zpair(cz[u][j][1]);
#pragma unroll
                        for (int tau = 0; tau < 2 / NG; ++tau) {
                            const int ti = j * (2 / NG) + tau;
                            int4_tile<MT, F16>(p, cw[u][ti], kt_base + 64 * ti, g, t, zlo, zhi, cg);
                        }
                        const float slo = bf16_bits_to_float(cs[u][j][0]), shi = bf16_bits_to_float(cs[u][j][1]);
#pragma unroll
                        for (int mt = 0; mt < MT; ++mt) {
                            acc[mt][0] = fmaf(slo, cg[mt][0], acc[mt][0]);
                            acc[mt][1] = fmaf(slo, cg[mt][1], acc[mt][1]);
                            acc[mt][2] = fmaf(shi, cg[mt][2], acc[mt][2]);
                            acc[mt][3] = fmaf(shi, cg[mt][3], acc[mt][3]);
                        }
                    }
                }
            }
        }
#pragma unroll
        for (int u = 0; u < UG; ++u) {
            cw[u][0] = nw[u][0];
            cw[u][1] = nw[u][1];
#pragma unroll
            for (int j = 0; j < NG; ++j) {
                cs[u][j][0] = ns[u][j][0];
                cs[u][j][1] = ns[u][j][1];
                cz[u][j][0] = nz[u][j][0];
                cz[u][j][1] = nz[u][j][1];
            }
        }
    }
}

template <int BITS, int MT, int LG = 128, bool F16 = false>
__global__ void __launch_bounds__(kGemvWarps * 32) gemv_kernel(const GemvParams p)
{
    __shared__ float red[kGemvWarps][MT * 4][32];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    const int ks = p.ks, rbs_per_cta = kGemvWarps / ks;
    const int nrb = p.N >> 4;
    const int units = (nrb + rbs_per_cta - 1) / rbs_per_cta;
    const int ks_i = warp % ks;
    // The next kernel on the stream may launch now (this grid is one wave,
    // every CTA resident); x and y wait for the preceding kernel.
    pdl_launch_dependents();
    pdl_wait();

    for (int unit = blockIdx.x; unit < units; unit += gridDim.x) {
        const int rb = unit * rbs_per_cta + warp / ks;
        float acc[MT][4];
#pragma unroll
        for (int mt = 0; mt < MT; ++mt)
            acc[mt][0] = acc[mt][1] = acc[mt][2] = acc[mt][3] = 0.f;
        if (rb < nrb) {
            if constexpr (BITS == 8) {
                const int T = (p.K + 63) / 64;
                gemv_int8_slice<MT, F16>(p, rb, (int)((long long)T * ks_i / ks), (int)((long long)T * (ks_i + 1) / ks),
                                    lane, acc);
            } else {
                const int B = p.K / 128; // 128-k blocks
                gemv_int4_slice<MT, LG, F16>(p, rb, (int)((long long)B * ks_i / ks), (int)((long long)B * (ks_i + 1) / ks),
                                        lane, acc);
            }
        }
        if (ks > 1) {
#pragma unroll
            for (int mt = 0; mt < MT; ++mt)
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    red[warp][mt * 4 + i][lane] = acc[mt][i];
            __syncthreads();
            if (ks_i == 0) {
                for (int s = 1; s < ks; ++s)
#pragma unroll
                    for (int mt = 0; mt < MT; ++mt)
#pragma unroll
                        for (int i = 0; i < 4; ++i)
                            acc[mt][i] += red[warp + s][mt * 4 + i][lane];
            }
            __syncthreads();
        }
        if (ks_i == 0 && rb < nrb) {
            const int n_lo = 16 * rb + g, n_hi = n_lo + 8;
            float s_lo = 1.f, s_hi = 1.f;
            if constexpr (BITS == 8) {
                s_lo = bf16_bits_to_float(__ldg(p.scales + n_lo));
                s_hi = bf16_bits_to_float(__ldg(p.scales + n_hi));
            }
#pragma unroll
            for (int mt = 0; mt < MT; ++mt) {
                const int m0 = 8 * mt + 2 * t, m1 = m0 + 1;
                if (m0 < p.M) {
                    p.y[(size_t)m0 * p.N + n_lo] = Act<F16>::out(acc[mt][0] * s_lo);
                    p.y[(size_t)m0 * p.N + n_hi] = Act<F16>::out(acc[mt][2] * s_hi);
                }
                if (m1 < p.M) {
                    p.y[(size_t)m1 * p.N + n_lo] = Act<F16>::out(acc[mt][1] * s_lo);
                    p.y[(size_t)m1 * p.N + n_hi] = Act<F16>::out(acc[mt][3] * s_hi);
                }
            }
        }
    }
}

template <int BITS, int MT, int LG = 128, bool F16 = false>
static cudaError_t launch_gemv_t(const GemvParams &p, int sm_count, cudaStream_t st)
{
    int occ = 1; // CTAs per SM, from the hardware occupancy query (cached per device)
    {
        const cudaError_t e = kernel_setup((const void *)gemv_kernel<BITS, MT, LG, F16>, 0, kGemvWarps * 32, 0, &occ);
        if (e != cudaSuccess)
            return e;
    }
    const int rbs_per_cta = kGemvWarps / p.ks;
    const int units = ((p.N >> 4) + rbs_per_cta - 1) / rbs_per_cta;
    int grid = occ * sm_count;
    if (grid > units)
        grid = units;
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(kGemvWarps * 32);
    cfg.stream = st;
    return cudaLaunchKernelEx(&cfg, gemv_kernel<BITS, MT, LG, F16>, p);
}

template <bool F16>
static cudaError_t launch_gemv_fmt(const GemvParams &p, int bits, int group, int sm_count, cudaStream_t st)
{
    const int mt = (p.M + 7) / 8;
    if (bits == 8) {
        if (mt == 1) return launch_gemv_t<8, 1, 128, F16>(p, sm_count, st);
        if (mt == 2) return launch_gemv_t<8, 2, 128, F16>(p, sm_count, st);
        return launch_gemv_t<8, 4, 128, F16>(p, sm_count, st);
    }
    if (group == 32) {
        if (mt == 1) return launch_gemv_t<4, 1, 32, F16>(p, sm_count, st);
        if (mt == 2) return launch_gemv_t<4, 2, 32, F16>(p, sm_count, st);
        return launch_gemv_t<4, 4, 32, F16>(p, sm_count, st);
    }
    if (group == 64) {
        if (mt == 1) return launch_gemv_t<4, 1, 64, F16>(p, sm_count, st);
        if (mt == 2) return launch_gemv_t<4, 2, 64, F16>(p, sm_count, st);
        return launch_gemv_t<4, 4, 64, F16>(p, sm_count, st);
    }
    if (mt == 1) return launch_gemv_t<4, 1, 128, F16>(p, sm_count, st);
    if (mt == 2) return launch_gemv_t<4, 2, 128, F16>(p, sm_count, st);
    return launch_gemv_t<4, 4, 128, F16>(p, sm_count, st);
}

cudaError_t launch_gemv(const LinearArgs &a, int ks, int sm_count, cudaStream_t st, bool f16)
{
    GemvParams p;
    p.x = a.x;
    p.M = a.M;
    p.K = a.K;
    p.N = a.N;
    p.wq = (const uint8_t *)a.wq;
    p.scales = (const uint16_t *)a.scales;
    p.zeros = (const uint8_t *)a.zeros;
    p.y = a.y;
    p.sh = Shape{a.bits, a.K, a.N, a.group};
    p.ks = ks;
    return f16 ? launch_gemv_fmt<true>(p, a.bits, a.group, sm_count, st)
               : launch_gemv_fmt<false>(p, a.bits, a.group, sm_count, st);
}

} // namespace wq
