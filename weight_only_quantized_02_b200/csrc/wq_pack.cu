// wq_pack.cu -- quantizers, packers and debug views of the packed layout.
//
// Quantizers turn fp32 source weights into the canonical W8A16 / W4A16
// tensors (the shapes of the decode workloads).  Every decision is taken in
// binary64 with IEEE round-to-nearest-even division, as in the CPU oracle.
// Packers rewrite canonical tensors into the layout of wq_layout.h.
#include <cmath>
#include <cstdint>
#include <cstring>

#include "wq_device.cuh"
#include "wq_internal.h"

namespace wq {

// ---------------------------------------------------------------------------
// binary64 -> bf16 rounding (device), from the IEEE-754 definition: find the
// quantum of |v|'s binade (8 significant bits; fixed 2^-133 below the
// smallest normal), round the exact count of quanta, scale back.
// ---------------------------------------------------------------------------
__device__ __forceinline__ double pow2_exact(int e) // 2^e, -1022 <= e <= 1023
{
    return __longlong_as_double((long long)(1023 + e) << 52);
}

__device__ uint16_t f64_to_bf16(double v, bool toward_pos_inf)
{
    if (v == 0.0)
        return signbit(v) ? 0x8000 : 0x0000;
    const bool neg = signbit(v);
    const double a = fabs(v);
    const int e = (int)((__double_as_longlong(a) >> 52) & 0x7FF) - 1023;
    const int qe = (e >= -126) ? e - 7 : -133;
    const double count = a * pow2_exact(-qe); // exact
    double r;
    if (toward_pos_inf)
        r = neg ? floor(count) : ceil(count);
    else
        r = rint(count); // ties to even
    const double res = r * pow2_exact(qe);
    if (res >= 0x1p128)
        return (toward_pos_inf && neg) ? 0xFF7F : (neg ? 0xFF80 : 0x7F80);
    const uint32_t fb = __float_as_uint((float)res); // exact
    return (uint16_t)((fb >> 16) | (neg ? 0x8000u : 0u));
}

// ---------------------------------------------------------------------------
// INT8 symmetric per-channel quantizer: one block per output row.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) quant_int8_kernel(const float *__restrict__ W, int K,
                                                         int8_t *__restrict__ q,
                                                         uint16_t *__restrict__ s)
{
    const int n = blockIdx.x;
    const float *row = W + (size_t)n * K;
    float amax = 0.f;
    for (int k = threadIdx.x; k < K; k += blockDim.x)
        amax = fmaxf(amax, fabsf(row[k]));
    for (int o = 16; o; o >>= 1)
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    __shared__ float red[8];
    __shared__ double s_d;
    if ((threadIdx.x & 31) == 0)
        red[threadIdx.x >> 5] = amax;
    __syncthreads();
    if (threadIdx.x == 0) {
        float m = 0.f;
        for (int i = 0; i < (int)(blockDim.x >> 5); ++i)
            m = fmaxf(m, red[i]);
        const uint16_t sb = f64_to_bf16((double)m / 127.0, false);
        s[n] = sb;
        s_d = (double)bf16_bits_to_float(sb);
    }
    __syncthreads();
    const double sd = s_d;
    for (int k = threadIdx.x; k < K; k += blockDim.x) {
        double v = 0.0;
        if (sd != 0.0) {
            v = rint((double)row[k] / sd);
            v = fmin(fmax(v, -127.0), 127.0);
        }
        q[(size_t)n * K + k] = (int8_t)v;
    }
}

// ---------------------------------------------------------------------------
// INT4 asymmetric group quantizer: a warp per (row, group of G), each lane
// taking words of 8 consecutive k (one canonical word) in turn.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) quant_int4_kernel(const float *__restrict__ W, int K, int N, int G,
                                                         uint32_t *__restrict__ q,
                                                         uint16_t *__restrict__ s,
                                                         uint32_t *__restrict__ z)
{
    const int KG = K / G, ZW = (KG + 7) / 8;
    const long long unit = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (unit >= (long long)N * KG)
        return; // the whole warp
    const int n = (int)(unit / KG), g = (int)(unit % KG);
    const float *src = W + (size_t)n * K + (size_t)g * G;
    float mn = 0.f, mx = 0.f;
    for (int k = lane; k < G; k += 32) {
        mn = fminf(mn, src[k]);
        mx = fmaxf(mx, src[k]);
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) {
        mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    }
    const double lo = (double)mn, hi = (double)mx; // lo <= 0 <= hi
    uint16_t sb = 0;
    double sd = 0.0;
    uint32_t zq = 0;
    if (hi - lo > 0.0) {
        sb = f64_to_bf16((hi - lo) / 15.0, true);
        sd = (double)bf16_bits_to_float(sb);
        zq = (uint32_t)fmin(fmax(rint(-lo / sd), 0.0), 15.0);
    }
    for (int wi = lane; wi < G / 8; wi += 32) {
        uint32_t word = 0;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            uint32_t qe = 0;
            if (sd != 0.0)
                qe = (uint32_t)fmin(fmax(rint((double)src[8 * wi + e] / sd) + (double)zq, 0.0), 15.0);
            word |= qe << (4 * e);
        }
        q[(size_t)n * (K / 8) + (size_t)g * (G / 8) + wi] = word;
    }
    if (lane == 0) {
        s[(size_t)n * KG + g] = sb;
        if (zq)
            atomicOr(&z[(size_t)n * ZW + g / 8], zq << (4 * (g % 8)));
    }
}

// ---------------------------------------------------------------------------
// Packers
// ---------------------------------------------------------------------------
__global__ void pack_int8_kernel(const int8_t *__restrict__ q, int K, int N, uint4 *__restrict__ out,
                                 size_t n_vec, Shape sh)
{
    const size_t idx = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (idx >= n_vec)
        return;
    // 16-byte vector u of block b: row r = u / 8 of the panel, chunk slot u % 8
    // holds chunk c = slot ^ (r % 8), i.e. k = 16c .. 16c+15 of the block
    const size_t b = idx / 1024;
    const int u = (int)(idx % 1024);
    const int p = (int)(b / sh.kblocks()), kb = (int)(b % sh.kblocks());
    const int r = u >> 3, c = (u & 7) ^ (r & 7);
    const int row = p * kPanelRows + r;
    const int k0 = kb * kBlockK + 16 * c;
    auto run = [&](int k) -> uint32_t {
        if (row >= N || k >= K)
            return 0u;
        return *reinterpret_cast<const uint32_t *>(q + (size_t)row * K + k);
    };
    out[idx] = make_uint4(run(k0), run(k0 + 4), run(k0 + 8), run(k0 + 12));
}

__device__ __forceinline__ uint32_t canon_nibble(const uint32_t *q, int K, int row, int k)
{
    return (q[(size_t)row * (K / 8) + k / 8] >> (4 * (k % 8))) & 0xFu;
}

__global__ void pack_int4_kernel(const uint32_t *__restrict__ q, int K, int N, uint4 *__restrict__ out,
                                 size_t n_vec, Shape sh)
{
    const size_t idx = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (idx >= n_vec)
        return;
    const int vec_per_block = sh.block_bytes() / 16, vec_per_rb = sh.rb_bytes() / 16;
    const size_t b = idx / vec_per_block;
    const int u = (int)(idx % vec_per_block);
    const int p = (int)(b / sh.kblocks()), kb = (int)(b % sh.kblocks());
    const int j = u / vec_per_rb, rem = u % vec_per_rb;
    const int t = rem / 32, l = rem % 32, g = l >> 2, tt = l & 3;
    const int n0 = p * kPanelRows + 16 * j;
    const int kt = kb * kBlockK + 64 * t;
    auto word = [&](int row, int ka, int kbb) -> uint32_t {
        if (row >= N)
            return 0u;
        uint32_t w = 0;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            const int k = (e < 4) ? ka + e : kbb + (e - 4);
            w |= canon_nibble(q, K, row, k) << (4 * int4_nibble_pos(e));
        }
        return w;
    };
    uint4 v;
    v.x = word(n0 + g, kt + 4 * tt, kt + 16 + 4 * tt);
    v.y = word(n0 + g + 8, kt + 4 * tt, kt + 16 + 4 * tt);
    v.z = word(n0 + g, kt + 32 + 4 * tt, kt + 48 + 4 * tt);
    v.w = word(n0 + g + 8, kt + 32 + 4 * tt, kt + 48 + 4 * tt);
    out[idx] = v;
}

// Folds a nonnegative binary32 value into the trailer's wmax_bits word
// (nonnegative floats order like their bit patterns): one atomic per warp.
__device__ __forceinline__ void wmax_fold(uint32_t *wmax_bits, float v)
{
    uint32_t b = __float_as_uint(v);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
        b = max(b, __shfl_xor_sync(0xffffffffu, b, o));
    if ((threadIdx.x & 31) == 0)
        atomicMax(wmax_bits, b);
}

__global__ void pack_scales_int8_kernel(const uint16_t *__restrict__ s, int N, uint16_t *__restrict__ out,
                                        int total, uint32_t *wmax_bits)
{
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    const uint16_t v = (i < total && i < N) ? s[i] : 0;
    if (i < total)
        out[i] = v;
    wmax_fold(wmax_bits, 128.f * fabsf(__uint_as_float((uint32_t)v << 16)));
}

// Layout group gl of row `row` takes canonical group gl * L / G (G = the
// quantization group: equal to L, or K for per-channel, repeated per block).
__global__ void pack_sz_int4_kernel(const uint16_t *__restrict__ s, const uint32_t *__restrict__ z, int K,
                                    int N, int G, uint16_t *__restrict__ s_out, uint8_t *__restrict__ z_out,
                                    Shape sh, uint32_t *wmax_bits)
{
    const int L = sh.group, KL = K / L;         // layout groups per row
    const int KG = K / G, ZW = (KG + 7) / 8;     // canonical groups per row, zero-point words
    const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    const long long total = (long long)sh.panels() * KL * kPanelRows;
    const int i = (int)(idx % kPanelRows);
    const long long pg = idx / kPanelRows;
    const int gl = (int)(pg % KL), p = (int)(pg / KL);
    const int g = (int)((long long)gl * L / G);
    const int row = p * kPanelRows + i;
    // largest |q - z| the zero point allows, times the scale
    float wm = 0.f;
    if (idx < total && row < N) {
        const uint32_t zz = (z[(size_t)row * ZW + g / 8] >> (4 * (g % 8))) & 0xFu;
        wm = fabsf(__uint_as_float((uint32_t)s[(size_t)row * KG + g] << 16)) * (float)max(zz, 15u - zz);
    }
    wmax_fold(wmax_bits, wm);
    if (idx >= total)
        return;
    s_out[idx] = row < N ? s[(size_t)row * KG + g] : 0;
    if ((i & 1) == 0) {
        uint32_t z0 = 0, z1 = 0;
        if (row < N)
            z0 = (z[(size_t)row * ZW + g / 8] >> (4 * (g % 8))) & 0xFu;
        if (row + 1 < N)
            z1 = (z[(size_t)(row + 1) * ZW + g / 8] >> (4 * (g % 8))) & 0xFu;
        z_out[pg * 64 + i / 2] = (uint8_t)(z0 | (z1 << 4));
    }
}

// group: the quantization group the caller packed (0 for INT8, K for
// per-channel INT4), recorded for wq_check_packed.
__global__ void write_trailer_kernel(uint8_t *wq, Shape sh, int group)
{
    Trailer t{};
    t.magic = kMagic;
    t.version = kLayoutVersion;
    t.bits = (uint32_t)sh.bits;
    t.K = (uint32_t)sh.K;
    t.N = (uint32_t)sh.N;
    t.group = (uint32_t)group;
    const size_t wb = sh.weight_bytes();
    t.layout_bytes_lo = (uint32_t)(wb & 0xffffffffu);
    t.layout_bytes_hi = (uint32_t)(wb >> 32);
    uint32_t *dst = reinterpret_cast<uint32_t *>(wq + wb);
    const uint32_t *src = reinterpret_cast<const uint32_t *>(&t);
    for (int i = 0; i < 16; ++i)
        dst[i] = src[i];
}

// ---------------------------------------------------------------------------
// Debug views: element (n, k) of the packed layout.
// ---------------------------------------------------------------------------
__device__ int packed_q(const uint8_t *wq, const Shape &sh, int n, int k)
{
    if (sh.bits == 8) {
        const int p = n / kPanelRows, kb = k / kBlockK;
        return (int)(int8_t)wq[sh.block_offset(p, kb) + int8_in_block(n % kPanelRows, k % kBlockK)];
    }
    const int rb = n >> 4, r = n & 15, g = r & 7, hi = r >> 3;
    const int tk = sh.tile_k();
    const int kt = k / tk, kk = k % tk;
    const uint8_t *tile = wq + sh.tile_offset(rb, kt);
    const int half = kk / 32, hk = kk % 32, run = hk / 16, t = (hk % 16) / 4;
    const int e = run * 4 + hk % 4;
    const int comp = half * 2 + hi;
    const uint32_t w = *reinterpret_cast<const uint32_t *>(tile + 16 * (4 * g + t) + 4 * comp);
    return (int)((w >> (4 * int4_nibble_pos(e))) & 0xFu);
}

// Zero point of row n in layout group gl.
__device__ int packed_z(const uint8_t *zeros, const Shape &sh, int n, int gl)
{
    const int p = n / kPanelRows, i = n % kPanelRows;
    const uint8_t b = zeros[((size_t)p * sh.groups() + gl) * 64 + i / 2];
    return (i & 1) ? (b >> 4) : (b & 0xF);
}

// z_out: one zero point per quantization group G of the caller ([N][K/G]).
__global__ void unpack_debug_kernel(const uint8_t *wq, const uint8_t *zeros, Shape sh, int G, int8_t *q_out,
                                    int8_t *z_out)
{
    const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    const long long total = (long long)sh.N * sh.K;
    if (idx >= total)
        return;
    const int n = (int)(idx / sh.K), k = (int)(idx % sh.K);
    q_out[idx] = (int8_t)packed_q(wq, sh, n, k);
    if (sh.bits == 4 && z_out && (k % G) == 0)
        z_out[(size_t)n * (sh.K / G) + k / G] = (int8_t)packed_z(zeros, sh, n, k / sh.group);
}

__global__ void dequant_debug_kernel(const uint8_t *wq, const uint16_t *scales, const uint8_t *zeros,
                                     Shape sh, float *w_out)
{
    const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    const long long total = (long long)sh.N * sh.K;
    if (idx >= total)
        return;
    const int n = (int)(idx / sh.K), k = (int)(idx % sh.K);
    const int q = packed_q(wq, sh, n, k);
    if (sh.bits == 8) {
        w_out[idx] = bf16_bits_to_float(scales[n]) * (float)q;
    } else {
        const int p = n / kPanelRows, i = n % kPanelRows, gl = k / sh.group;
        const float s = bf16_bits_to_float(scales[((size_t)p * sh.groups() + gl) * kPanelRows + i]);
        w_out[idx] = s * (float)(q - packed_z(zeros, sh, n, gl));
    }
}

// ---------------------------------------------------------------------------
// Host launchers
// ---------------------------------------------------------------------------
static inline unsigned nblk(long long total, int threads) { return (unsigned)((total + threads - 1) / threads); }

cudaError_t launch_quantize_int8(const float *W, int K, int N, int8_t *q, uint16_t *s, cudaStream_t st)
{
    quant_int8_kernel<<<N, 256, 0, st>>>(W, K, q, s);
    return cudaGetLastError();
}

cudaError_t launch_quantize_int4(const float *W, int K, int N, int G, uint32_t *q, uint16_t *s, uint32_t *z,
                                 cudaStream_t st)
{
    const int KG = K / G, ZW = (KG + 7) / 8;
    cudaError_t e = cudaMemsetAsync(z, 0, (size_t)N * ZW * sizeof(uint32_t), st);
    if (e != cudaSuccess)
        return e;
    const long long units = (long long)N * KG;
    quant_int4_kernel<<<nblk(units, 8), 256, 0, st>>>(W, K, N, G, q, s, z);
    return cudaGetLastError();
}

cudaError_t launch_pack_int8(const int8_t *q, const uint16_t *s, int K, int N, void *wq, void *s_out,
                             cudaStream_t st)
{
    const Shape sh{8, K, N, 0};
    const size_t n_vec = sh.weight_bytes() / 16;
    write_trailer_kernel<<<1, 1, 0, st>>>((uint8_t *)wq, sh, 0); // first: wmax_bits starts at 0
    pack_int8_kernel<<<nblk((long long)n_vec, 256), 256, 0, st>>>(q, K, N, (uint4 *)wq, n_vec, sh);
    const int total = sh.panels() * kPanelRows;
    pack_scales_int8_kernel<<<nblk(total, 256), 256, 0, st>>>(s, N, (uint16_t *)s_out, total,
                                                              const_cast<uint32_t *>(trailer_wmax(wq, sh)));
    return cudaGetLastError();
}

cudaError_t launch_pack_int4(const uint32_t *q, const uint16_t *s, const uint32_t *z, int K, int N, int G,
                             void *wq, void *s_out, void *z_out, cudaStream_t st)
{
    const Shape sh{4, K, N, layout_group(K, G)};
    const size_t n_vec = sh.weight_bytes() / 16;
    write_trailer_kernel<<<1, 1, 0, st>>>((uint8_t *)wq, sh, G); // first: wmax_bits starts at 0
    pack_int4_kernel<<<nblk((long long)n_vec, 256), 256, 0, st>>>(q, K, N, (uint4 *)wq, n_vec, sh);
    const long long total = (long long)sh.panels() * sh.groups() * kPanelRows;
    pack_sz_int4_kernel<<<nblk(total, 256), 256, 0, st>>>(s, z, K, N, G, (uint16_t *)s_out, (uint8_t *)z_out, sh,
                                                          const_cast<uint32_t *>(trailer_wmax(wq, sh)));
    return cudaGetLastError();
}

cudaError_t launch_unpack_debug(const void *wq, const void *zeros, const Shape &sh, int G, int8_t *q_out,
                                int8_t *z_out, cudaStream_t st)
{
    const long long total = (long long)sh.N * sh.K;
    unpack_debug_kernel<<<nblk(total, 256), 256, 0, st>>>((const uint8_t *)wq, (const uint8_t *)zeros, sh, G,
                                                         q_out, z_out);
    return cudaGetLastError();
}

cudaError_t launch_dequant_debug(const void *wq, const void *scales, const void *zeros, const Shape &sh,
                                 float *w_out, cudaStream_t st)
{
    const long long total = (long long)sh.N * sh.K;
    dequant_debug_kernel<<<nblk(total, 256), 256, 0, st>>>((const uint8_t *)wq, (const uint16_t *)scales,
                                                          (const uint8_t *)zeros, sh, w_out);
    return cudaGetLastError();
}

} // namespace wq
