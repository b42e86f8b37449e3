// wq_topk.cu -- the vocabulary head's top-k: the k largest logits of every
// token row and their indices, for sampling ("Fused LM Head + Top-k",
// tileInfer README, Features list; the distributed variant gathers only these
// k per rank instead of the whole vocabulary).
//
// The logits come from the layer's own kernels into a scratch buffer (bf16,
// M x N, L2-resident at decode sizes: 4.9 MB for 16 tokens of a 152064-entry
// vocabulary, against 779 MB of INT8 weights); two small kernels then select:
//   part   grid (P, M): CTA (p, m) takes logits [p S, p S + S) of token m and
//          keeps its k largest, in index order;
//   merge  grid M: CTA m takes the P k candidates of token m (in index
//          order, since the slices are) and writes the k largest, descending.
// Both select with a radix select on 16-bit order-preserving keys (a bf16
// logit has 16 bits): two passes of an 8-bit histogram find the k-th
// largest key t exactly; every key above t is kept, and of the keys equal
// to t the ones with the lowest indices, found by an order-preserving
// compaction.  The k survivors of the merge are sorted (descending value,
// then ascending index), so the result is unique and deterministic: ties
// between equal logits go to the lower index.
#include <cstdint>

#include <cuda_bf16.h>

#include "wq.h"
#include "wq_device.cuh"
#include "wq_internal.h"

namespace wq {

namespace {

constexpr int kTopkThreads = 512;
constexpr int kTopkWarps = kTopkThreads / 32;
// Logits per part CTA: 4096, or 8192 where the grid of 4096-logit slices
// would not fit the GPU at once (four CTAs per SM).
constexpr int kPartSlice = 4096, kPartSliceWide = 8192;
constexpr long long kTopkWaveCtas = 4 * 148; // four 512-thread CTAs on each of a B200's 148 SMs

// bf16 bits -> a 16-bit key that orders like the value (-0 and +0 equal).
__device__ __forceinline__ uint32_t order16(uint16_t b)
{
    if ((b & 0x7FFFu) == 0)
        b = 0;
    return (b & 0x8000u) ? (uint32_t)(~b & 0xFFFFu) : (uint32_t)(b | 0x8000u);
}

__device__ __forceinline__ uint16_t value16(uint32_t key16)
{
    return (uint16_t)((key16 & 0x8000u) ? (key16 & 0x7FFFu) : (~key16 & 0xFFFFu));
}

// Exact k-th largest of the n keys in s (16-bit keys), by two 8-bit passes;
// every thread of the CTA calls it.  Returns t and, in *ties, how many keys
// equal to t belong to the k largest.
template <typename Key>
__device__ uint32_t radix_select16(const Key *s, int n, int k, uint32_t *hist, int *ties)
{
    __shared__ uint32_t s_prefix;
    __shared__ int s_rank;
    __shared__ int s_wsum[8], c_bin[256], c_inc[256];
    uint32_t *wh = hist + (threadIdx.x >> 5) * 256; // one 256-bin histogram per warp
    if (threadIdx.x == 0) {
        s_prefix = 0;
        s_rank = k;
    }
    for (int pass = 1; pass >= 0; --pass) {
        for (int i = threadIdx.x; i < kTopkWarps * 256; i += blockDim.x)
            hist[i] = 0;
        __syncthreads();
        const uint32_t prefix = s_prefix, shift = 8 * pass;
        const uint32_t hi_mask = pass == 1 ? 0u : 0xFF00u;
        // one histogram per warp spreads the contention of the few bins
        // that logits crowd into
        for (int i = threadIdx.x; i < n; i += blockDim.x) {
            const uint32_t key = s[i];
            if ((key & hi_mask) == prefix)
                atomicAdd(&wh[(key >> shift) & 0xFFu], 1u);
        }
        __syncthreads();
        // fold the warp histograms and find the digit holding the rank-th
        // largest key: thread j takes bin 255 - j, so an inclusive scan over
        // the threads counts the keys at or above each bin, and exactly one
        // bin has the rank-th largest between its exclusive and inclusive
        // counts (the selected keys number at least the rank)
        const int rank = s_rank;
        if (threadIdx.x < 256) {
            const int d = 255 - (int)threadIdx.x, lane = threadIdx.x & 31;
            int c = 0;
            for (int w = 0; w < kTopkWarps; ++w)
                c += (int)hist[w * 256 + d];
            int inc = c;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int u = __shfl_up_sync(0xffffffffu, inc, o);
                if (lane >= o)
                    inc += u;
            }
            if (lane == 31)
                s_wsum[threadIdx.x >> 5] = inc;
            c_bin[threadIdx.x] = c;
            c_inc[threadIdx.x] = inc;
        }
        __syncthreads();
        if (threadIdx.x < 256) {
            int inc = c_inc[threadIdx.x];
            for (int w = 0; w < (int)(threadIdx.x >> 5); ++w)
                inc += s_wsum[w];
            const int exc = inc - c_bin[threadIdx.x];
            if (exc < rank && inc >= rank) {
                s_rank = rank - exc;
                s_prefix = prefix | ((uint32_t)(255 - threadIdx.x) << shift);
            }
        }
        __syncthreads();
    }
    *ties = s_rank;
    return s_prefix;
}

// Keeps the k largest of the n keys of s (index i of s is global index
// gidx[i], or base + i when gidx is null), in index order: the keys above t
// and the first `ties` keys equal to t.  Writes 64-bit keys (value key << 48
// | ~index) to out[0..k).  Warp w takes the keys [w span, (w + 1) span), 32
// consecutive keys at a time, so the ballots of the lanes, the chunks in
// turn and the warp totals scanned in warp order give every survivor its
// position in index order; lanes read consecutive keys (no bank conflicts).
// scratch: 2 * kTopkWarps ints.
template <typename Key>
__device__ void compact_topk(const Key *s, int n, int k, uint32_t t, int ties, const uint32_t *gidx,
                             uint32_t base, unsigned long long *out, int *scratch)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int span = (n + kTopkWarps - 1) / kTopkWarps;
    const int w0 = min(n, warp * span), w1 = min(n, w0 + span);
    int ca = 0, ce = 0;
    for (int i0 = w0; i0 < w1; i0 += 32) {
        const int i = i0 + lane;
        const uint32_t key = i < w1 ? (uint32_t)s[i] : 0u;
        ca += __popc(__ballot_sync(0xffffffffu, i < w1 && key > t));
        ce += __popc(__ballot_sync(0xffffffffu, i < w1 && key == t));
    }
    if (lane == 0) {
        scratch[warp] = ca;
        scratch[kTopkWarps + warp] = ce;
    }
    __syncthreads();
    int pa = 0, pe = 0; // keys above t / equal to t before this warp's range
    for (int w = 0; w < warp; ++w) {
        pa += scratch[w];
        pe += scratch[kTopkWarps + w];
    }
    const uint32_t lt = (1u << lane) - 1u;
    for (int i0 = w0; i0 < w1; i0 += 32) {
        const int i = i0 + lane;
        const uint32_t key = i < w1 ? (uint32_t)s[i] : 0u;
        const bool above = i < w1 && key > t, equal = i < w1 && key == t;
        const uint32_t ma = __ballot_sync(0xffffffffu, above), me = __ballot_sync(0xffffffffu, equal);
        const int ra = pa + __popc(ma & lt), re = pe + __popc(me & lt);
        int pos = -1;
        if (above) // above-t keys and the kept ties interleave in index order
            pos = ra + min(re, ties);
        else if (equal && re < ties)
            pos = ra + re;
        if (pos >= 0 && pos < k)
            out[pos] = ((unsigned long long)key << 48) | (uint32_t)~(gidx ? gidx[i] : base + (uint32_t)i);
        pa += __popc(ma);
        pe += __popc(me);
    }
    __syncthreads(); // scratch reusable
}

// CTA (p, m): the k largest logits of token m among [p S, p S + S) -> cand.
template <int S>
__global__ void __launch_bounds__(kTopkThreads) topk_part_kernel(const uint16_t *__restrict__ logits, int N, int k,
                                                                 unsigned long long *__restrict__ cand)
{
    __shared__ uint16_t s_key[S];
    __shared__ uint32_t s_hist[kTopkWarps * 256];
    __shared__ int s_scan[2 * kTopkWarps];
    const int p = blockIdx.x, m = blockIdx.y, P = gridDim.x;
    const int n0 = p * S, n = min(S, N - n0);
    const uint16_t *row = logits + (size_t)m * N + n0;
    pdl_launch_dependents(); // the merge may launch; it waits for this grid before reading
    pdl_wait();              // the logits come from the preceding kernel
    { // every thread's logits in flight together, then their keys
        constexpr int J = S / kTopkThreads;
        uint16_t v[J];
#pragma unroll
        for (int j = 0; j < J; ++j) {
            const int i = threadIdx.x + j * kTopkThreads;
            v[j] = i < n ? row[i] : (uint16_t)0;
        }
#pragma unroll
        for (int j = 0; j < J; ++j) {
            const int i = threadIdx.x + j * kTopkThreads;
            if (i < n)
                s_key[i] = (uint16_t)order16(v[j]);
        }
    }
    __syncthreads();
    unsigned long long *out = cand + ((size_t)m * P + p) * k;
    const int kk = min(k, n);
    int ties = 0;
    const uint32_t t = radix_select16(s_key, n, kk, s_hist, &ties);
    compact_topk(s_key, n, kk, t, ties, nullptr, (uint32_t)n0, out, s_scan);
    for (int i = kk + threadIdx.x; i < k; i += blockDim.x)
        out[i] = 0ull; // a slice shorter than k: padding below every real key
}

// CTA m: the k largest of the P k candidates of token m, sorted.
__global__ void __launch_bounds__(kTopkThreads) topk_merge_kernel(const unsigned long long *__restrict__ cand, int P,
                                                                  int k, uint16_t *__restrict__ vals,
                                                                  int32_t *__restrict__ idx)
{
    extern __shared__ uint32_t sm[];
    const int C = P * k;
    uint32_t *s_key = sm, *s_idx = sm + C;                              // [C] each
    uint32_t *s_hist = s_idx + C;                                       // [kTopkWarps * 256]
    int *s_scan = reinterpret_cast<int *>(s_hist + kTopkWarps * 256); // [2 * kTopkWarps]
    __shared__ unsigned long long s_best[kTopkMaxK];
    const int m = blockIdx.x;
    const unsigned long long *src = cand + (size_t)m * C;
    pdl_launch_dependents();
    pdl_wait(); // the candidates come from the part kernel
#pragma unroll 4
    for (int i = threadIdx.x; i < C; i += blockDim.x) {
        const unsigned long long c = __ldcg(src + i);
        s_key[i] = (uint32_t)(c >> 48); // padding (0) is below every real key
        s_idx[i] = ~(uint32_t)c;
    }
    for (int i = threadIdx.x; i < kTopkMaxK; i += blockDim.x)
        s_best[i] = 0ull; // slots past k: below every real key, so the sort below keeps them last
    __syncthreads();
    int ties = 0;
    const uint32_t t = radix_select16(s_key, C, k, s_hist, &ties);
    compact_topk(s_key, C, k, t, ties, s_idx, 0u, s_best, s_scan);
    __syncthreads();
    if (threadIdx.x < 32) { // bitonic sort of the 64 slots, descending, one warp
        for (int size = 2; size <= kTopkMaxK; size <<= 1)
            for (int stride = size >> 1; stride > 0; stride >>= 1) {
                const int i = threadIdx.x; // 32 pairs
                const int lo = 2 * i - (i & (stride - 1)), hi = lo + stride;
                const bool desc = (lo & size) == 0;
                const unsigned long long a = s_best[lo], b = s_best[hi];
                if ((a < b) == desc) {
                    s_best[lo] = b;
                    s_best[hi] = a;
                }
                __syncwarp();
            }
    }
    __syncthreads();
    for (int i = threadIdx.x; i < k; i += blockDim.x) {
        const unsigned long long key = s_best[i];
        vals[(size_t)m * k + i] = value16((uint32_t)(key >> 48));
        idx[(size_t)m * k + i] = (int32_t)~(uint32_t)key;
    }
}

size_t merge_smem(int P, int k) { return (size_t)2 * P * k * 4 + kTopkWarps * 256 * 4 + 2 * kTopkWarps * 4; }

} // namespace

// P slices of S logits; the merge holds P k candidates in shared memory (at
// most 200 KB).
bool topk_plan(int M, int N, int k, int *S, int *P, int *T)
{
    if (M < 1 || N < 1 || k < 1 || k > kTopkMaxK || k > N)
        return false;
    const int narrow = (N + kPartSlice - 1) / kPartSlice;
    const int sl = (long long)narrow * M <= kTopkWaveCtas ? kPartSlice : kPartSliceWide;
    const int p = (N + sl - 1) / sl;
    if (merge_smem(p, k) > 200 * 1024)
        return false;
    *S = sl;
    *P = p;
    *T = p * k;
    return true;
}

size_t topk_ws_bytes(int M, int N, int k)
{
    int S, P, T;
    if (!topk_plan(M, N, k, &S, &P, &T))
        return 0;
    const size_t logits = ((size_t)M * N * 2 + 255) / 256 * 256;
    return logits + (size_t)M * P * k * sizeof(unsigned long long);
}

cudaError_t launch_topk(const uint16_t *logits, int M, int N, int k, void *cand_ws, uint16_t *vals, int32_t *idx,
                        cudaStream_t st)
{
    int S, P, T;
    if (!topk_plan(M, N, k, &S, &P, &T))
        return cudaErrorInvalidValue;
    const size_t msm = merge_smem(P, k);
    cudaError_t e = kernel_setup((const void *)topk_merge_kernel, msm, 0, 0, nullptr);
    if (e != cudaSuccess)
        return e;
    unsigned long long *cand = static_cast<unsigned long long *>(cand_ws);
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cfg.stream = st;
    cfg.gridDim = dim3(P, M);
    cfg.blockDim = dim3(kTopkThreads);
    e = S == kPartSlice ? cudaLaunchKernelEx(&cfg, topk_part_kernel<kPartSlice>, logits, N, k, cand)
                        : cudaLaunchKernelEx(&cfg, topk_part_kernel<kPartSliceWide>, logits, N, k, cand);
    if (e != cudaSuccess)
        return e;
    cfg.gridDim = dim3(M);
    cfg.dynamicSmemBytes = msm;
    return cudaLaunchKernelEx(&cfg, topk_merge_kernel, (const unsigned long long *)cand, P, k, vals, idx);
}

} // namespace wq
