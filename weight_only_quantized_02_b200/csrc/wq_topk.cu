// wq_topk.cu -- the vocabulary head's top-k: the k largest logits of every
// token row and their indices, for sampling ("Fused LM Head + Top-k",
// tileInfer README, Features list; the distributed variant gathers only these
// k per rank instead of the whole vocabulary).
//
// The logits come from the layer's own kernels into a scratch buffer (bf16,
// M x N, L2-resident at decode sizes: 4.9 MB for 16 tokens of a 152064-entry
// vocabulary, against 779 MB of INT8 weights); two small kernels then select:
//   part   grid (P, M): CTA (p, m) takes logits [p S, p S + S) of token m,
//          sorts them in shared memory and keeps its k largest;
//   merge  grid M: CTA m sorts the P k candidates of token m and writes the
//          k largest, descending.
// Keys are 64-bit: an order-preserving image of the binary32 value in the high
// half and the complement of the index in the low half, so a descending sort
// puts larger values first and, among equal values, the lower index first:
// the result is unique and deterministic.
#include <cstdint>

#include <cuda_bf16.h>

#include "wq.h"
#include "wq_internal.h"

namespace wq {

namespace {

constexpr int kTopkThreads = 512;

__device__ __forceinline__ unsigned long long topk_key(uint16_t bf16_bits, uint32_t index)
{
    uint32_t u = (uint32_t)bf16_bits << 16;
    if ((u << 1) == 0u)
        u = 0u; // -0 and +0 are one value (and tie on the index)
    const uint32_t ord = (u & 0x80000000u) ? ~u : (u | 0x80000000u); // monotone in the value
    return ((unsigned long long)ord << 32) | (uint32_t)~index;
}

__device__ __forceinline__ uint16_t key_value(unsigned long long key)
{
    const uint32_t ord = (uint32_t)(key >> 32);
    const uint32_t u = (ord & 0x80000000u) ? (ord ^ 0x80000000u) : ~ord;
    return (uint16_t)(u >> 16);
}

__device__ __forceinline__ int32_t key_index(unsigned long long key) { return (int32_t)~(uint32_t)key; }

// Bitonic sort of n = 2^j keys in shared memory, descending; all threads of
// the CTA call it.
__device__ void bitonic_desc(unsigned long long *s, int n)
{
    for (int size = 2; size <= n; size <<= 1) {
        for (int stride = size >> 1; stride > 0; stride >>= 1) {
            for (int i = threadIdx.x; i < (n >> 1); i += blockDim.x) {
                const int lo = 2 * i - (i & (stride - 1)), hi = lo + stride;
                const bool desc = (lo & size) == 0;
                const unsigned long long a = s[lo], b = s[hi];
                if ((a < b) == desc) {
                    s[lo] = b;
                    s[hi] = a;
                }
            }
            __syncthreads();
        }
    }
}

// CTA (p, m): the k largest keys among logits[m][p S .. min(N, p S + S)).
__global__ void __launch_bounds__(kTopkThreads) topk_part_kernel(const uint16_t *__restrict__ logits, int N, int S,
                                                                 int k, unsigned long long *__restrict__ cand)
{
    extern __shared__ unsigned long long sk[];
    const int p = blockIdx.x, m = blockIdx.y, P = gridDim.x;
    const int n0 = p * S;
    const uint16_t *row = logits + (size_t)m * N;
    for (int i = threadIdx.x; i < S; i += blockDim.x) {
        const int n = n0 + i;
        sk[i] = n < N ? topk_key(row[n], (uint32_t)n) : 0ull; // 0: below every real key
    }
    __syncthreads();
    bitonic_desc(sk, S);
    unsigned long long *out = cand + ((size_t)m * P + p) * k;
    for (int i = threadIdx.x; i < k; i += blockDim.x)
        out[i] = sk[i];
}

// CTA m: the k largest of the P k candidates of token m (padded to T = 2^j).
__global__ void __launch_bounds__(kTopkThreads) topk_merge_kernel(const unsigned long long *__restrict__ cand, int P,
                                                                  int k, int T, uint16_t *__restrict__ vals,
                                                                  int32_t *__restrict__ idx)
{
    extern __shared__ unsigned long long sk[];
    const int m = blockIdx.x;
    const unsigned long long *src = cand + (size_t)m * P * k;
    for (int i = threadIdx.x; i < T; i += blockDim.x)
        sk[i] = i < P * k ? src[i] : 0ull;
    __syncthreads();
    bitonic_desc(sk, T);
    for (int i = threadIdx.x; i < k; i += blockDim.x) {
        vals[(size_t)m * k + i] = key_value(sk[i]);
        idx[(size_t)m * k + i] = key_index(sk[i]);
    }
}

int pow2_at_least(long long v)
{
    int p = 1;
    while (p < v)
        p <<= 1;
    return p;
}

} // namespace

// Slice S (a power of two, 2048 .. 16384) such that the merge of the
// ceil(N / S) slices' k candidates fits 16384 keys (128 KB of shared memory).
bool topk_plan(int N, int k, int *S, int *P, int *T)
{
    if (N < 1 || k < 1 || k > kTopkMaxK || k > N)
        return false;
    for (int s = 2048; s <= 16384; s <<= 1) {
        const int p = (N + s - 1) / s;
        const int t = pow2_at_least((long long)p * k);
        if (t <= 16384) {
            *S = s;
            *P = p;
            *T = t;
            return true;
        }
    }
    return false;
}

size_t topk_ws_bytes(int M, int N, int k)
{
    int S, P, T;
    if (M < 1 || !topk_plan(N, k, &S, &P, &T))
        return 0;
    const size_t logits = ((size_t)M * N * 2 + 255) / 256 * 256;
    return logits + (size_t)M * P * k * sizeof(unsigned long long);
}

cudaError_t launch_topk(const uint16_t *logits, int M, int N, int k, void *cand_ws, uint16_t *vals, int32_t *idx,
                        cudaStream_t st)
{
    int S, P, T;
    if (!topk_plan(N, k, &S, &P, &T))
        return cudaErrorInvalidValue;
    cudaError_t e = kernel_setup((const void *)topk_part_kernel, (size_t)S * 8, 0, 0, nullptr);
    if (e != cudaSuccess)
        return e;
    e = kernel_setup((const void *)topk_merge_kernel, (size_t)T * 8, 0, 0, nullptr);
    if (e != cudaSuccess)
        return e;
    unsigned long long *cand = static_cast<unsigned long long *>(cand_ws);
    topk_part_kernel<<<dim3(P, M), kTopkThreads, (size_t)S * 8, st>>>(logits, N, S, k, cand);
    topk_merge_kernel<<<M, kTopkThreads, (size_t)T * 8, st>>>(cand, P, k, T, vals, idx);
    return cudaGetLastError();
}

} // namespace wq
