// wq_internal.h -- declarations shared by the C ABI and the kernel files.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_runtime_api.h>

#include "wq_layout.h"

namespace wq {

// Tokens per kernel launch; wq_linear takes up to kMaxTokens and runs longer
// inputs as consecutive chunks of kChunkTokens.
constexpr int kChunkTokens = 128;
constexpr int kMaxTokens = 65536;

struct LinearArgs {
    const uint16_t *x;
    int M, K, N;
    const void *wq, *scales, *zeros;
    int bits, group;
    uint16_t *y;
};

// Split-K workspace: [counters, 256-byte padded][partials].
// Counters: a region of fixed size, the same for every shape, so that one
// workspace serves layers of any N in turn (a smaller layer's partials never
// land on a larger layer's counters): 8 tickets per 128-row panel for up to
// kMaxN output channels (one per 16-row block; the GEMM uses the first
// panel-count entries), then two grid counters of the integer path
// (ws_grid_counter), then kResRows 64-bit residual sums of the integer
// tensor-core path's exactness guard (one per token row).  Every kernel
// leaves the counters it used at zero.  GEMM with S splits: partials
// [S][M][N].  Stream-K GEMV: partials [CTAs <= kSkMaxCtas][2][128 rows][8 *
// ceil(M/8) tokens].
constexpr int kSkMaxCtas = 512;
constexpr int kResRows = 64;
constexpr int kMaxN = 1 << 20;                     // output channels of a layer
constexpr int kCounterPanels = kMaxN / 128;
inline size_t ws_counter_words() { return (size_t)kCounterPanels * 8 + 2 + 2 * kResRows; }
inline size_t ws_counter_bytes() { return (ws_counter_words() * 4 + 255) / 256 * 256; }
inline size_t ws_grid_counter() { return (size_t)kCounterPanels * 8; } // word index of the first
inline size_t ws_res_counter() { return ws_grid_counter() + 2; }       // word index, 8-byte aligned
inline size_t ws_bytes(int M, int N, int S)
{
    return ws_counter_bytes() + (S > 1 ? (size_t)S * M * N * sizeof(float) : 0);
}
inline int gemm_token_tile(int M) { return M <= 16 ? 16 : M <= 32 ? 32 : M <= 64 ? 64 : 128; }
inline size_t ws_bytes_gemm_sk(int M, int N)
{
    return ws_counter_bytes() + (size_t)kSkMaxCtas * 2 * 128 * gemm_token_tile(M) * sizeof(float);
}
inline size_t ws_bytes_gemv_sk(int M, int N)
{
    const int tok = 8 * ((M + 7) / 8);
    return ws_counter_bytes() + (size_t)kSkMaxCtas * 2 * 128 * tok * sizeof(float);
}

// Integer tensor-core GEMMs (W8A16 and W4A16): M <= kI8MaxM, K <= kI8MaxK,
// persistent CTAs: INT8 two per SM up to 48 digit rows (16 tokens), else one,
// INT4 one, with at most kI8MaxCtas per CTA-per-SM.  Workspace: [counters]
// [digit blocks KB x NR x 128][partials: INT8 int32 (2 or 1) kI8MaxCtas x 2 x
// NR x 128, INT4 fp32 kI8MaxCtas x 2 x NR/3 x 128].
constexpr int kI8MaxM = 64;
static_assert(kI8MaxM <= kResRows, "one residual sum per token row");
constexpr int kI4MaxM = 32; // W4A16 on the integer path
constexpr int kI8MaxK = 65536;
constexpr int kI8MaxCtas = 160;
int i8_digit_rows(int M);
size_t ws_bytes_gemm_i8(int M, int K, int N);

cudaError_t launch_quantize_int8(const float *W, int K, int N, int8_t *q, uint16_t *s, cudaStream_t st);
cudaError_t launch_quantize_int4(const float *W, int K, int N, int G, uint32_t *q, uint16_t *s, uint32_t *z,
                                 cudaStream_t st);
cudaError_t launch_pack_int8(const int8_t *q, const uint16_t *s, int K, int N, void *wq, void *s_out,
                             cudaStream_t st);
cudaError_t launch_pack_int4(const uint32_t *q, const uint16_t *s, const uint32_t *z, int K, int N, int G,
                             void *wq, void *s_out, void *z_out, cudaStream_t st);
cudaError_t launch_unpack_debug(const void *wq, const void *zeros, const Shape &sh, int G, int8_t *q_out,
                                int8_t *z_out, cudaStream_t st);
cudaError_t launch_dequant_debug(const void *wq, const void *scales, const void *zeros, const Shape &sh,
                                 float *w_out, cudaStream_t st);

// GEMV: ks = K slices per 16-row block (1, 2, 4, 8); M <= 32; f16: fp16
// activations and outputs instead of bf16.
cudaError_t launch_gemv(const LinearArgs &a, int ks, int sm_count, cudaStream_t st, bool f16 = false);

// Stream-K GEMV: ctas_per_sm = 0 (occupancy) or 1/2; ws >= ws_bytes_gemv_sk.
cudaError_t launch_gemv_sk(const LinearArgs &a, int ctas_per_sm, void *ws, int sm_count, cudaStream_t st);
cudaError_t read_gemv_sk_error(int *code, cudaStream_t st);

// Allocation-free stream-K GEMV (scratch in a fixed device array of the
// library); M <= noalloc_max_m(), N <= noalloc_max_n().
cudaError_t launch_gemv_sk_noalloc(const LinearArgs &a, int sm_count, cudaStream_t st);
int noalloc_max_m();
int noalloc_max_n();

// GEMM: split = K splits (1..32); ws holds counters + partials when split > 1.
cudaError_t launch_gemm(const LinearArgs &a, int split, void *ws, int sm_count, cudaStream_t st);

// Stream-K GEMM: ctas_per_sm = 0 (default) or 1/2; ws >= ws_bytes_gemm_sk.
cudaError_t launch_gemm_sk(const LinearArgs &a, int ctas_per_sm, void *ws, int sm_count, cudaStream_t st);
cudaError_t read_gemm_sk_error(int *code, cudaStream_t st);

// Role-split W4A16 stream-K GEMM (GEMM_W4): one CTA per SM (16 warps; 20 at
// 64 tokens); ws >= ws_bytes_gemm_sk.
cudaError_t launch_gemm_w4(const LinearArgs &a, void *ws, int sm_count, cudaStream_t st);
cudaError_t read_gemm_w4_error(int *code, cudaStream_t st);

// Integer tensor-core GEMM: ws >= ws_bytes_gemm_i8 / ws_bytes_gemm_i4 (always needed).
cudaError_t launch_gemm_i8(const LinearArgs &a, void *ws, int sm_count, cudaStream_t st);
cudaError_t read_gemm_i8_error(int *code, cudaStream_t st);
size_t ws_bytes_gemm_i4(int M, int K, int N);
cudaError_t launch_gemm_i4(const LinearArgs &a, void *ws, int sm_count, cudaStream_t st);
cudaError_t read_gemm_i4_error(int *code, cudaStream_t st);

// Integer GEMV (mma.sync m16n8k32 on the packed codes): M <= kGiMaxM,
// K <= kI8MaxK, the 16-warp CTA's dynamic shared memory (digit rows, INT4
// digit sums, stash of partial sums: gi_smem_bytes) at most kGiMaxSmem;
// split 1 = one 16-warp CTA per SM, 2 = two 8-warp CTAs;
// at most kGiMaxCtas * 8 warps.  Workspace: [counters][partials
// kGiMaxCtas x 8 x 2 x 16 x NR x 4 bytes], NR = 8 * gi_ntiles(M).
constexpr int kGiMaxM = 8;
constexpr int kGiMaxCtas = 448;
constexpr int kGiMaxSmem = 226 * 1024;
int gi_ntiles(int M);
size_t gi_smem_bytes(int bits, int M, int K);
bool gi_fits(int bits, int M, int K);
size_t ws_bytes_gemv_i8(int M, int K, int N);
cudaError_t launch_gemv_i8(const LinearArgs &a, int split, void *ws, int sm_count, cudaStream_t st);

// Top-k of the vocabulary head (wq_topk.cu): k <= kTopkMaxK.  topk_plan
// picks the slice S (P slices, merge of T keys); topk_ws_bytes is the
// scratch of wq_linear_topk (bf16 logits M x N, then M x P x k candidates);
// launch_topk selects from logits already in that scratch.
constexpr int kTopkMaxK = 64;
bool topk_plan(int M, int N, int k, int *S, int *P, int *T);
size_t topk_ws_bytes(int M, int N, int k);
cudaError_t launch_topk(const uint16_t *logits, int M, int N, int k, void *cand_ws, uint16_t *vals, int32_t *idx,
                        cudaStream_t st);

// Launch preparation of one kernel on the current device: raises its
// dynamic shared-memory limit to smem_optin bytes (0: leave it) the first
// time it is launched on that device, and returns in *occ (if not NULL) its
// resident CTAs per SM for `threads` threads and `smem` bytes of dynamic
// shared memory (at least 1).  Both are cached per (device, kernel), under a
// mutex: a kernel attribute belongs to one device's context, so a launch on a
// second device repeats the set-up there.
cudaError_t kernel_setup(const void *func, size_t smem_optin, int threads, size_t smem, int *occ);

// Reads and clears the device error word of the current device.
cudaError_t read_device_error(int *code, cudaStream_t st);

// A bounded wait that runs out (limit_ns) and records the timeout.
cudaError_t launch_wait_selftest(uint64_t limit_ns, cudaStream_t st);

} // namespace wq
