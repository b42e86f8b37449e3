/*
 * wq.h -- C ABI of the weight-only quantized linear layer for LLM decode on
 * NVIDIA B200 (sm_100a).
 *
 *     y[M][N] = x[M][K] . dequant(Wq)^T        (bf16 in, bf16 out)
 *
 * Two weight formats:
 *   W8A16  int8 weights, one bf16 scale per output channel, no zero point:
 *          w[n][k] = s[n] * q[n][k]
 *          ("Per-channel W8A16 quantization", tileInfer README, Features
 *          table.)
 *   W4A16  unsigned 4-bit weights q in [0,15] with a bf16 scale and a 4-bit
 *          zero point per (group of `group` consecutive k, output channel;
 *          group 32, 64, 128, or K for one pair per output channel):
 *          w[n][k] = s[n][k/group] * (q[n][k] - z[n][k/group])
 *          (A WnA16 kernel shared by several checkpoint formats needs the same
 *          layout, scales, zero points and group size. This is the review of
 *          Figure 4 in "Toward a Cleaner Quantization Stack in SGLang".)
 *
 * Four kernel families sit behind one call:
 *   - a GEMV for decode-sized M, with register-level dequantization and
 *     128-bit weight loads (the GEMV row of the tileInfer README, Features
 *     table). Its fp32 dot products run on mma.sync tensor-core fragments.
 *   - a small-M GEMM (tcgen05 tensor cores, accumulators in tensor memory)
 *     with split-K and a fixed-order fp32 reduction ("split_k" auto-tuning,
 *     Mit han lab Llm awq Kernel Selection Thresholds, The Insight).
 *   - on the integer tensor cores (tcgen05 kind::i8): W8A16 (M <= 64) on the
 *     raw INT8 codes, W4A16 (M <= 32) on the exact integers q - z. The per-channel scale factors out of the k sum, x is
 *     written per token row as an integer X = round(x * 2^e), ties to even,
 *     with e = min(21 - E, 127) for 2^E <= max|x| < 2^(E+1), so |X| < 2^22
 *     (three base-256 digits) and every element within 2^14 of the row's
 *     largest is exact. The sums over k are exact int32, and
 *     y = s * 2^-e * sum is formed in binary64 before the bf16 rounding.
 *   - the integer GEMV (M <= 8): the same integer sums on mma.sync
 *     m16n8k32 s8 fragments taken straight from the packed codes; for
 *     W4A16 the zero point enters through the activations' digit sum per
 *     group and the group scale is applied in fp32 per group.
 * A per-(M,K,N,bits,group) dispatcher picks the kernel and split factor. It
 * starts from an untuned rule (the page's threshold: fewer than 8 tokens ->
 * a GEMV, else a GEMM; within each, the kernel measured fastest on B200 where
 * the workspace allows it: the integer GEMV; the integer tensor-core GEMM for
 * W8A16 up to 64 tokens, the role-split GEMM for W4A16; else the stream-K or
 * row-block GEMV and the split-8 GEMM) and is overridden by measured timings
 * (wq_tune).
 *
 * Conventions for every entry point:
 *   - The return value is a wq_status: 0 on success, negative on error.
 *     No call aborts, traps or throws.
 *   - "device" pointers are CUDA device pointers on the current device.
 *     "host" pointers are ordinary host memory.
 *   - The caller owns every buffer. No call allocates device memory, except
 *     wq_tune, which allocates and frees its timing events and rotation
 *     copies of the packed weights (about three L2 sizes, at least two
 *     copies).
 *   - Work is enqueued on `stream` (0 = legacy default stream). Calls return
 *     after the enqueue, with no implicit synchronization, unless the entry
 *     says "synchronizes".
 *   - bf16 values are passed as their uint16_t bit patterns.
 *   - Shape rules: 1 <= N <= 1048576, N % 16 == 0. W8A16: group == 0,
 *     K % 32 == 0.
 *     W4A16: K % 128 == 0 and group 32, 64, 128 or K (per channel: one
 *     scale and zero point per output row). 1 <= M <= 65536; a kernel takes
 *     at most 128 tokens (32 for groups of 32 and 64 k, which run on the
 *     row-block GEMV only), and wq_linear runs a larger M (prefill) as
 *     consecutive chunks.
 *     x, y and every packed buffer must be 16-byte aligned.
 *   - Packed buffers are written by wq_pack_int8 / wq_pack_int4 and are
 *     opaque. wq_packed_bytes gives their sizes. Their layout is described
 *     in the library's design notes.
 */
#ifndef WQ_H
#define WQ_H

#include <stddef.h>
#include <stdint.h>

#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    WQ_OK = 0,
    WQ_ERR_NULL = -1,      /* a required pointer is NULL */
    WQ_ERR_SHAPE = -2,     /* M, K or N outside the shape rules */
    WQ_ERR_ALIGN = -3,     /* a pointer is not 16-byte aligned */
    WQ_ERR_GROUP = -4,     /* unsupported bits / group combination */
    WQ_ERR_HEADER = -5,    /* packed trailer does not match the arguments */
    WQ_ERR_WORKSPACE = -6, /* split > 1 needs a larger split-K workspace */
    WQ_ERR_CUDA = -7,      /* a CUDA runtime call or a launch failed */
    WQ_ERR_TUNING = -8,    /* tuning file unreadable or malformed */
    WQ_ERR_TIMEOUT = -9,   /* a bounded device-side wait gave up */
    WQ_ERR_ARCH = -10,     /* device is not sm_100 (B200 class) */
    WQ_ERR_VARIANT = -11   /* forced variant / split not valid for the shape */
} wq_status;

/* Kernel variants (wq_linear_forced, wq_get_choice). */
#define WQ_VARIANT_AUTO (-1)
#define WQ_VARIANT_GEMV 0    /* stream-K GEMV, M <= 32: TMA-fed ring, mma.sync; needs the workspace */
#define WQ_VARIANT_GEMM 1    /* tcgen05 split-K GEMM, M <= 128 */
#define WQ_VARIANT_GEMV_RB 2 /* row-block GEMV, M <= 32, direct 128-bit loads; no workspace */
#define WQ_VARIANT_GEMM_SK 3 /* stream-K tcgen05 GEMM, M <= 128, persistent; needs the workspace */
#define WQ_VARIANT_I8MMA 4   /* stream-K tcgen05 kind::i8: W8A16 (M <= 64) on the raw codes,
                                W4A16 (M <= 32) on q - z; K <= 65536; needs the workspace */
#define WQ_VARIANT_GEMV_I8 5 /* GEMV on mma.sync m16n8k32 s8 (the packed codes as they are,
                                activations as exact digits in shared memory): each CTA owns whole
                                16-row blocks, the rest are cut stream-K style across CTAs; M <= 8,
                                3 * M * K bytes of digits plus 16-48 KB of partial sums <= 226 KB;
                                split 1 = one 16-warp CTA per SM, 2 = two 8-warp CTAs per SM; needs
                                the workspace */
#define WQ_VARIANT_GEMM_W4 6 /* W4A16 only, M <= 128: stream-K tcgen05 GEMM with one CTA per SM
                                (16 warps; 20 at 64 tokens), every role (weight and x loads, dequantization, MMA, group
                                rescale) on its own warps with its own ring; needs the workspace */

/* Static description of a status code. Host. Never NULL. */
const char *wq_strerror(int status);

/* Library version: major * 10000 + minor * 100 + patch. Host. */
int wq_version(void);

/* Byte sizes of the three packed buffers for a weight of shape [N][K].
 * bits = 8 (group must be 0) or 4 (group 32, 64, 128 or K; per channel,
 * group K, is stored as group 128 with each row's scale and zero point
 * repeated in every 128-k block, so it runs on every kernel). zero_bytes is 0 for
 * INT8. Any output pointer may be NULL. Host, no device work. */
int wq_packed_bytes(int bits, int K, int N, int group, size_t *wq_bytes,
                    size_t *scale_bytes, size_t *zero_bytes);

/* ---------------------------------------------------------------------
 * Quantizers: fp32 source weights -> canonical quantized tensors.
 * These are how the workloads' weights are made. They are not the layer
 * itself. Every decision is taken in binary64, as in the CPU oracle, so
 * the codes are bit-exact with it.
 * ------------------------------------------------------------------- */

/* Symmetric per-output-channel INT8 (per-channel W8A16, tileInfer README,
 * Features table).
 *   W       device, fp32 [N][K], row-major
 *   q_out   device, int8 [N][K]
 *   s_out   device, bf16 [N]:  s = bf16_rne(max_k |W[n][k]| / 127)
 *   q = clamp(rint(W / s), -127, 127), ties to even. A row with s == 0 gets q = 0.
 * One CUDA block per row. */
int wq_quantize_int8(const float *W, int K, int N, int8_t *q_out, uint16_t *s_out,
                     cudaStream_t stream);

/* Asymmetric INT4 with `group` consecutive k per scale / zero point.
 *   W       device, fp32 [N][K]
 *   q_out   device, uint32 [N][K/8]; nibble j of word (n,c) = q[n][8c+j]
 *   s_out   device, bf16 [N][K/group]: s = bf16 rounded toward +inf of
 *           (hi - lo) / 15, where lo = min(min W, 0) and hi = max(max W, 0)
 *   z_out   device, uint32 [N][ceil(K/group/8)]; nibble j of word (n,c) is
 *           z[n][8c+j] = clamp(rint(-lo / s), 0, 15). Unused nibbles are 0.
 *   q = clamp(rint(W / s) + z, 0, 15). A group with hi == lo gets s = z = q = 0. */
int wq_quantize_int4(const float *W, int K, int N, int group, uint32_t *q_out,
                     uint16_t *s_out, uint32_t *z_out, cudaStream_t stream);

/* ---------------------------------------------------------------------
 * Packers: canonical tensors -> the GPU layout read by every kernel.
 * Packing is a separate step from running the layer: the scheme-vs-kernel
 * split of "Toward a Cleaner Quantization Stack in SGLang", Figure 1.
 * ------------------------------------------------------------------- */

/* q: device int8 [N][K]; scales: device bf16 [N].
 * wq_out / scales_out: device buffers of wq_packed_bytes(8, K, N, 0, ...). */
int wq_pack_int8(const int8_t *q, const uint16_t *scales, int K, int N, void *wq_out,
                 void *scales_out, cudaStream_t stream);

/* q: device uint32 [N][K/8] (low nibble first); scales: device bf16
 * [N][K/group]; zeros: device uint32 [N][ceil(K/group/8)].
 * Outputs sized by wq_packed_bytes(4, K, N, group, ...). */
int wq_pack_int4(const uint32_t *q, const uint16_t *scales, const uint32_t *zeros, int K,
                 int N, int group, void *wq_out, void *scales_out, void *zeros_out,
                 cudaStream_t stream);

/* Reads the 64-byte trailer that the packers write after the packed weights
 * and checks it against (bits, K, N, group). Returns WQ_ERR_HEADER on a
 * mismatch. Synchronizes `stream`, so call it once at load time, not per
 * step. */
int wq_check_packed(const void *Wq, int bits, int K, int N, int group, cudaStream_t stream);

/* ---------------------------------------------------------------------
 * The layer.
 * ------------------------------------------------------------------- */

/* y = x . dequant(Wq)^T.
 *   x       device, bf16 [M][K], row-major, 16-byte aligned
 *   Wq, scales, zeros   device, packed by wq_pack_int8 / wq_pack_int4
 *           (zeros = NULL for INT8)
 *   group   0 for INT8 per-channel, 128 for INT4
 *   y       device, bf16 [M][N], row-major, 16-byte aligned. Every element
 *           is written: bf16_rne of the fp32-accumulated sum.
 * The kernel and split factor come from the dispatcher (tuned table, else
 * the default rule).  M > 128 runs as chunks of 128 tokens (the last one
 * ragged), one kernel each, in order on the stream, each streaming the
 * weights once and each with the dispatcher's choice for its own size; if a
 * chunk fails its status is returned and the chunks before it stay
 * enqueued. The stream-K kernels, the integer path and a GEMM
 * split > 1 use the workspace registered with wq_set_workspace for the
 * current device. With no workspace (or too small a one), decode-sized M
 * falls back to the row-block GEMV and the GEMM runs unsplit, so wq_linear
 * never fails for lack of workspace. Calls that share a workspace must not overlap on the
 * GPU (keep them on one stream). */
int wq_linear(const uint16_t *x, int M, int K, const void *Wq, const void *scales,
              const void *zeros, int group, int N, uint16_t *y, cudaStream_t stream);

/* wq_linear with fp16 activations and fp16 outputs (x fp16 [M][K], y fp16
 * [M][N], as their uint16_t bit patterns; the packed weights and their bf16
 * scales are the same).  Runs the row-block GEMV, 32 tokens per launch, with
 * the dequantized weights as exact fp16 integers and fp32 accumulation; y is
 * rounded to fp16, to nearest even.  The FP16 half of the validation matrix
 * of the Marlin register and launch scheduling benchmark, "Validation and
 * limits".  1 <= M <= 65536; other rules as wq_linear.  Needs no workspace. */
int wq_linear_f16(const uint16_t *x, int M, int K, const void *Wq, const void *scales,
                  const void *zeros, int group, int N, uint16_t *y, cudaStream_t stream);

/* wq_linear with an explicit kernel variant (WQ_VARIANT_*) and split factor.
 * variant = WQ_VARIANT_AUTO, or split = 0, leaves that choice to the dispatcher.
 * GEMV: split = CTAs per SM, 1..4, capped by occupancy (the K range of
 *       every CTA is set by the stream-K partition).
 * GEMV_RB: split = K-slices per 16-row block, one of 1, 2, 4, 8.
 * GEMM_SK: split = CTAs per SM, 1 or 2, capped by the tile's resources.
 * GEMM: split = K-splits, 1 <= split <= min(32, ceil(K/128)).
 * I8MMA: split = 1 (one persistent CTA per SM).
 * GEMV_I8: split = 1 (one 16-warp CTA per SM) or 2 (two 8-warp CTAs per SM).
 * GEMM_W4: split = 1.
 * Returns WQ_ERR_VARIANT if the pair does not fit the shape. */
int wq_linear_forced(const uint16_t *x, int M, int K, const void *Wq, const void *scales,
                     const void *zeros, int group, int N, uint16_t *y, int variant, int split,
                     cudaStream_t stream);

/* wq_linear_forced with an explicit split-K workspace, for callers that run
 * several layers on concurrent streams (ws = NULL: the registered one). */
int wq_linear_ex(const uint16_t *x, int M, int K, const void *Wq, const void *scales,
                 const void *zeros, int group, int N, uint16_t *y, int variant, int split,
                 void *ws, size_t ws_bytes, cudaStream_t stream);

/* wq_linear for callers that cannot allocate device memory when they run
 * the layer: code inside a captured CUDA graph or an allocator's critical
 * section, runtimes whose device memory is pre-partitioned, and plugin hosts
 * that hand over only input and output buffers. The pages have no
 * counterpart; this entry exists for those callers.
 * It runs the stream-K GEMV. Its tickets and partial sums sit in a fixed
 * array of about 4 MiB inside the library's device image. Every GPU that
 * loads the library holds that array until the process exits. No call here
 * allocates or frees memory.
 *   Limits: 1 <= M <= 8 and N <= 262144. Larger shapes return WQ_ERR_SHAPE
 *   before anything is enqueued. Other arguments are as for wq_linear.
 *   The first call on a device looks up the array's device address (with
 *   that device current). Make that first call before any stream capture.
 *   Every call shares the array and enqueues a small memset of its tickets,
 *   so calls that overlap on the GPU race: keep them on one stream. */
int wq_linear_noalloc(const uint16_t *x, int M, int K, const void *Wq, const void *scales,
                      const void *zeros, int group, int N, uint16_t *y, cudaStream_t stream);

/* The vocabulary head's top-k for sampling ("Fused LM Head + Top-k",
 * tileInfer README, Features list): for every token row m the k largest
 * logits of y = x . dequant(Wq)^T and their indices, without returning y.
 *   vals    device, bf16 [M][k]: the k largest logits of row m, descending
 *   idx     device, int32 [M][k]: their output indices; among equal logits
 *           the lower index comes first, so the result is unique
 *   ws      device scratch of at least wq_topk_workspace_bytes(M, N, k)
 *           bytes, 16-byte aligned, owned by the caller (the logits pass
 *           through it as bf16, then the candidates of the selection)
 *   1 <= M <= 128, 1 <= k <= 64, k <= N; other arguments as wq_linear.
 * The logits come from the dispatcher's kernel (with the workspace
 * registered by wq_set_workspace, as wq_linear); two selection kernels
 * follow on the same stream.  Returns WQ_ERR_SHAPE outside the limits,
 * WQ_ERR_WORKSPACE for a scratch that is too small. */
int wq_linear_topk(const uint16_t *x, int M, int K, const void *Wq, const void *scales,
                   const void *zeros, int group, int N, int k, uint16_t *vals, int32_t *idx,
                   void *ws, size_t ws_bytes, cudaStream_t stream);

/* Scratch bytes of wq_linear_topk; 0 for arguments out of its limits. Host. */
size_t wq_topk_workspace_bytes(int M, int N, int k);

/* Bytes of workspace for M tokens, a K x N weight and GEMM splits up to
 * max_split: enough for every variant of that shape (M > 128: of its
 * 128-token chunks, which share the workspace one after another). It holds
 * a counter region of the same size for every shape (257 KiB: eight ticket
 * counters per 128-channel panel of the largest N, then the integer path's
 * grid counters and residual sums), so one workspace sized for the largest
 * of several layers serves them all in turn, and after it the largest of
 * the GEMM's fp32 partials [split][M][N], the stream-K kernels' per-CTA
 * panel partials, the integer path's int32 per-CTA partials, and the
 * integer GEMV's per-warp partials. Returns 0 for M, K, N or max_split < 1.
 * Host. */
size_t wq_workspace_bytes(int M, int K, int N, int max_split);

/* Registers a caller-owned device workspace for the current device, used by
 * wq_linear. Zeroes its counters with a synchronous cudaMemset. The kernels
 * leave the counters at zero after every call. ws = NULL unregisters. */
int wq_set_workspace(void *ws, size_t bytes);

/* ---------------------------------------------------------------------
 * Dispatcher / tuner. The table is keyed by (device name, SM count, M, K, N,
 * bits, group) and guarded by a mutex.
 * ------------------------------------------------------------------- */

/* Times every valid (variant, split) for the shape with CUDA events, as
 * decode runs it: R copies of the packed weights (R >= 2, spanning about
 * three L2 sizes, so no call finds its weights in L2) are called back to
 * back in rotation with the caller's x and y; `warmup` untimed and `iters`
 * timed rotations per candidate, per-call time = rotation time / R. It
 * keeps the fastest by the mean of the middle half of its sorted times. On an exact tie the later, larger
 * split wins, as in the split_k auto-tune loop of Mit han lab Llm awq Kernel
 * Selection Thresholds, The Insight. Overwrites y. Synchronizes `stream`.
 * Needs a registered workspace that fits split 32 to try every split.
 * M > 128 tunes the 128-token chunk shape on the first 128 rows of x. */
int wq_tune(const uint16_t *x, int M, int K, const void *Wq, const void *scales,
            const void *zeros, int group, int N, uint16_t *y, int warmup, int iters,
            cudaStream_t stream);

/* The (variant, split) that wq_linear would use for this shape now (M > 128:
 * for its full 128-token chunks). Host. */
int wq_get_choice(int M, int K, int N, int bits, int group, int *variant, int *split);

/* Sets one table entry by hand (for tests and offline tables). Host. */
int wq_set_choice(int M, int K, int N, int bits, int group, int variant, int split);

/* Drops every tuned entry. Host. */
int wq_clear_tuning(void);

/* Text file, one entry per line. Host. WQ_ERR_TUNING on a malformed line;
 * in that case the table is left unchanged.
 * The environment variable WQ_TUNING_FILE names a table that is loaded the
 * same way when the library is loaded. If it cannot be read or parsed,
 * every automatic choice (wq_linear; wq_linear_forced and wq_linear_ex
 * with WQ_VARIANT_AUTO; wq_get_choice) returns WQ_ERR_TUNING; forced
 * variants still run. */
int wq_save_tuning(const char *path);
int wq_load_tuning(const char *path);

/* ---------------------------------------------------------------------
 * Debug views of the packed layout (for the bit-exact tests).
 * ------------------------------------------------------------------- */

/* Unpacks the packed weights to integers: q_out int8 [N][K] (INT4: 0..15;
 * INT8: -128..127) and, for INT4, z_out int8 [N][K/group]. Device pointers. */
int wq_unpack_debug(const void *Wq, const void *zeros, int bits, int K, int N, int group,
                    int8_t *q_out, int8_t *z_out, cudaStream_t stream);

/* Dequantized weights in fp32, w_out [N][K]. s*(q - z) is exact in fp32. */
int wq_dequant_debug(const void *Wq, const void *scales, const void *zeros, int bits, int K,
                     int N, int group, float *w_out, cudaStream_t stream);

/* Reads and clears the device-side error word that a kernel sets when a
 * bounded wait gives up. Returns WQ_OK or WQ_ERR_TIMEOUT. Synchronizes
 * `stream`. */
int wq_device_error(cudaStream_t stream);

/* Failure detection under test. Enqueues one small kernel whose thread
 * waits, through the same bounded wait every kernel uses (an mbarrier
 * try_wait loop against %globaltimer), on an mbarrier that nothing
 * completes, with the limit shortened to limit_us microseconds (1 ..
 * 2000000; the kernels use 2 s). The wait gives up, the kernel records
 * WQ_ERR_TIMEOUT in the device error word and returns: no trap, no fault,
 * the context stays usable. A following wq_device_error returns
 * WQ_ERR_TIMEOUT (and clears it). Returns WQ_ERR_SHAPE for a limit out of
 * range, WQ_ERR_CUDA if the launch fails. */
int wq_wait_selftest(int limit_us, cudaStream_t stream);

/* Debug views of the integer GEMV's (WQ_VARIANT_GEMV_I8) work split, for a
 * grid of G CTAs (1..448) of `warps` warps (16: split 1, 8: split 2), bits 4
 * or 8, 1 <= K <= 65536, N a positive multiple of 16. The pages have no
 * counterpart; the tests check the split with them. Host only, no GPU.
 * Row blocks are 16 output channels; a chunk is the D consecutive 128-k
 * blocks of one row block that a warp takes together (D = 4 for INT8, 6
 * for INT4; a row block's last chunk may be shorter).
 *   wq_gemv_i8_plan: meta[4] = {chunks per row block CPR, row blocks each
 *   CTA owns LB (CTA c owns c LB .. c LB + LB - 1), first shared row block
 *   RB0 = G LB, chunks of the shared row blocks RL}; runs[G][warps][4] =
 *   {first row block, its first chunk, number of chunks, 1 if the warp takes
 *   shared chunks}: a warp's chunks are consecutive, row-block-major.
 *   wq_gemv_i8_contributors: for shared row block rb (RB0 <= rb < N/16),
 *   the warps (global index c * warps + w) whose chunks meet it, in the
 *   order their partials are summed, and each one's partial slot (0 if rb
 *   is the warp's first row block, else 1); warp_ids and slots hold at
 *   least CPR entries, *count receives the number.
 * Both return WQ_ERR_SHAPE for arguments out of range (or a split beyond
 * 32-bit index arithmetic), WQ_ERR_NULL for a null pointer. */
int wq_gemv_i8_plan(int bits, int K, int N, int G, int warps, int *meta, int *runs);
int wq_gemv_i8_contributors(int bits, int K, int N, int G, int warps, int rb, int *warp_ids, int *slots,
                            int *count);

/* Debug view of the stream-K cuts shared by the persistent kernels (the
 * stream-K GEMV and GEMM, GEMM_W4, the integer tensor-core GEMMs), computed
 * by the kernels' own partition code on the host (no GPU). The pages have
 * no counterpart beyond naming stream-K ("Marlin register and launch
 * scheduling benchmark"); the tests check the partition with it.
 * The weights are U units (128-row panel x 128-k block, panel-major, KB
 * k-blocks per panel); CTA c of G takes units [start[c], start[c + 1]).
 *   start[G + 1]    each CTA's first unit (start[G] = U)
 *   first[G + 1]    each CTA's first panel, start[c] / KB
 *   owner_table[U]  the CTA whose range holds unit u, by the binary search
 *                   over the per-CTA table (the fix-ups' lookup)
 *   owner_div[U]    the same by the division form
 * Host buffers owned by the caller. Returns WQ_ERR_NULL for a null pointer,
 * WQ_ERR_SHAPE unless 1 <= G <= U <= 2^31 - 1 and KB >= 1 (every launcher
 * caps its grid at the unit count). */
int wq_stream_k_plan(long long U, int G, int KB, int *start, int *first, int *owner_table, int *owner_div);

#ifdef __cplusplus
}
#endif

#endif /* WQ_H */
