// wq_api.cu -- the C ABI (include/wq.h): argument checks, the dispatcher
// table and tuner, the split-K workspace registry and the debug views.
#include <algorithm>
#include <cerrno>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <map>
#include <mutex>
#include <string>
#include <tuple>
#include <vector>

#include "wq.h"
#include "wq_internal.h"
#include "wq_layout.h"

using namespace wq;

namespace {

// ---------------------------------------------------------------------------
// Device facts (cached per device)
// ---------------------------------------------------------------------------
struct DeviceInfo {
    bool ok = false;
    int sm_count = 0, major = 0, minor = 0;
    std::string name;
};

std::mutex g_mu;
std::map<int, DeviceInfo> g_dev;
std::map<int, std::pair<void *, size_t>> g_ws; // registered workspace per device

int current_device_info(DeviceInfo *out)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess)
        return WQ_ERR_CUDA;
    std::lock_guard<std::mutex> lk(g_mu);
    auto it = g_dev.find(dev);
    if (it == g_dev.end()) {
        cudaDeviceProp prop;
        if (cudaGetDeviceProperties(&prop, dev) != cudaSuccess)
            return WQ_ERR_CUDA;
        DeviceInfo d;
        d.ok = true;
        d.sm_count = prop.multiProcessorCount;
        d.major = prop.major;
        d.minor = prop.minor;
        d.name = prop.name;
        it = g_dev.emplace(dev, d).first;
    }
    *out = it->second;
    return WQ_OK;
}

// Status of the table named by the environment variable WQ_TUNING_FILE,
// loaded when the library is loaded (WQ_OK when the variable is unset).
int g_env_tuning = WQ_OK;

std::string device_key(const DeviceInfo &d)
{
    std::string n = d.name;
    std::replace(n.begin(), n.end(), '|', '_');
    return n + "|" + std::to_string(d.sm_count);
}

// ---------------------------------------------------------------------------
// Dispatcher table
// ---------------------------------------------------------------------------
using Key = std::tuple<std::string, int, int, int, int, int>; // device, M, K, N, bits, group
struct Choice {
    int variant, split;
    float us;
};
std::map<Key, Choice> g_table;

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// group 0: INT8 per channel; otherwise INT4 with `group` k per scale (32,
// 64, 128, or K for per channel; check_weight_shape has the rules).
int bits_of_group(int group, int *bits)
{
    if (group < 0)
        return WQ_ERR_GROUP;
    *bits = group == 0 ? 8 : 4;
    return WQ_OK;
}

int check_weight_shape(int bits, int K, int N, int group)
{
    if (bits == 8 && group != 0)
        return WQ_ERR_GROUP;
    if (bits == 4 && group != 32 && group != 64 && group != 128 && !(group == K && K > 0))
        return WQ_ERR_GROUP;
    if (bits != 4 && bits != 8)
        return WQ_ERR_GROUP;
    if (K <= 0 || N <= 0 || N % 16 != 0 || N > kMaxN)
        return WQ_ERR_SHAPE;
    if (bits == 8 && K % 32 != 0)
        return WQ_ERR_SHAPE;
    if (bits == 4 && K % 128 != 0)
        return WQ_ERR_SHAPE;
    if ((long long)K * N > (1LL << 40))
        return WQ_ERR_SHAPE;
    return WQ_OK;
}

int max_gemm_split(int K) { return std::min(32, (K + kBlockK - 1) / kBlockK); }

bool i8_fits(int bits, int M, int K)
{
    return ((bits == 8 && M <= kI8MaxM) || (bits == 4 && M <= kI4MaxM)) && K <= kI8MaxK;
}
size_t ws_bytes_imma(int bits, int M, int K, int N)
{
    return bits == 8 ? ws_bytes_gemm_i8(M, K, N) : ws_bytes_gemm_i4(M, K, N);
}

// The INT4 layout group of the caller's group (0 for INT8).
int lgroup_of(int bits, int K, int group) { return bits == 8 ? 0 : layout_group(K, group); }

// Tokens per kernel launch: groups of 32 or 64 k run on the row-block GEMV only.
int chunk_tokens(int bits, int lgroup) { return (bits == 4 && lgroup != 128) ? 32 : kChunkTokens; }

bool choice_valid(int variant, int split, int M, int K, int bits, int lgroup = 128)
{
    if (bits == 4 && lgroup != 128) // the row-block GEMV is the one kernel with 32- and 64-k groups
        return variant == WQ_VARIANT_GEMV_RB && M <= 32 && (split == 1 || split == 2 || split == 4 || split == 8);
    if (variant == WQ_VARIANT_I8MMA)
        return i8_fits(bits, M, K) && split == 1;
    if (variant == WQ_VARIANT_GEMV_I8)
        return gi_fits(bits, M, K) && (split == 1 || split == 2);
    if (variant == WQ_VARIANT_GEMV)
        return M <= 32 && split >= 1 && split <= 4;
    if (variant == WQ_VARIANT_GEMV_RB)
        return M <= 32 && (split == 1 || split == 2 || split == 4 || split == 8);
    if (variant == WQ_VARIANT_GEMM)
        return M <= 128 && split >= 1 && split <= max_gemm_split(K);
    if (variant == WQ_VARIANT_GEMM_SK)
        return M <= 128 && (split == 1 || split == 2);
    if (variant == WQ_VARIANT_GEMM_W4)
        return bits == 4 && M <= 128 && split == 1;
    return false;
}

// Row-block GEMV K-slices: keep about 32 warps per SM busy.
int default_rb_slices(int K, int N, int sm_count)
{
    const long long rbs = N / 16;
    int ks = 1;
    while (ks < 8 && rbs * ks < (long long)sm_count * 32)
        ks *= 2;
    while (ks > 1 && K / 128 < ks)
        ks /= 2;
    return ks;
}

// Untuned rule: the pages' threshold, fewer than 8 tokens -> a GEMV, else a
// GEMM (Mit han lab Llm awq Kernel Selection Thresholds, The Insight), and
// within each the kernel that measured fastest on B200 across the five
// workloads, workspace permitting: the integer GEMV; the integer
// tensor-core GEMM for W8A16 (M <= 64); the role-split GEMM for W4A16.
// Without a workspace: the row-block GEMV, else the pages' split_k = 8 GEMM
// (run unsplit when no workspace holds its partials).
Choice default_choice(int M, int K, int N, int bits, int sm_count, bool have_ws = true, bool have_i8_ws = true,
                      bool have_gi_ws = true, bool have_w4_ws = true, int lgroup = 128)
{
    if (bits == 4 && lgroup != 128)
        return {WQ_VARIANT_GEMV_RB, default_rb_slices(K, N, sm_count), 0.f};
    if (M < 8) {
        if (gi_fits(bits, M, K) && have_gi_ws)
            return {WQ_VARIANT_GEMV_I8, 1, 0.f};
        if (have_ws)
            return {WQ_VARIANT_GEMV, 3, 0.f};
        return {WQ_VARIANT_GEMV_RB, default_rb_slices(K, N, sm_count), 0.f};
    }
    if (bits == 8 && i8_fits(bits, M, K) && have_i8_ws)
        return {WQ_VARIANT_I8MMA, 1, 0.f};
    if (bits == 4 && have_w4_ws)
        return {WQ_VARIANT_GEMM_W4, 1, 0.f};
    return {WQ_VARIANT_GEMM, std::min(8, max_gemm_split(K)), 0.f};
}

int lookup_choice(const DeviceInfo &d, int M, int K, int N, int bits, int group, Choice *c)
{
    const int lg = lgroup_of(bits, K, group);
    {
        std::lock_guard<std::mutex> lk(g_mu);
        auto it = g_table.find(Key{device_key(d), M, K, N, bits, group});
        if (it != g_table.end()) {
            *c = it->second;
            return WQ_OK;
        }
    }
    *c = default_choice(M, K, N, bits, d.sm_count, true, true, true, true, lg);
    return WQ_OK;
}

int cuda_status(cudaError_t e) { return e == cudaSuccess ? WQ_OK : WQ_ERR_CUDA; }

// One call of at most kChunkTokens tokens: the dispatcher's (or the forced)
// kernel for this M.
int linear_chunk(const uint16_t *x, int M, int K, const void *Wq, const void *scales, const void *zeros, int group,
                 int N, uint16_t *y, int variant, int split, void *ws, size_t ws_bytes_given, cudaStream_t stream)
{
    int bits = 0;
    int st = bits_of_group(group, &bits);
    if (st != WQ_OK)
        return st;
    if (!x || !Wq || !scales || !y || (bits == 4 && !zeros))
        return WQ_ERR_NULL;
    if ((st = check_weight_shape(bits, K, N, group)) != WQ_OK)
        return st;
    const int lg = lgroup_of(bits, K, group);
    if (M < 1 || M > chunk_tokens(bits, lg))
        return WQ_ERR_SHAPE;
    if (!aligned16(x) || !aligned16(y) || !aligned16(Wq) || !aligned16(scales) || (zeros && !aligned16(zeros)))
        return WQ_ERR_ALIGN;
    DeviceInfo d;
    if ((st = current_device_info(&d)) != WQ_OK)
        return st;
    if (d.major != 10)
        return WQ_ERR_ARCH;

    // the workspace this call would use (explicit, else the registered one)
    void *w = ws;
    size_t have = ws_bytes_given;
    if (!w) {
        int dev = 0;
        cudaGetDevice(&dev);
        std::lock_guard<std::mutex> lk(g_mu);
        auto it = g_ws.find(dev);
        if (it != g_ws.end()) {
            w = it->second.first;
            have = it->second.second;
        }
    }
    if (w && !aligned16(w))
        return WQ_ERR_ALIGN;
    const bool sk_ws_ok = w && have >= ws_bytes_gemv_sk(M, N);
    const bool i8_ws_ok = w && i8_fits(bits, M, K) && have >= ws_bytes_imma(bits, M, K, N);
    const bool gi_ws_ok = w && gi_fits(bits, M, K) && have >= ws_bytes_gemv_i8(M, K, N);

    if (variant == WQ_VARIANT_AUTO && g_env_tuning != WQ_OK)
        return g_env_tuning; // the table named by WQ_TUNING_FILE did not load
    Choice c;
    lookup_choice(d, M, K, N, bits, group, &c);
    if (variant != WQ_VARIANT_AUTO) {
        c.variant = variant;
        if (split <= 0)
            c.split = variant == WQ_VARIANT_GEMV      ? 3
                      : variant == WQ_VARIANT_GEMV_RB ? default_rb_slices(K, N, d.sm_count)
                      : variant == WQ_VARIANT_GEMM_SK ? 2
                      : variant == WQ_VARIANT_I8MMA   ? 1
                      : variant == WQ_VARIANT_GEMV_I8 ? 1
                      : variant == WQ_VARIANT_GEMM_W4 ? 1
                                                      : std::min(8, max_gemm_split(K));
    }
    if (split > 0)
        c.split = split;
    if (variant == WQ_VARIANT_AUTO) {
        const bool w4_ws_ok = w && have >= ws_bytes_gemm_sk(M, N);
        if (!choice_valid(c.variant, c.split, M, K, bits, lg) || (c.variant == WQ_VARIANT_I8MMA && !i8_ws_ok) ||
            (c.variant == WQ_VARIANT_GEMV_I8 && !gi_ws_ok) || (c.variant == WQ_VARIANT_GEMM_W4 && !w4_ws_ok))
            c = default_choice(M, K, N, bits, d.sm_count, sk_ws_ok, i8_ws_ok, gi_ws_ok, w4_ws_ok, lg);
        if (c.variant == WQ_VARIANT_GEMV && !sk_ws_ok)
            c = {WQ_VARIANT_GEMV_RB, default_rb_slices(K, N, d.sm_count), 0.f};
        // an automatic choice never fails for lack of workspace: split-K GEMM
        // without a large enough workspace runs unsplit
        if (c.variant == WQ_VARIANT_GEMM && c.split > 1 && (!w || have < ws_bytes(M, N, c.split)))
            c.split = 1;
        if (c.variant == WQ_VARIANT_GEMM_SK && (!w || have < ws_bytes_gemm_sk(M, N)))
            c = {WQ_VARIANT_GEMM, 1, 0.f};
    }
    if (!choice_valid(c.variant, c.split, M, K, bits, lg))
        return WQ_ERR_VARIANT;

    LinearArgs a{x, M, K, N, Wq, scales, zeros, bits, bits == 8 ? 0 : lg, y};
    if (c.variant == WQ_VARIANT_GEMV_I8) {
        if (!gi_ws_ok)
            return WQ_ERR_WORKSPACE;
        return cuda_status(launch_gemv_i8(a, c.split, w, d.sm_count, stream));
    }
    if (c.variant == WQ_VARIANT_I8MMA) {
        if (!i8_ws_ok)
            return WQ_ERR_WORKSPACE;
        return cuda_status(bits == 8 ? launch_gemm_i8(a, w, d.sm_count, stream)
                                     : launch_gemm_i4(a, w, d.sm_count, stream));
    }
    if (c.variant == WQ_VARIANT_GEMV_RB)
        return cuda_status(launch_gemv(a, c.split, d.sm_count, stream));
    if (c.variant == WQ_VARIANT_GEMV) {
        if (!sk_ws_ok)
            return WQ_ERR_WORKSPACE;
        return cuda_status(launch_gemv_sk(a, c.split, w, d.sm_count, stream));
    }
    if (c.variant == WQ_VARIANT_GEMM_SK) {
        if (!w || have < ws_bytes_gemm_sk(M, N))
            return WQ_ERR_WORKSPACE;
        return cuda_status(launch_gemm_sk(a, c.split, w, d.sm_count, stream));
    }
    if (c.variant == WQ_VARIANT_GEMM_W4) {
        if (!w || have < ws_bytes_gemm_sk(M, N))
            return WQ_ERR_WORKSPACE;
        return cuda_status(launch_gemm_w4(a, w, d.sm_count, stream));
    }
    if (c.split > 1 && (!w || have < ws_bytes(M, N, c.split)))
        return WQ_ERR_WORKSPACE;
    return cuda_status(launch_gemm(a, c.split, c.split > 1 ? w : nullptr, d.sm_count, stream));
}

// The layer for any M up to kMaxTokens: runs of kChunkTokens tokens, one
// kernel each, in order on the stream (x and y advance by whole token rows,
// so every chunk keeps their 16-byte alignment).  Each chunk streams the
// weights once; the chunks share the workspace one after another.  A
// failing chunk returns its status; the chunks before it are already
// enqueued.
int linear_impl(const uint16_t *x, int M, int K, const void *Wq, const void *scales, const void *zeros, int group,
                int N, uint16_t *y, int variant, int split, void *ws, size_t ws_bytes_given, cudaStream_t stream)
{
    int bits = 0;
    if (bits_of_group(group, &bits) != WQ_OK)
        return WQ_ERR_GROUP;
    const int chunk = chunk_tokens(bits, lgroup_of(bits, K, group));
    if (M <= chunk)
        return linear_chunk(x, M, K, Wq, scales, zeros, group, N, y, variant, split, ws, ws_bytes_given, stream);
    if (M > kMaxTokens)
        return WQ_ERR_SHAPE;
    if (!x || !y)
        return WQ_ERR_NULL;
    for (int m0 = 0; m0 < M; m0 += chunk) {
        const int mc = std::min(chunk, M - m0);
        const int st = linear_chunk(x + (size_t)m0 * K, mc, K, Wq, scales, zeros, group, N, y + (size_t)m0 * N,
                                    variant, split, ws, ws_bytes_given, stream);
        if (st != WQ_OK)
            return st;
    }
    return WQ_OK;
}

} // namespace

namespace wq {

namespace {
struct SetupKey {
    int dev;
    const void *func;
    bool operator<(const SetupKey &o) const { return dev != o.dev ? dev < o.dev : func < o.func; }
};
struct SetupState {
    size_t optin = 0;
    std::map<std::pair<int, size_t>, int> occ; // (threads, smem) -> CTAs per SM
};
std::mutex g_setup_mu;
std::map<SetupKey, SetupState> g_setup;
} // namespace

cudaError_t kernel_setup(const void *func, size_t smem_optin, int threads, size_t smem, int *occ)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess)
        return e;
    std::lock_guard<std::mutex> lk(g_setup_mu);
    SetupState &s = g_setup[SetupKey{dev, func}];
    if (smem_optin > s.optin) {
        e = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_optin);
        if (e != cudaSuccess)
            return e;
        s.optin = smem_optin;
    }
    if (occ) {
        const auto k = std::make_pair(threads, smem);
        auto it = s.occ.find(k);
        if (it == s.occ.end()) {
            int o = 0;
            e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&o, func, threads, smem);
            if (e != cudaSuccess)
                return e;
            it = s.occ.emplace(k, o > 0 ? o : 1).first;
        }
        *occ = it->second;
    }
    return cudaSuccess;
}

} // namespace wq

// ===========================================================================
// C ABI
// ===========================================================================
extern "C" {

const char *wq_strerror(int status)
{
    switch (status) {
    case WQ_OK: return "ok";
    case WQ_ERR_NULL: return "a required pointer is NULL";
    case WQ_ERR_SHAPE: return "M, K or N outside the supported shape rules";
    case WQ_ERR_ALIGN: return "a pointer is not 16-byte aligned";
    case WQ_ERR_GROUP: return "unsupported bits/group combination (INT8: group 0, INT4: group 128)";
    case WQ_ERR_HEADER: return "packed-weight trailer does not match the arguments";
    case WQ_ERR_WORKSPACE: return "split-K workspace missing or too small";
    case WQ_ERR_CUDA: return "CUDA runtime error";
    case WQ_ERR_TUNING: return "tuning file unreadable or malformed";
    case WQ_ERR_TIMEOUT: return "a bounded device-side wait gave up";
    case WQ_ERR_ARCH: return "device is not sm_100 (B200 class)";
    case WQ_ERR_VARIANT: return "forced variant/split not valid for this shape";
    default: return "unknown status";
    }
}

int wq_version(void) { return 200; }

int wq_packed_bytes(int bits, int K, int N, int group, size_t *wq_bytes, size_t *scale_bytes, size_t *zero_bytes)
{
    const int st = check_weight_shape(bits, K, N, group);
    if (st != WQ_OK)
        return st;
    const Shape sh{bits, K, N, lgroup_of(bits, K, group)};
    if (wq_bytes)
        *wq_bytes = sh.wq_bytes();
    if (scale_bytes)
        *scale_bytes = sh.scale_bytes();
    if (zero_bytes)
        *zero_bytes = sh.zero_bytes();
    return WQ_OK;
}

int wq_quantize_int8(const float *W, int K, int N, int8_t *q_out, uint16_t *s_out, cudaStream_t stream)
{
    if (!W || !q_out || !s_out)
        return WQ_ERR_NULL;
    if (K <= 0 || N <= 0)
        return WQ_ERR_SHAPE;
    return cuda_status(launch_quantize_int8(W, K, N, q_out, s_out, stream));
}

int wq_quantize_int4(const float *W, int K, int N, int group, uint32_t *q_out, uint16_t *s_out, uint32_t *z_out,
                     cudaStream_t stream)
{
    if (!W || !q_out || !s_out || !z_out)
        return WQ_ERR_NULL;
    if (K <= 0 || N <= 0 || K % 128 != 0)
        return WQ_ERR_SHAPE;
    if (group != 32 && group != 64 && group != 128 && group != K)
        return WQ_ERR_GROUP;
    return cuda_status(launch_quantize_int4(W, K, N, group, q_out, s_out, z_out, stream));
}

int wq_pack_int8(const int8_t *q, const uint16_t *scales, int K, int N, void *wq_out, void *scales_out,
                 cudaStream_t stream)
{
    if (!q || !scales || !wq_out || !scales_out)
        return WQ_ERR_NULL;
    const int st = check_weight_shape(8, K, N, 0);
    if (st != WQ_OK)
        return st;
    if (!aligned16(q) || !aligned16(wq_out) || !aligned16(scales_out))
        return WQ_ERR_ALIGN;
    return cuda_status(launch_pack_int8(q, scales, K, N, wq_out, scales_out, stream));
}

int wq_pack_int4(const uint32_t *q, const uint16_t *scales, const uint32_t *zeros, int K, int N, int group,
                 void *wq_out, void *scales_out, void *zeros_out, cudaStream_t stream)
{
    if (!q || !scales || !zeros || !wq_out || !scales_out || !zeros_out)
        return WQ_ERR_NULL;
    const int st = check_weight_shape(4, K, N, group);
    if (st != WQ_OK)
        return st;
    if (!aligned16(wq_out) || !aligned16(scales_out) || !aligned16(zeros_out))
        return WQ_ERR_ALIGN;
    return cuda_status(launch_pack_int4(q, scales, zeros, K, N, group, wq_out, scales_out, zeros_out, stream));
}

int wq_check_packed(const void *Wq, int bits, int K, int N, int group, cudaStream_t stream)
{
    if (!Wq)
        return WQ_ERR_NULL;
    int st = check_weight_shape(bits, K, N, group);
    if (st != WQ_OK)
        return st;
    const Shape sh{bits, K, N, lgroup_of(bits, K, group)};
    Trailer t;
    if (cudaMemcpyAsync(&t, (const uint8_t *)Wq + sh.weight_bytes(), sizeof t, cudaMemcpyDeviceToHost, stream) !=
            cudaSuccess ||
        cudaStreamSynchronize(stream) != cudaSuccess)
        return WQ_ERR_CUDA;
    const size_t wb = sh.weight_bytes();
    if (t.magic != kMagic || t.version != kLayoutVersion || t.bits != (uint32_t)bits || t.K != (uint32_t)K ||
        t.N != (uint32_t)N || t.group != (uint32_t)group || t.layout_bytes_lo != (uint32_t)(wb & 0xffffffffu) ||
        t.layout_bytes_hi != (uint32_t)(wb >> 32))
        return WQ_ERR_HEADER;
    return WQ_OK;
}

int wq_linear(const uint16_t *x, int M, int K, const void *Wq, const void *scales, const void *zeros, int group,
              int N, uint16_t *y, cudaStream_t stream)
{
    return linear_impl(x, M, K, Wq, scales, zeros, group, N, y, WQ_VARIANT_AUTO, 0, nullptr, 0, stream);
}

int wq_linear_forced(const uint16_t *x, int M, int K, const void *Wq, const void *scales, const void *zeros,
                     int group, int N, uint16_t *y, int variant, int split, cudaStream_t stream)
{
    return linear_impl(x, M, K, Wq, scales, zeros, group, N, y, variant, split, nullptr, 0, stream);
}

int wq_linear_ex(const uint16_t *x, int M, int K, const void *Wq, const void *scales, const void *zeros, int group,
                 int N, uint16_t *y, int variant, int split, void *ws, size_t ws_bytes_given, cudaStream_t stream)
{
    return linear_impl(x, M, K, Wq, scales, zeros, group, N, y, variant, split, ws, ws_bytes_given, stream);
}

int wq_linear_noalloc(const uint16_t *x, int M, int K, const void *Wq, const void *scales, const void *zeros,
                      int group, int N, uint16_t *y, cudaStream_t stream)
{
    int bits = 0;
    int st = bits_of_group(group, &bits);
    if (st != WQ_OK)
        return st;
    if (!x || !Wq || !scales || !y || (bits == 4 && !zeros))
        return WQ_ERR_NULL;
    if ((st = check_weight_shape(bits, K, N, group)) != WQ_OK)
        return st;
    if (bits == 4 && lgroup_of(bits, K, group) != 128)
        return WQ_ERR_GROUP; // the stream-K GEMV reads the group-128 layout
    if (M < 1 || M > noalloc_max_m() || N > noalloc_max_n())
        return WQ_ERR_SHAPE;
    if (!aligned16(x) || !aligned16(y) || !aligned16(Wq) || !aligned16(scales) || (zeros && !aligned16(zeros)))
        return WQ_ERR_ALIGN;
    DeviceInfo d;
    if ((st = current_device_info(&d)) != WQ_OK)
        return st;
    if (d.major != 10)
        return WQ_ERR_ARCH;
    LinearArgs a{x, M, K, N, Wq, scales, zeros, bits, bits == 8 ? 0 : 128, y};
    return cuda_status(launch_gemv_sk_noalloc(a, d.sm_count, stream));
}

int wq_linear_f16(const uint16_t *x, int M, int K, const void *Wq, const void *scales, const void *zeros, int group,
                  int N, uint16_t *y, cudaStream_t stream)
{
    int bits = 0;
    int st = bits_of_group(group, &bits);
    if (st != WQ_OK)
        return st;
    if (!x || !Wq || !scales || !y || (bits == 4 && !zeros))
        return WQ_ERR_NULL;
    if ((st = check_weight_shape(bits, K, N, group)) != WQ_OK)
        return st;
    if (M < 1 || M > kMaxTokens)
        return WQ_ERR_SHAPE;
    if (!aligned16(x) || !aligned16(y) || !aligned16(Wq) || !aligned16(scales) || (zeros && !aligned16(zeros)))
        return WQ_ERR_ALIGN;
    DeviceInfo d;
    if ((st = current_device_info(&d)) != WQ_OK)
        return st;
    if (d.major != 10)
        return WQ_ERR_ARCH;
    const int lg = lgroup_of(bits, K, group), ks = default_rb_slices(K, N, d.sm_count);
    for (int m0 = 0; m0 < M; m0 += 32) { // the row-block GEMV: 32 tokens per launch
        const int mc = std::min(32, M - m0);
        LinearArgs a{x + (size_t)m0 * K, mc, K, N, Wq, scales, zeros, bits, bits == 8 ? 0 : lg, y + (size_t)m0 * N};
        if ((st = cuda_status(launch_gemv(a, ks, d.sm_count, stream, true))) != WQ_OK)
            return st;
    }
    return WQ_OK;
}

size_t wq_topk_workspace_bytes(int M, int N, int k)
{
    if (M > kChunkTokens)
        return 0;
    return topk_ws_bytes(M, N, k);
}

int wq_linear_topk(const uint16_t *x, int M, int K, const void *Wq, const void *scales, const void *zeros, int group,
                   int N, int k, uint16_t *vals, int32_t *idx, void *ws, size_t ws_bytes_given, cudaStream_t stream)
{
    if (M < 1 || M > kChunkTokens || k < 1 || k > kTopkMaxK || k > N)
        return WQ_ERR_SHAPE;
    if (!vals || !idx || !ws)
        return WQ_ERR_NULL;
    const size_t need = topk_ws_bytes(M, N, k);
    if (need == 0)
        return WQ_ERR_SHAPE;
    if (!aligned16(ws))
        return WQ_ERR_ALIGN;
    if (ws_bytes_given < need)
        return WQ_ERR_WORKSPACE;
    // the logits, into the scratch, by the dispatcher's kernel
    uint16_t *logits = static_cast<uint16_t *>(ws);
    const int st = linear_impl(x, M, K, Wq, scales, zeros, group, N, logits, WQ_VARIANT_AUTO, 0, nullptr, 0, stream);
    if (st != WQ_OK)
        return st;
    void *cand = static_cast<uint8_t *>(ws) + ((size_t)M * N * 2 + 255) / 256 * 256;
    return cuda_status(launch_topk(logits, M, N, k, cand, vals, idx, stream));
}

size_t wq_workspace_bytes(int M, int K, int N, int max_split)
{
    if (M < 1 || K < 1 || N < 1 || max_split < 1)
        return 0;
    M = std::min(M, kChunkTokens); // longer inputs run in chunks that share the workspace
    size_t b = std::max(ws_bytes(M, N, max_split), ws_bytes_gemm_sk(M, N));
    if (M <= 32)
        b = std::max(b, ws_bytes_gemv_sk(M, N));
    if (M <= kI8MaxM && K <= kI8MaxK)
        b = std::max(b, std::max(ws_bytes_gemm_i8(M, K, N), ws_bytes_gemm_i4(M, K, N)));
    if (M <= kGiMaxM && K <= kI8MaxK)
        b = std::max(b, ws_bytes_gemv_i8(M, K, N));
    return b;
}

int wq_set_workspace(void *ws, size_t bytes)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess)
        return WQ_ERR_CUDA;
    if (ws && !aligned16(ws))
        return WQ_ERR_ALIGN;
    if (ws && bytes > 0) {
        if (cudaMemset(ws, 0, bytes) != cudaSuccess || cudaDeviceSynchronize() != cudaSuccess)
            return WQ_ERR_CUDA;
    }
    std::lock_guard<std::mutex> lk(g_mu);
    if (!ws)
        g_ws.erase(dev);
    else
        g_ws[dev] = {ws, bytes};
    return WQ_OK;
}

// ---------------------------------------------------------------------------
// Tuner
// ---------------------------------------------------------------------------
int wq_tune(const uint16_t *x, int M, int K, const void *Wq, const void *scales, const void *zeros, int group,
            int N, uint16_t *y, int warmup, int iters, cudaStream_t stream)
{
    int bits = 0;
    int st = bits_of_group(group, &bits);
    if (st != WQ_OK)
        return st;
    DeviceInfo d;
    if ((st = current_device_info(&d)) != WQ_OK)
        return st;
    if (warmup < 0 || iters < 1 || M < 1 || M > kMaxTokens)
        return WQ_ERR_SHAPE;
    if ((st = check_weight_shape(bits, K, N, group)) != WQ_OK)
        return st;
    const int lg = lgroup_of(bits, K, group);
    M = std::min(M, chunk_tokens(bits, lg)); // longer inputs: the chunk shape, timed on the first chunk
    std::vector<std::pair<int, int>> cands;
    if (bits == 4 && lg != 128) {
        for (int ks : {1, 2, 4, 8})
            cands.push_back({WQ_VARIANT_GEMV_RB, ks});
    } else if (M <= 32) {
        for (int c : {1, 2, 3})
            cands.push_back({WQ_VARIANT_GEMV, c});
        for (int ks : {1, 2, 4, 8})
            cands.push_back({WQ_VARIANT_GEMV_RB, ks});
    }
    for (int s : {1, 2, 4, 8, 16, 32})
        if (s <= max_gemm_split(K))
            cands.push_back({WQ_VARIANT_GEMM, s});
    for (int c : {1, 2})
        cands.push_back({WQ_VARIANT_GEMM_SK, c});
    if (i8_fits(bits, M, K))
        cands.push_back({WQ_VARIANT_I8MMA, 1});
    if (bits == 4)
        cands.push_back({WQ_VARIANT_GEMM_W4, 1});
    if (gi_fits(bits, M, K))
        for (int c : {1, 2})
            cands.push_back({WQ_VARIANT_GEMV_I8, c});

    // Decode runs its layers back to back, each streaming its own weights
    // from HBM while the next one is launched behind it.  The tuner times
    // the same thing: R copies of the packed weights spanning at least three
    // L2 sizes, called back to back in rotation, one event pair around each
    // full rotation (per call = rotation time / R), so no call finds its
    // weights in L2 and launch overlap counts as it does in a decode step.
    // Copy contents do not affect timing; they are the caller's weights.
    int l2 = 0;
    int tdev = 0;
    cudaGetDevice(&tdev);
    cudaDeviceGetAttribute(&l2, cudaDevAttrL2CacheSize, tdev);
    size_t wb = 0, sb = 0, zb = 0;
    if ((st = wq_packed_bytes(bits, K, N, group, &wb, &sb, &zb)) != WQ_OK)
        return st;
    const size_t wb_al = (wb + 255) / 256 * 256, sb_al = (sb + 255) / 256 * 256, zb_al = (zb + 255) / 256 * 256;
    const size_t copy_bytes = wb_al + sb_al + zb_al;
    const int R = (int)std::max<size_t>(2, std::min<size_t>(64, (3 * (size_t)l2 + copy_bytes - 1) / copy_bytes));
    uint8_t *rot = nullptr;
    if (cudaMalloc(&rot, copy_bytes * R) != cudaSuccess)
        return WQ_ERR_CUDA;
    std::vector<const void *> rw(R), rs(R), rz(R);
    for (int c = 0; c < R; ++c) {
        uint8_t *base = rot + copy_bytes * c;
        rw[c] = base;
        rs[c] = base + wb_al;
        rz[c] = zb ? base + wb_al + sb_al : nullptr;
        bool okc = cudaMemcpyAsync(base, Wq, wb, cudaMemcpyDeviceToDevice, stream) == cudaSuccess &&
                   cudaMemcpyAsync(base + wb_al, scales, sb, cudaMemcpyDeviceToDevice, stream) == cudaSuccess &&
                   (!zb || cudaMemcpyAsync(base + wb_al + sb_al, zeros, zb, cudaMemcpyDeviceToDevice, stream) ==
                               cudaSuccess);
        if (!okc) {
            cudaFree(rot);
            return WQ_ERR_CUDA;
        }
    }
    auto rotation = [&](int v, int s) {
        int rc = WQ_OK;
        for (int c = 0; c < R && rc == WQ_OK; ++c)
            rc = linear_impl(x, M, K, rw[c], rs[c], rz[c], group, N, y, v, s, nullptr, 0, stream);
        return rc;
    };
    cudaEvent_t e0, e1;
    cudaEventCreate(&e0);
    cudaEventCreate(&e1);
    Choice best{-1, 0, 0.f};
    int result = WQ_OK;
    for (auto [v, s] : cands) {
        int rc = WQ_OK;
        for (int i = 0; i < std::max(1, warmup) && rc == WQ_OK; ++i)
            rc = rotation(v, s);
        if (rc != WQ_OK)
            continue; // e.g. no workspace large enough for this split
        std::vector<float> t;
        for (int i = 0; i < iters && rc == WQ_OK; ++i) {
            cudaEventRecord(e0, stream);
            rc = rotation(v, s);
            cudaEventRecord(e1, stream);
            if (cudaEventSynchronize(e1) != cudaSuccess) {
                rc = WQ_ERR_CUDA;
                break;
            }
            float ms = 0.f;
            cudaEventElapsedTime(&ms, e0, e1);
            t.push_back(ms * 1000.f / R);
        }
        if (rc != WQ_OK) {
            if (rc == WQ_ERR_CUDA)
                result = rc;
            continue;
        }
        // The event clock ticks in about 1 us steps, as coarse as the
        // differences between candidates: take the mean of the middle half
        // of the sorted times (the median's robustness, finer resolution).
        std::sort(t.begin(), t.end());
        const size_t lo = t.size() / 4, hi = t.size() - t.size() / 4;
        float med = 0.f;
        for (size_t i = lo; i < hi; ++i)
            med += t[i];
        med /= (float)(hi - lo);
        if (const char *lg = getenv("WQ_TUNE_LOG"); lg && *lg && *lg != '0')
            fprintf(stderr, "wq_tune M=%d K=%d N=%d bits=%d group=%d variant=%d split=%d us=%.3f\n", M, K, N,
                    bits, group, v, s, med);
        // ">=": on an exact tie the later (larger) split wins (Mit han lab Llm awq
        // Kernel Selection Thresholds, The Insight: the split_k auto-tune)
        if (best.variant < 0 || best.us >= med)
            best = {v, s, med};
    }
    cudaEventDestroy(e0);
    cudaEventDestroy(e1);
    cudaStreamSynchronize(stream);
    cudaFree(rot);
    if (result != WQ_OK)
        return result;
    if (best.variant < 0)
        return WQ_ERR_VARIANT;
    std::lock_guard<std::mutex> lk(g_mu);
    g_table[Key{device_key(d), M, K, N, bits, group}] = best;
    return WQ_OK;
}

int wq_get_choice(int M, int K, int N, int bits, int group, int *variant, int *split)
{
    if (!variant || !split)
        return WQ_ERR_NULL;
    if (g_env_tuning != WQ_OK)
        return g_env_tuning;
    DeviceInfo d;
    int st = current_device_info(&d);
    if (st != WQ_OK)
        return st;
    Choice c;
    lookup_choice(d, std::min(M, chunk_tokens(bits, lgroup_of(bits, K, group))), K, N, bits, group, &c);
    *variant = c.variant;
    *split = c.split;
    return WQ_OK;
}

int wq_set_choice(int M, int K, int N, int bits, int group, int variant, int split)
{
    DeviceInfo d;
    int st = current_device_info(&d);
    if (st != WQ_OK)
        return st;
    if (check_weight_shape(bits, K, N, group) != WQ_OK || !choice_valid(variant, split, M, K, bits, lgroup_of(bits, K, group)))
        return WQ_ERR_VARIANT;
    std::lock_guard<std::mutex> lk(g_mu);
    g_table[Key{device_key(d), M, K, N, bits, group}] = Choice{variant, split, 0.f};
    return WQ_OK;
}

int wq_clear_tuning(void)
{
    std::lock_guard<std::mutex> lk(g_mu);
    g_table.clear();
    return WQ_OK;
}

int wq_save_tuning(const char *path)
{
    if (!path)
        return WQ_ERR_NULL;
    FILE *f = fopen(path, "w");
    if (!f)
        return WQ_ERR_TUNING;
    std::lock_guard<std::mutex> lk(g_mu);
    fprintf(f, "# wq tuning v1: device|sms M K N bits group variant split us_per_call\n");
    for (auto &kv : g_table) {
        const auto &k = kv.first;
        fprintf(f, "%s %d %d %d %d %d %d %d %.3f\n", std::get<0>(k).c_str(), std::get<1>(k), std::get<2>(k),
                std::get<3>(k), std::get<4>(k), std::get<5>(k), kv.second.variant, kv.second.split, kv.second.us);
    }
    const bool bad = ferror(f) != 0;
    fclose(f);
    return bad ? WQ_ERR_TUNING : WQ_OK;
}

// Host-only parser (no CUDA calls), so it can be tested without a GPU.
int wq_load_tuning(const char *path)
{
    if (!path)
        return WQ_ERR_NULL;
    FILE *f = fopen(path, "r");
    if (!f)
        return WQ_ERR_TUNING;
    std::map<Key, Choice> loaded;
    char line[1024];
    bool bad = false;
    while (fgets(line, sizeof line, f)) {
        const size_t len = strlen(line);
        if (len == 0 || line[0] == '#' || line[0] == '\n')
            continue;
        if (line[len - 1] != '\n' && !feof(f)) {
            bad = true;
            break;
        }
        // device key is everything up to the first '|' plus the SM count token
        char *bar = strchr(line, '|');
        if (!bar) {
            bad = true;
            break;
        }
        char *rest = strchr(bar, ' ');
        if (!rest) {
            bad = true;
            break;
        }
        std::string dkey(line, rest - line);
        int M, K, N, bits, group, variant, split;
        float us;
        char tail;
        const int n = sscanf(rest, " %d %d %d %d %d %d %d %f %c", &M, &K, &N, &bits, &group, &variant, &split, &us,
                             &tail);
        if (n != 8 || check_weight_shape(bits, K, N, group) != WQ_OK || M < 1 || M > 128 ||
            !choice_valid(variant, split, M, K, bits, lgroup_of(bits, K, group))) {
            bad = true;
            break;
        }
        loaded[Key{dkey, M, K, N, bits, group}] = Choice{variant, split, us};
    }
    fclose(f);
    if (bad)
        return WQ_ERR_TUNING;
    std::lock_guard<std::mutex> lk(g_mu);
    for (auto &kv : loaded)
        g_table[kv.first] = kv.second;
    return WQ_OK;
}

// ---------------------------------------------------------------------------
// Debug views
// ---------------------------------------------------------------------------
int wq_unpack_debug(const void *Wq, const void *zeros, int bits, int K, int N, int group, int8_t *q_out,
                    int8_t *z_out, cudaStream_t stream)
{
    if (!Wq || !q_out || (bits == 4 && (!zeros || !z_out)))
        return WQ_ERR_NULL;
    const int st = check_weight_shape(bits, K, N, group);
    if (st != WQ_OK)
        return st;
    return cuda_status(
        launch_unpack_debug(Wq, zeros, Shape{bits, K, N, lgroup_of(bits, K, group)}, group, q_out, z_out, stream));
}

int wq_dequant_debug(const void *Wq, const void *scales, const void *zeros, int bits, int K, int N, int group,
                     float *w_out, cudaStream_t stream)
{
    if (!Wq || !scales || !w_out || (bits == 4 && !zeros))
        return WQ_ERR_NULL;
    const int st = check_weight_shape(bits, K, N, group);
    if (st != WQ_OK)
        return st;
    return cuda_status(
        launch_dequant_debug(Wq, scales, zeros, Shape{bits, K, N, lgroup_of(bits, K, group)}, w_out, stream));
}

int wq_wait_selftest(int limit_us, cudaStream_t stream)
{
    if (limit_us < 1 || limit_us > 2000000)
        return WQ_ERR_SHAPE;
    DeviceInfo d;
    int st = current_device_info(&d);
    if (st != WQ_OK)
        return st;
    return cuda_status(launch_wait_selftest((uint64_t)limit_us * 1000u, stream));
}

int wq_device_error(cudaStream_t stream)
{
    int a = 0, b = 0, c = 0, e = 0, f = 0, h = 0;
    if (read_device_error(&a, stream) != cudaSuccess || read_gemv_sk_error(&b, stream) != cudaSuccess ||
        read_gemm_sk_error(&c, stream) != cudaSuccess || read_gemm_i8_error(&e, stream) != cudaSuccess ||
        read_gemm_i4_error(&f, stream) != cudaSuccess || read_gemm_w4_error(&h, stream) != cudaSuccess)
        return WQ_ERR_CUDA;
    return (a == 0 && b == 0 && c == 0 && e == 0 && f == 0 && h == 0) ? WQ_OK : WQ_ERR_TIMEOUT;
}

} // extern "C"

// WQ_TUNING_FILE: a dispatcher table (the wq_save_tuning format) loaded when
// the library is loaded, so a deployment can ship measured choices without
// code.  A file that cannot be read or parsed makes every automatic choice
// (wq_linear, wq_get_choice) return WQ_ERR_TUNING; forced variants still run.
namespace {
struct EnvTuningLoader {
    EnvTuningLoader()
    {
        const char *path = getenv("WQ_TUNING_FILE");
        if (path && *path)
            g_env_tuning = wq_load_tuning(path);
    }
} g_env_tuning_loader;
} // namespace
