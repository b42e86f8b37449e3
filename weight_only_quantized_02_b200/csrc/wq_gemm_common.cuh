// wq_gemm_common.cuh -- helpers shared by the tcgen05 GEMM kernels:
// dequantization of packed weights straight into the register layout of a
// tensor-memory store (natural k order, exact integers as bf16): a 16-row
// INT4 tile for tcgen05.st 16x256b, one row's INT8 chunks for 32x32b.
#pragma once

#include <cudaTypedefs.h>

#include "wq_device.cuh"

namespace wq {

// One INT4 tile (16 rows x 64 k) -> the 16 registers of a tcgen05.st
// 16x256b.x4 store: the exact integers (q - z) as bf16, natural k order.
__device__ __forceinline__ void int4_tile_regs(const uint4 &w, uint32_t zlo, uint32_t zhi, uint32_t (&r)[16])
{
    auto d = [](uint32_t word, int i, uint32_t zz) { return bf16x2_sub(nib_pair_bf16(word >> (4 * i)), zz); };
    r[0] = d(w.x, 0, zlo);
    r[1] = d(w.x, 1, zlo);
    r[2] = d(w.y, 0, zhi);
    r[3] = d(w.y, 1, zhi);
    r[4] = d(w.x, 2, zlo);
    r[5] = d(w.x, 3, zlo);
    r[6] = d(w.y, 2, zhi);
    r[7] = d(w.y, 3, zhi);
    r[8] = d(w.z, 0, zlo);
    r[9] = d(w.z, 1, zlo);
    r[10] = d(w.w, 0, zhi);
    r[11] = d(w.w, 1, zhi);
    r[12] = d(w.z, 2, zlo);
    r[13] = d(w.z, 3, zlo);
    r[14] = d(w.w, 2, zhi);
    r[15] = d(w.w, 3, zhi);
}

// Two INT8 chunks of one row (k = 16c .. 16c+31, natural order) -> the 16
// registers of one thread's tcgen05.st 32x32b.x16 store: bf16 pairs of the
// exact codes, column j = k pair (2j, 2j+1).
__device__ __forceinline__ void int8_chunks_regs(const uint4 &w0, const uint4 &w1, uint32_t (&r)[16])
{
    const uint32_t v[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const uint32_t u = v[i] ^ 0x80808080u;
        r[2 * i] = s8pair_bf16(u, 0);
        r[2 * i + 1] = s8pair_bf16(u, 1);
    }
}

inline PFN_cuTensorMapEncodeTiled_v12000 get_encode_fn()
{
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    }
    return fn;
}

// 2-D tensor map over x [M][K] bf16: boxes of 64 k x NT token rows,
// 128-byte swizzle (the UMMA K-major canonical layout); rows past M read 0.
template <int NT>
inline bool make_x_map(CUtensorMap *map, const uint16_t *x, int M, int K)
{
    auto fn = get_encode_fn();
    if (!fn)
        return false;
    const cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)M};
    const cuuint64_t strides[1] = {(cuuint64_t)K * 2};
    const cuuint32_t box[2] = {64, (cuuint32_t)NT};
    const cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<uint16_t *>(x), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

} // namespace wq
