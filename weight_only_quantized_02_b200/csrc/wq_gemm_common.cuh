// wq_gemm_common.cuh -- helpers shared by the tcgen05 GEMM kernels:
// dequantization of a packed 16-row tile straight into the register layout
// of a tcgen05.st 16x256b store (natural k order, exact integers as bf16).
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

// One INT8 tile (16 rows x 32 k) -> 8 registers of a 16x256b.x2 store: exact q.
__device__ __forceinline__ void int8_tile_regs(const uint4 &w, uint32_t (&r)[8])
{
    const uint32_t ux = w.x ^ 0x80808080u, uy = w.y ^ 0x80808080u;
    const uint32_t uz = w.z ^ 0x80808080u, uw = w.w ^ 0x80808080u;
    r[0] = s8pair_bf16(ux, 0);
    r[1] = s8pair_bf16(ux, 1);
    r[2] = s8pair_bf16(uy, 0);
    r[3] = s8pair_bf16(uy, 1);
    r[4] = s8pair_bf16(uz, 0);
    r[5] = s8pair_bf16(uz, 1);
    r[6] = s8pair_bf16(uw, 0);
    r[7] = s8pair_bf16(uw, 1);
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
