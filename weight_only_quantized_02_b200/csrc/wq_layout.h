// wq_layout.h -- the packed weight layout shared by the packers, the GEMV
// and the GEMM.  Host and device.
//
// Weights of shape [N][K] are cut into 128-row panels p and 128-k blocks kb.
// A (panel, k-block) block is contiguous (16 KB INT8, 8 KB INT4), blocks in
// panel-major order, so a panel's whole K range is one contiguous run.
//
// INT8 block: the tcgen05 K-major canonical layout with 128-byte swizzle.
// Row r (0..127) of the block sits at (r/8)*1024 + (r%8)*128; its 16-byte
// chunk c (k = 16c .. 16c+15, natural order) sits at chunk slot c ^ (r%8) of
// that 128-byte row.  A 1-D bulk copy of the block into 1024-byte aligned
// shared memory is therefore directly the A operand of a tcgen05.mma
// kind::i8 (8-row groups 1024 B apart, K advanced 32 B per instruction).
// The same bytes serve the register paths: one thread per row reads its
// 16-byte chunks without bank conflicts (eight consecutive rows hit the
// eight chunk slots), and an mma.sync lane (g, t) reads chunk c of rows g
// and g+8, whose four 32-bit words feed four m16n8k16 steps (k-slots 2t,
// 2t+1, 2t+8, 2t+9 taken from a run of four consecutive k).
//
// INT4 block: 8 row-blocks j of 16 rows, each holding 2 tiles of 512 bytes
// (64 k each).  Inside a tile, lane l = 4g + t (g = l/4, t = l%4) owns the
// 16 bytes at offset 16 l:
//
//   INT4 tile (k base kt):  .x = row g,   runs a = kt+4t, b = kt+16+4t
//                           .y = row g+8, runs a, b
//                           .z = row g,   runs c = kt+32+4t, d = kt+48+4t
//                           .w = row g+8, runs c, d
//   an INT4 word holding runs (a, b) stores nibble positions
//   [a0, a2, b0, b2, a1, a3, b1, b3], so (word >> 4i) & 0x000F000F yields the
//   natural pairs (a0,a1), (a2,a3), (b0,b1), (b2,b3) for i = 0..3.
//
// This is the m16n8k16 mma.sync A fragment of a 16-row block (rows g, g+8,
// k-slots 2t, 2t+1, 2t+8, 2t+9 taken from a run of four consecutive k), and
// also the register layout of a tcgen05.st 16x256b store of the same rows
// into tensor memory in natural k order; a warp's 128-bit load of a tile is
// one contiguous 512-byte segment.
//
// Rows past N and k past K are zero in both formats.
// Scales: INT8 bf16 [P*128] (s[n], zero past N).  INT4 bf16 [P][K/L][128]
// for the layout group L = 32, 64 or 128 (k = L g .. L g + L - 1 share one
// scale and zero point).  Zeros (INT4): [P][K/L][128 nibbles = 64 bytes],
// row i at nibble i (low nibble first).  Per-channel INT4 (one scale and
// zero point per row, group = K) is stored as L = 128 with the row's pair
// repeated in every 128-k block, so it runs on every group-128 kernel.
// A 64-byte trailer follows the packed weights.
#pragma once

#include <cstddef>
#include <cstdint>

#ifdef __CUDACC__
#define WQ_HD __host__ __device__ __forceinline__
#else
#define WQ_HD inline
#endif

namespace wq {

constexpr int kPanelRows = 128;
constexpr int kBlockK = 128;
constexpr int kTileBytes = 512;
constexpr int kTrailerBytes = 64;
constexpr uint32_t kMagic = 0x32425157u; // "WQB2"
constexpr uint32_t kLayoutVersion = 3;

struct Shape {
    int bits;  // 4 or 8
    int K, N;
    int group; // INT4: the layout group L (32, 64 or 128); INT8: 0
    WQ_HD int panels() const { return (N + kPanelRows - 1) / kPanelRows; }
    WQ_HD int kblocks() const { return (K + kBlockK - 1) / kBlockK; }
    WQ_HD int tile_k() const { return bits == 4 ? 64 : 32; }
    WQ_HD int tiles_per_block() const { return kBlockK / tile_k(); }
    WQ_HD int rb_bytes() const { return tiles_per_block() * kTileBytes; }        // one 16-row block, 128 k
    WQ_HD int block_bytes() const { return 8 * rb_bytes(); }                       // one panel, 128 k
    WQ_HD size_t weight_bytes() const { return (size_t)panels() * kblocks() * block_bytes(); }
    WQ_HD size_t wq_bytes() const { return weight_bytes() + kTrailerBytes; }
    WQ_HD int groups() const { return bits == 8 ? 0 : K / group; } // INT4 scale groups per row
    WQ_HD size_t scale_bytes() const
    {
        return bits == 8 ? (size_t)panels() * kPanelRows * 2
                         : (size_t)panels() * groups() * kPanelRows * 2;
    }
    WQ_HD size_t zero_bytes() const { return bits == 8 ? 0 : (size_t)panels() * groups() * 64; }
    // INT4: byte offset of tile (row-block rb = 16-row index, k tile index kt)
    WQ_HD size_t tile_offset(int rb, int kt) const
    {
        const int p = rb >> 3, j = rb & 7;
        const int tpb = tiles_per_block();
        const int kb = kt / tpb, t = kt % tpb;
        return ((size_t)(p * kblocks() + kb) * 8 + j) * rb_bytes() + (size_t)t * kTileBytes;
    }
    WQ_HD size_t block_offset(int p, int kb) const { return (size_t)(p * kblocks() + kb) * block_bytes(); }
};

// The layout group of an INT4 weight quantized with `group` consecutive k per
// scale: per-channel (group == K > 128) is stored as 128.
WQ_HD int layout_group(int K, int group) { return (group == K && K > 128) ? 128 : group; }

// INT8: byte offset of element (r, kk) inside its block (r = row in the
// panel 0..127, kk = k in the block 0..127).
WQ_HD int int8_in_block(int r, int kk)
{
    return (r >> 3) * 1024 + (r & 7) * 128 + ((((kk >> 4) ^ (r & 7)) & 7) << 4) + (kk & 15);
}

// INT8: byte offset of the 16-byte chunk c of row r inside its block.
WQ_HD int int8_chunk_in_block(int r, int c) { return (r >> 3) * 1024 + (r & 7) * 128 + (((c ^ (r & 7)) & 7) << 4); }

// wmax_bits: binary32 bits of an upper bound of max |w| over the whole
// weight, the bound the integer path's exactness guard uses: for INT4 the
// largest max(z, 15 - z) s over the groups (the largest |q - z| a group's
// zero point allows, times its scale), for INT8 the largest 128 s.
struct Trailer {
    uint32_t magic, version, bits, K, N, group, layout_bytes_lo, layout_bytes_hi;
    uint32_t wmax_bits;
    uint32_t reserved[7];
};
static_assert(sizeof(Trailer) == kTrailerBytes, "trailer is 64 bytes");

// Device address of the trailer's wmax_bits word of packed weights wq.
inline const uint32_t *trailer_wmax(const void *wq, const Shape &sh)
{
    return reinterpret_cast<const uint32_t *>(static_cast<const uint8_t *>(wq) + sh.weight_bytes() +
                                              8 * sizeof(uint32_t));
}

// Position of element k (0..7 relative to the word's 8-k group) inside an
// INT4 word: runs a = k 0..3, b = k 4..7 -> nibble positions.
WQ_HD int int4_nibble_pos(int e) // e in 0..7: a0..a3 = 0..3, b0..b3 = 4..7
{
    // positions [a0, a2, b0, b2, a1, a3, b1, b3]
    constexpr int pos[8] = {0, 4, 1, 5, 2, 6, 3, 7};
    return pos[e];
}

} // namespace wq
