// tile_transpose.cuh -- a 128x128 tile of FP8 codes staged in shared memory
// and written out transposed, for the kernels that emit a second, transposed
// copy of their codes (the operand a weight-gradient GEMM reads along the
// other dimension).
#pragma once

#include <cstdint>

#include "fp8q_device.cuh"
#include "lane_vec.cuh"

namespace fp8q {

constexpr int kTT = 128;  // tile side; also the smem row pitch in bytes

// Byte offset of code (r, c) in the shared tile.  The 16-byte column group is
// XORed with tile-row bits 4..6, so the read-out's 32 lanes -- 8 row bands of
// 16 rows x 4 column words -- hit 32 distinct banks.  16-byte runs stay
// contiguous, so the cast can store whole lane vectors.
__device__ __forceinline__ int tile_off(int r, int c) { return r * kTT + (c ^ (((r >> 4) & 7) << 4)); }

// Lane geometry of a full 128x128 tile: one lane vector (16 or 32 bytes of
// x) per slice, 16 tile rows per warp.
template <typename T, int BYTES>
struct TileGeom {
    static constexpr int kVecPerRow = kTT / LaneVec<T, BYTES>::kElems;  // lane slices per tile row
    static constexpr int kRowsPerLoad = 32 / kVecPerRow;               // tile rows per warp-wide load
    static constexpr int kLoads = 16 / kRowsPerLoad;                   // lane vectors per thread
};

// Cast a full tile held in registers (v[i] = tile row lr0 + i*kRowsPerLoad,
// slice vec_in_row): codes to q (if any) and into the shared code tile.
template <typename T, int FMT, int BYTES, bool WITH_AMAX>
__device__ __forceinline__ void tile_cast(const typename LaneVec<T, BYTES>::In (&v)[TileGeom<T, BYTES>::kLoads],
                                          uint64_t s2, uint8_t* q,
                                          int64_t cols, int64_t r0, int64_t c0, uint8_t* tile, int lr0,
                                          int vec_in_row, float& a) {
    using V = LaneVec<T, BYTES>;
    using G = TileGeom<T, BYTES>;
#pragma unroll
    for (int i = 0; i < G::kLoads; ++i) {
        if (WITH_AMAX) a = fmaxf(a, V::amax(v[i]));
        const typename V::Out c = V::template cast<FMT>(v[i], s2);
        const int lr = lr0 + i * G::kRowsPerLoad;
        if (q != nullptr) st_stream(reinterpret_cast<typename V::Out*>(q + (r0 + lr) * cols + c0) + vec_in_row, c);
        *reinterpret_cast<typename V::Out*>(tile + tile_off(lr, vec_in_row * V::kElems)) = c;
    }
}

// qt from the shared code tile.  Warp w writes qt rows c0+16w..c0+16w+15;
// lane l takes tile rows 16(l&7)..+15 and tile columns 16w+4(l>>3)..+3.  It
// reads 16 words (4 codes of one tile row each), transposes them in 4x4-byte
// blocks with byte permutes, and writes 16 codes into each of its 4 qt rows;
// the 8 lanes that share a qt row cover its 128 bytes, so each store
// instruction writes 4 whole lines.
__device__ __forceinline__ void tile_transpose_out(const uint8_t* tile, uint8_t* qt, int64_t rows, int64_t r0,
                                                   int64_t c0, int lane, int warp) {
    const int rq = (lane & 7) * 16, cq = warp * 16 + (lane >> 3) * 4;
    uint32_t wv[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) wv[i] = *reinterpret_cast<const uint32_t*>(tile + tile_off(rq + i, cq));
    uint32_t o[4][4];  // o[j][g]: column cq+j, rows rq+4g..rq+4g+3
#pragma unroll
    for (int g = 0; g < 4; ++g) {
        const uint32_t w0 = wv[4 * g], w1 = wv[4 * g + 1], w2 = wv[4 * g + 2], w3 = wv[4 * g + 3];
        const uint32_t lo01 = __byte_perm(w0, w1, 0x5140), lo23 = __byte_perm(w2, w3, 0x5140);
        const uint32_t hi01 = __byte_perm(w0, w1, 0x7362), hi23 = __byte_perm(w2, w3, 0x7362);
        o[0][g] = __byte_perm(lo01, lo23, 0x5410);
        o[1][g] = __byte_perm(lo01, lo23, 0x7632);
        o[2][g] = __byte_perm(hi01, hi23, 0x5410);
        o[3][g] = __byte_perm(hi01, hi23, 0x7632);
    }
#pragma unroll
    for (int j = 0; j < 4; ++j)
        st_stream(reinterpret_cast<uint4*>(qt + (c0 + cq + j) * rows + r0 + rq),
                  make_uint4(o[j][0], o[j][1], o[j][2], o[j][3]));
}

}  // namespace fp8q
