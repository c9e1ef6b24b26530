// scale_layout.cu -- block scales between the dense row-major layout and the
// tensor-core (block-scaled MMA) tile layout.
//
// The layout (pwq_internal.h, mma_scale_offset): per batch slab, tiles of 128
// rows x 4 scale columns, 512 contiguous bytes each, ordered along the scale
// columns within a 128-row band and band after band; inside a tile, line
// r % 32 (16 bytes) holds rows r, r + 32, r + 64, r + 96, four scale bytes
// each.  That is the shape in which the sm_100 block-scaled MMA takes its
// scale factors into tensor memory (PTX ISA, tcgen05.cp with the
// 32x128b.warpx4 shape: 32 lines of 16 bytes fanned out to four warps) and
// cuBLAS's 1D block-scaling-factor layout.  The quantisers can write it
// directly (mxfp8_quant_grouped_mma, nvfp4_quant_grouped_mma); these
// kernels convert arrays written in the dense layout, either way.
//
// One thread per 16-byte line: four scale rows of four bytes each.  Bytes
// past the last row or column are zero in the tile layout and are not
// written back to the dense one.
#include "pwq_internal.h"

namespace pwq {
namespace {

constexpr int kThreads = 256;

struct LayoutArgs {
    const uint8_t* src;
    uint8_t* dst;
    uint32_t M, S, col_tiles;
    uint64_t lines;              // B * slab_bytes / 16
    uint64_t lines_per_slab;
    int rows4;                   // S % 4 == 0 and the dense base 4-byte aligned: 4-byte dense accesses
};

// Dense row m, columns 4 * ct .. 4 * ct + 3 of slab b as one little-endian word (0 past the edges).
__device__ __forceinline__ uint32_t dense_word(const LayoutArgs& a, uint64_t b, uint32_t m, uint32_t ct) {
    if (m >= a.M) return 0u;
    const uint8_t* row = a.src + (b * a.M + m) * (uint64_t)a.S;
    const uint32_t c0 = ct * 4u;
    if (a.rows4) return *reinterpret_cast<const uint32_t*>(row + c0);
    uint32_t w = 0u;
#pragma unroll
    for (int k = 0; k < 4; ++k)
        if (c0 + k < a.S) w |= (uint32_t)row[c0 + k] << (8 * k);
    return w;
}

__global__ void __launch_bounds__(kThreads) scales_to_mma_kernel(const LayoutArgs a) {
    for (uint64_t L = blockIdx.x * (uint64_t)blockDim.x + threadIdx.x; L < a.lines;
         L += (uint64_t)gridDim.x * blockDim.x) {
        const uint64_t b = L / a.lines_per_slab;
        const uint64_t in_slab = L - b * a.lines_per_slab;
        const uint64_t tile = in_slab >> 5;
        const uint32_t r32 = (uint32_t)(in_slab & 31u);
        const uint32_t band = (uint32_t)(tile / a.col_tiles), ct = (uint32_t)(tile - (uint64_t)band * a.col_tiles);
        uint4 v;
        v.x = dense_word(a, b, band * 128u + r32, ct);
        v.y = dense_word(a, b, band * 128u + 32u + r32, ct);
        v.z = dense_word(a, b, band * 128u + 64u + r32, ct);
        v.w = dense_word(a, b, band * 128u + 96u + r32, ct);
        *reinterpret_cast<uint4*>(a.dst + L * 16u) = v;
    }
}

__device__ __forceinline__ void store_dense_word(const LayoutArgs& a, uint64_t b, uint32_t m, uint32_t ct,
                                                 uint32_t w) {
    if (m >= a.M) return;
    uint8_t* row = a.dst + (b * a.M + m) * (uint64_t)a.S;
    const uint32_t c0 = ct * 4u;
    if (a.rows4) {
        *reinterpret_cast<uint32_t*>(row + c0) = w;
        return;
    }
#pragma unroll
    for (int k = 0; k < 4; ++k)
        if (c0 + k < a.S) row[c0 + k] = (uint8_t)(w >> (8 * k));
}

__global__ void __launch_bounds__(kThreads) scales_from_mma_kernel(const LayoutArgs a) {
    for (uint64_t L = blockIdx.x * (uint64_t)blockDim.x + threadIdx.x; L < a.lines;
         L += (uint64_t)gridDim.x * blockDim.x) {
        const uint64_t b = L / a.lines_per_slab;
        const uint64_t in_slab = L - b * a.lines_per_slab;
        const uint64_t tile = in_slab >> 5;
        const uint32_t r32 = (uint32_t)(in_slab & 31u);
        const uint32_t band = (uint32_t)(tile / a.col_tiles), ct = (uint32_t)(tile - (uint64_t)band * a.col_tiles);
        const uint4 v = *reinterpret_cast<const uint4*>(a.src + L * 16u);
        store_dense_word(a, b, band * 128u + r32, ct, v.x);
        store_dense_word(a, b, band * 128u + 32u + r32, ct, v.y);
        store_dense_word(a, b, band * 128u + 64u + r32, ct, v.z);
        store_dense_word(a, b, band * 128u + 96u + r32, ct, v.w);
    }
}

LayoutArgs layout_args(const uint8_t* src, uint8_t* dst, const uint8_t* dense, int64_t B, int64_t M, int64_t S) {
    LayoutArgs a;
    a.src = src;
    a.dst = dst;
    a.M = (uint32_t)M;
    a.S = (uint32_t)S;
    a.col_tiles = (uint32_t)mma_scale_col_tiles(S);
    a.lines_per_slab = (uint64_t)mma_scale_slab_bytes(M, S) / 16u;
    a.lines = (uint64_t)B * a.lines_per_slab;
    a.rows4 = S % 4 == 0 && (uintptr_t)dense % 4 == 0;
    return a;
}

int layout_grid(uint64_t lines) {
    return persistent_grid((int64_t)((lines + kThreads - 1) / kThreads), 8);
}

}  // namespace

cudaError_t launch_scales_to_mma(const uint8_t* dense, int64_t B, int64_t M, int64_t S, uint8_t* mma,
                                 cudaStream_t s) {
    const LayoutArgs a = layout_args(dense, mma, dense, B, M, S);
    if (a.lines == 0) return cudaSuccess;
    scales_to_mma_kernel<<<layout_grid(a.lines), kThreads, 0, s>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_scales_from_mma(const uint8_t* mma, int64_t B, int64_t M, int64_t S, uint8_t* dense,
                                   cudaStream_t s) {
    const LayoutArgs a = layout_args(mma, dense, dense, B, M, S);
    if (a.lines == 0) return cudaSuccess;
    scales_from_mma_kernel<<<layout_grid(a.lines), kThreads, 0, s>>>(a);
    return cudaGetLastError();
}

}  // namespace pwq
