// requant.cu -- FP8 block-wise weights (E4M3 codes, FP32 scale per 128x128
// tile) straight into a rollout format, without the BF16 tensor in HBM.
// Source: "低精度训练与 Rollout", "FP8 训练 + FP8 Rollout" / "实现说明" item 3
// (on a weight update the FP8 training weights are dequantised to BF16 and
// then quantised into the rollout format); the formats as in fp8_block.cu,
// mxfp8.cu and nvfp4.cu.
//
// The result is defined as quant(dequant(q, s)) with y = bf16(fl(dec(q) * s))
// and is computed exactly so: every kernel dequantises its codes in registers
// with the same expression as fp8_block_dequant and quantises those BF16
// values with the same arithmetic as the BF16 quantisers.  One shortcut is
// exact: the amax of a set of y that share one tile scale is
// bf16(fl(dec(mc) * |s|)) for the set's largest code magnitude mc, because
// the rounding is monotone and symmetric in sign.
//
//   FP8 block -> FP8 block: one CTA per 128x128 tile (persistent grid); each
//     thread holds 64 codes (8-byte loads, 16 threads per tile row), one
//     barrier combines the warp maxima, then codes are re-encoded against
//     the new tile scale by the verified reciprocal path.  2 B per element.
//   FP8 block -> MXFP8: a chunk walk like mxfp8_quant's; four lanes hold one
//     1x32 block (which never leaves its 128-wide tile), the block amax comes
//     from the largest code magnitude and the tile scale.  2 + 1/32 B per
//     element.
//   FP8 block -> NVFP4: the NVFP4 amax and encode kernels with an FP8 source
//     (nvfp4.cu).
#include <algorithm>

#include "pwq_internal.h"

namespace pwq {
namespace {

constexpr int kThreads = 256;
constexpr int kTile = 128;
constexpr int kRowsPerPass = kThreads / 16;    // 16 rows of 16 threads x 8 codes
constexpr int kChunks = kTile / kRowsPerPass;  // 8 chunks of 8 codes per thread

struct TileArgs {
    const char* q;            // E4M3 codes in
    char* q2;                 // E4M3 codes out (may be q)
    int64_t q_bs, q_rs, o_bs, o_rs;   // bytes
    const float* s;           // [B][TM][TN] in
    float* s2;                // [B][TM][TN] out (may be s)
    int rows, cols;
    uint32_t tiles;           // B * TM * TN
    FastDiv tiles_n, tiles_mn;
};

template <bool kFast>
__device__ __forceinline__ uint2 requant8(uint2 c, float s, float s2, float r2) {
    const uint4 y = fp8_dequant8(c, s);
    float q[8];
    quotients8<kFast>(y, s2, r2, q);
    return make_uint2(e4m3x4(q[0], q[1], q[2], q[3]), e4m3x4(q[4], q[5], q[6], q[7]));
}

__global__ void __launch_bounds__(kThreads, 4) fp8_requant_fp8_kernel(const __grid_constant__ TileArgs a) {
    __shared__ uint32_t red[2][kThreads / 32];
    const uint32_t tid = threadIdx.x, lane = tid & 31u, warp = tid >> 5;
    const int ccol = (int)(tid & 15u) * 8;
    const int row0 = (int)(tid >> 4);
    uint32_t par = 0;
    for (uint32_t t = blockIdx.x; t < a.tiles; t += gridDim.x, par ^= 1u) {
        const uint32_t b = fdiv(t, a.tiles_mn);
        const uint32_t rem = t - b * a.tiles_mn.d;
        const uint32_t tm = fdiv(rem, a.tiles_n);
        const uint32_t tn = rem - tm * a.tiles_n.d;
        const float s = a.s[t];
        const char* qt = a.q + (int64_t)b * a.q_bs + (int64_t)tm * kTile * a.q_rs + (int64_t)tn * kTile;
        char* ot = a.q2 + (int64_t)b * a.o_bs + (int64_t)tm * kTile * a.o_rs + (int64_t)tn * kTile;
        const int rows_here = min(kTile, a.rows - (int)tm * kTile);
        const int cols_here = min(kTile, a.cols - (int)tn * kTile);
        const bool full = rows_here == kTile && cols_here == kTile;
        uint2 v[kChunks];
        if (full) {
#pragma unroll
            for (int j = 0; j < kChunks; ++j) v[j] = ld_stream_v2(qt + (int64_t)(row0 + kRowsPerPass * j) * a.q_rs + ccol);
        } else {
#pragma unroll
            for (int j = 0; j < kChunks; ++j) {
                const int r = row0 + kRowsPerPass * j;
                uint64_t w = 0u;
                if (r < rows_here) {
                    const unsigned char* src = reinterpret_cast<const unsigned char*>(qt + (int64_t)r * a.q_rs);
                    for (int c = ccol; c < min(ccol + 8, cols_here); ++c) w |= (uint64_t)src[c] << (8 * (c - ccol));
                }
                v[j] = make_uint2((uint32_t)w, (uint32_t)(w >> 32));
            }
        }
        uint32_t m = 0u;
#pragma unroll
        for (int j = 0; j < kChunks; ++j) m = max(m, e4m3_maxmag8(v[j]));
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, o));
        if (lane == 0u) red[par][warp] = m;
        __syncthreads();   // codes of the tile all read (in place is safe from here on)
#pragma unroll
        for (int w = 0; w < kThreads / 32; ++w) m = max(m, red[par][w]);
        const float amax = __uint_as_float(fp8_amax_bits16(m, s) << 16);
        const float s2 = fp8_tile_scale(amax);
        if (tid == 0) a.s2[t] = s2;
        const bool fast = div_fast_ok(s2);   // CTA-uniform
        const float r2 = fast ? __frcp_rn(s2) : 0.0f;
        uint2 o[kChunks];
#pragma unroll
        for (int j = 0; j < kChunks; ++j) o[j] = fast ? requant8<true>(v[j], s, s2, r2) : requant8<false>(v[j], s, s2, r2);
        if (full) {
#pragma unroll
            for (int j = 0; j < kChunks; ++j) st_v2(ot + (int64_t)(row0 + kRowsPerPass * j) * a.o_rs + ccol, o[j]);
        } else {
#pragma unroll
            for (int j = 0; j < kChunks; ++j) {
                const int r = row0 + kRowsPerPass * j;
                if (r >= rows_here) continue;
                unsigned char* dst = reinterpret_cast<unsigned char*>(ot + (int64_t)r * a.o_rs);
                const uint64_t w = (uint64_t)o[j].x | ((uint64_t)o[j].y << 32);
                for (int c = ccol; c < min(ccol + 8, cols_here); ++c) dst[c] = (unsigned char)(w >> (8 * (c - ccol)));
            }
        }
    }
}

constexpr int kUnroll = 4;
constexpr uint32_t kSpan = 32u * kUnroll;   // chunks per warp span

struct MxArgs {
    const char* q;            // E4M3 codes in
    char* q2;                 // E4M3 codes out (may be q)
    int64_t q_bs, q_rs, o_bs, o_rs;   // bytes
    const float* s;           // [B][TM][TN]
    uint8_t* e;               // dense [B][M][N/32]
    uint32_t chunks;          // B * M * N / 8
    uint32_t tm, tn;          // tiles per column, per row
    FastDiv cpr, rows;        // chunks per row (N / 8), M
    int dense;
};

__global__ void __launch_bounds__(kThreads) fp8_requant_mxfp8_kernel(const __grid_constant__ MxArgs a) {
    const uint32_t lane = threadIdx.x & 31u;
    const uint32_t gwarp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const uint32_t nwarps = (gridDim.x * blockDim.x) >> 5;
    for (uint32_t base = gwarp * kSpan; base < a.chunks; base += nwarps * kSpan) {
        uint2 v[kUnroll];
        float s[kUnroll];
        int64_t oo[kUnroll];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const uint32_t c = base + u * 32u + lane;
            const uint32_t R = fdiv(c, a.cpr);           // row over all batches
            const uint32_t k = c - R * a.cpr.d;          // chunk within the row
            const uint32_t b = fdiv(R, a.rows);
            const uint32_t m = R - b * a.rows.d;
            int64_t io;
            if (a.dense) {
                io = (int64_t)c * 8;
                oo[u] = io;
            } else {
                io = (int64_t)b * a.q_bs + (int64_t)m * a.q_rs + (int64_t)k * 8;
                oo[u] = (int64_t)b * a.o_bs + (int64_t)m * a.o_rs + (int64_t)k * 8;
            }
            v[u] = make_uint2(0u, 0u);
            s[u] = 0.0f;
            if (c < a.chunks) {
                v[u] = ld_stream_v2(a.q + io);
                s[u] = __ldg(a.s + ((int64_t)b * a.tm + (m >> 7)) * a.tn + (k >> 4));
            }
        }
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const uint32_t c = base + u * 32u + lane;
            // four lanes hold one 1x32 block, inside one 128-wide tile
            uint32_t mc = e4m3_maxmag8(v[u]);
            mc = max(mc, __shfl_xor_sync(0xffffffffu, mc, 1));
            mc = max(mc, __shfl_xor_sync(0xffffffffu, mc, 2));
            const int e = ue8m0_exponent(fp8_amax_bits16(mc, s[u]));
            const float inv = exp2i(-e);   // exact power of two
            const uint4 y = fp8_dequant8(v[u], s[u]);
            uint2 out;
            out.x = e4m3x4(__fmul_rn(bf16_lo(y.x), inv), __fmul_rn(bf16_hi(y.x), inv),
                           __fmul_rn(bf16_lo(y.y), inv), __fmul_rn(bf16_hi(y.y), inv));
            out.y = e4m3x4(__fmul_rn(bf16_lo(y.z), inv), __fmul_rn(bf16_hi(y.z), inv),
                           __fmul_rn(bf16_lo(y.w), inv), __fmul_rn(bf16_hi(y.w), inv));
            if (c < a.chunks) {
                st_v2(a.q2 + oo[u], out);
                if ((lane & 3u) == 0u) a.e[c >> 2] = (uint8_t)(e + 127);
            }
        }
    }
}

}  // namespace

cudaError_t launch_fp8_requant_fp8(const View& q, const float* s, const View& q2, float* s2, cudaStream_t st) {
    TileArgs a;
    a.q = q.ptr;
    a.q2 = q2.ptr;
    a.q_bs = q.bstride;
    a.q_rs = q.rstride;
    a.o_bs = q2.bstride;
    a.o_rs = q2.rstride;
    a.s = s;
    a.s2 = s2;
    a.rows = (int)q.rows;
    a.cols = (int)q.cols;
    const uint32_t tm = (uint32_t)((q.rows + kTile - 1) / kTile);
    const uint32_t tn = (uint32_t)((q.cols + kTile - 1) / kTile);
    a.tiles = (uint32_t)q.batch * tm * tn;
    a.tiles_n = make_fastdiv(tn);
    a.tiles_mn = make_fastdiv(tm * tn);
    if (a.tiles == 0) return cudaSuccess;
    const int grid = persistent_grid(a.tiles, 4);
    fp8_requant_fp8_kernel<<<grid, kThreads, 0, st>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_fp8_requant_mxfp8(const View& q, const float* s, const View& q2, uint8_t* e, cudaStream_t st) {
    MxArgs a;
    a.q = q.ptr;
    a.q2 = q2.ptr;
    a.q_bs = q.bstride;
    a.q_rs = q.rstride;
    a.o_bs = q2.bstride;
    a.o_rs = q2.rstride;
    a.s = s;
    a.e = e;
    a.chunks = (uint32_t)(q.batch * q.rows * (q.cols / 8));
    a.tm = (uint32_t)((q.rows + kTile - 1) / kTile);
    a.tn = (uint32_t)((q.cols + kTile - 1) / kTile);
    a.cpr = make_fastdiv((uint32_t)std::max<int64_t>(1, q.cols / 8));
    a.rows = make_fastdiv((uint32_t)std::max<int64_t>(1, q.rows));
    a.dense = q.rstride == q.cols && q2.rstride == q2.cols &&
              (q.batch == 1 || (q.bstride == q.rows * q.cols && q2.bstride == q2.rows * q2.cols));
    if (a.chunks == 0) return cudaSuccess;
    const int grid = persistent_grid((a.chunks + kThreads * kUnroll - 1) / (kThreads * kUnroll), 8);
    fp8_requant_mxfp8_kernel<<<grid, kThreads, 0, st>>>(a);
    return cudaGetLastError();
}

}  // namespace pwq
