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
//   FP8 block -> FP8 block: one CTA per 128x128 tile (persistent grid);
//     the TMA path (fp8_block.cu, 16-byte aligned code rows) stages tiles in
//     a ring and maps every code through a per-tile 256-entry table (within
//     a tile the output code is a function of the input code alone); the
//     fallback here holds 64 codes per thread (8-byte loads, 16 threads per
//     tile row), one barrier combines the warp maxima, then codes are
//     re-encoded against the new tile scale by the verified reciprocal path.
//     2 B per element.
//   FP8 block -> MXFP8: a block walk like mxfp8_quant's; with 16-byte
//     aligned code rows one lane holds one 1x32 block (which never leaves
//     its 128-wide tile), whose amax comes from the largest code magnitude
//     and the tile scale; 8-byte aligned rows take a per-tensor kernel of
//     8-code chunks, four lanes per block.  2 + 1/32 B per element.
//   FP8 block -> NVFP4: the NVFP4 single-pass kernel with an FP8 source
//     (nvfp4.cu).
#include <algorithm>

#include "pwq_internal.h"

namespace pwq {
namespace {

constexpr int kThreads = 256;
constexpr int kTile = 128;
constexpr int kRowsPerPass = kThreads / 16;    // 16 rows of 16 threads x 8 codes
constexpr int kChunks = kTile / kRowsPerPass;  // 8 chunks of 8 codes per thread

// One tensor of a grouped FP8 -> FP8 launch.
struct RqTensor {
    const char* q;            // E4M3 codes in
    char* q2;                 // E4M3 codes out (may be q)
    int64_t q_bs, q_rs, o_bs, o_rs;   // bytes
    const float* s;           // [B][TM][TN] in
    float* s2;                // [B][TM][TN] out (may be s)
    int rows, cols;
    uint32_t tile_begin;      // first tile of this tensor in the launch
    FastDiv tiles_n, tiles_mn;
};

struct TileArgs {
    RqTensor t[kMaxLaunchTensors];
    int n;
    uint32_t total_tiles;
};

// Where tile `tile` of the launch lives, and its old scale.
struct TileWork {
    const char* qt;
    char* ot;
    int64_t q_rs, o_rs;
    float* s2;                // address of the new scale
    float s;
    int rows_here, cols_here;
};

__device__ __forceinline__ TileWork tile_work(const TileArgs& a, uint32_t tile) {
    int i = 0;
    for (int k = 1; k < a.n; ++k)
        if (tile >= a.t[k].tile_begin) i = k;
    const RqTensor& T = a.t[i];
    const uint32_t lt = tile - T.tile_begin;
    const uint32_t b = fdiv(lt, T.tiles_mn);
    const uint32_t rem = lt - b * T.tiles_mn.d;
    const uint32_t tm = fdiv(rem, T.tiles_n);
    const uint32_t tn = rem - tm * T.tiles_n.d;
    TileWork w;
    w.qt = T.q + (int64_t)b * T.q_bs + (int64_t)tm * kTile * T.q_rs + (int64_t)tn * kTile;
    w.ot = T.q2 + (int64_t)b * T.o_bs + (int64_t)tm * kTile * T.o_rs + (int64_t)tn * kTile;
    w.q_rs = T.q_rs;
    w.o_rs = T.o_rs;
    w.s2 = T.s2 + lt;
    w.s = T.s[lt];
    w.rows_here = min(kTile, T.rows - (int)tm * kTile);
    w.cols_here = min(kTile, T.cols - (int)tn * kTile);
    return w;
}

__device__ __forceinline__ void load_tile(const TileWork& w, int row0, int ccol, uint2 (&v)[kChunks]) {
    if (w.rows_here == kTile && w.cols_here == kTile) {
#pragma unroll
        for (int j = 0; j < kChunks; ++j) v[j] = ld_stream_v2(w.qt + (int64_t)(row0 + kRowsPerPass * j) * w.q_rs + ccol);
    } else {
#pragma unroll
        for (int j = 0; j < kChunks; ++j) {
            const int r = row0 + kRowsPerPass * j;
            uint64_t x = 0u;
            if (r < w.rows_here) {
                const unsigned char* src = reinterpret_cast<const unsigned char*>(w.qt + (int64_t)r * w.q_rs);
                for (int c = ccol; c < min(ccol + 8, w.cols_here); ++c) x |= (uint64_t)src[c] << (8 * (c - ccol));
            }
            v[j] = make_uint2((uint32_t)x, (uint32_t)(x >> 32));
        }
    }
}

// Persistent CTAs over the tiles of all tensors of the launch; each thread
// holds the codes of the next tile (loads in flight) while it re-encodes the
// current one.
__global__ void __launch_bounds__(kThreads, 3) fp8_requant_fp8_kernel(const __grid_constant__ TileArgs a) {
    __shared__ uint32_t red[2][kThreads / 32];
    const uint32_t tid = threadIdx.x, lane = tid & 31u, warp = tid >> 5;
    const int ccol = (int)(tid & 15u) * 8;
    const int row0 = (int)(tid >> 4);
    uint32_t t = blockIdx.x;
    if (t >= a.total_tiles) return;
    TileWork w = tile_work(a, t);
    uint2 v[kChunks];
    load_tile(w, row0, ccol, v);
    for (uint32_t par = 0;; par ^= 1u) {
        const uint32_t tn = t + gridDim.x;
        TileWork nw;
        uint2 nv[kChunks];
        if (tn < a.total_tiles) {
            nw = tile_work(a, tn);
            load_tile(nw, row0, ccol, nv);
        }
        uint32_t m = 0u;
#pragma unroll
        for (int j = 0; j < kChunks; ++j) m = __vmaxu2(m, e4m3_maxmag_lanes(v[j]));
        m = e4m3_maxmag_fin(m);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, o));
        if (lane == 0u) red[par][warp] = m;
        __syncthreads();   // codes of the tile all read (in place is safe from here on)
#pragma unroll
        for (int k = 0; k < kThreads / 32; ++k) m = max(m, red[par][k]);
        const float amax = __uint_as_float(fp8_amax_bits16(m, w.s) << 16);
        const float s2 = fp8_tile_scale(amax);
        if (tid == 0) *w.s2 = s2;
        const bool fast = div_fast_ok(s2);   // CTA-uniform
        const float r2 = fast ? __frcp_rn(s2) : 0.0f;
        uint2 o[kChunks];
#pragma unroll
        for (int j = 0; j < kChunks; ++j) o[j] = fast ? fp8_requant8<true>(v[j], w.s, s2, r2) : fp8_requant8<false>(v[j], w.s, s2, r2);
        if (w.rows_here == kTile && w.cols_here == kTile) {
#pragma unroll
            for (int j = 0; j < kChunks; ++j) st_v2(w.ot + (int64_t)(row0 + kRowsPerPass * j) * w.o_rs + ccol, o[j]);
        } else {
#pragma unroll
            for (int j = 0; j < kChunks; ++j) {
                const int r = row0 + kRowsPerPass * j;
                if (r >= w.rows_here) continue;
                unsigned char* dst = reinterpret_cast<unsigned char*>(w.ot + (int64_t)r * w.o_rs);
                const uint64_t x = (uint64_t)o[j].x | ((uint64_t)o[j].y << 32);
                for (int c = ccol; c < min(ccol + 8, w.cols_here); ++c) dst[c] = (unsigned char)(x >> (8 * (c - ccol)));
            }
        }
        if (tn >= a.total_tiles) break;
        t = tn;
        w = nw;
#pragma unroll
        for (int j = 0; j < kChunks; ++j) v[j] = nv[j];
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

// Grouped FP8 -> MXFP8 (16-byte aligned code rows): each lane takes
// kMxBlocksPerLane 1x32 blocks a warp span apart, loading all their codes
// (two 16-byte loads each) and tile scales before encoding any, then two
// 16-byte stores and a scale byte per block.  One block per lane measured
// 1.43 ms per 36-layer sweep, two 1.32, four 1.27, eight (126 registers)
// 1.49.
struct MxBlkTensor {
    const char* q;
    char* q2;
    int64_t q_bs, q_rs, o_bs, o_rs;   // bytes
    const float* s;           // [B][TM][TN]
    uint8_t* e;               // dense [B][M][N/32]
    uint32_t chunks;          // 32-code blocks: B * M * N / 32
    uint32_t slot_begin;      // multiple of one warp span (32 kMxBlocksPerLane)
    uint32_t tm, tn;
    FastDiv cpr, rows;        // blocks per row (N / 32), M
    int dense;
};

// 32-code blocks per lane per step of the block walk (their loads in
// flight together)
constexpr uint32_t kMxBlocksPerLane = 4;
// CTAs launched per SM: about 4 are resident at the 64 registers a lane
// takes, and the rest start as those finish; measured faster (1.27 against
// 1.30 ms per 36-layer sweep) than a grid of resident CTAs only
constexpr int kMxGridPerSm = 8;

struct MxBlkArgs {
    MxBlkTensor t[kMaxLaunchTensors];
    int n;
    uint32_t total_slots;
};

__device__ __forceinline__ uint2 mx_encode8(uint4 y, float inv) {
    const uint64_t inv2 = f32x2(inv, inv);
    const uint32_t wv[4] = {y.x, y.y, y.z, y.w};
    float2 p[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        uint32_t lo;
        asm("mul.lo.u32 %0, %1, 0x10000;" : "=r"(lo) : "r"(wv[k]));
        p[k] = f32x2_split(mul_f32x2(f32x2_bits(lo, wv[k] & 0xffff0000u), inv2));
    }
    return make_uint2(e4m3x4(p[0].x, p[0].y, p[1].x, p[1].y), e4m3x4(p[2].x, p[2].y, p[3].x, p[3].y));
}

__global__ void __launch_bounds__(kThreads) fp8_requant_mxfp8_block_kernel(const __grid_constant__ MxBlkArgs a) {
    const uint32_t lane = threadIdx.x & 31u;
    const uint32_t gwarp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const uint32_t nwarps = (gridDim.x * blockDim.x) >> 5;
    constexpr uint32_t kSpan = 32u * kMxBlocksPerLane;
    for (uint32_t slot = gwarp * kSpan; slot < a.total_slots; slot += nwarps * kSpan) {
        int ti = 0;
        for (int k = 1; k < a.n; ++k)
            if (slot >= a.t[k].slot_begin) ti = k;
        const MxBlkTensor& T = a.t[ti];
        // every block's codes and tile scale are loaded before any is used:
        // kMxBlocksPerLane x 32 bytes in flight per lane
        uint4 v[kMxBlocksPerLane][2];
        float sc[kMxBlocksPerLane];
        uint32_t bis[kMxBlocksPerLane];
        int64_t oos[kMxBlocksPerLane];
#pragma unroll
        for (int u = 0; u < (int)kMxBlocksPerLane; ++u) {
            const uint32_t bi = slot - T.slot_begin + lane + 32u * u;   // 32-code block
            bis[u] = bi;
            v[u][0] = v[u][1] = make_uint4(0u, 0u, 0u, 0u);
            sc[u] = 0.0f;
            oos[u] = 0;
            if (bi >= T.chunks) continue;
            const uint32_t R = fdiv(bi, T.cpr);           // row over all batches
            const uint32_t k = bi - R * T.cpr.d;          // block within the row
            const uint32_t b = fdiv(R, T.rows);
            const uint32_t m = R - b * T.rows.d;
            int64_t io;
            if (T.dense) {
                io = (int64_t)bi * 32;
                oos[u] = io;
            } else {
                io = (int64_t)b * T.q_bs + (int64_t)m * T.q_rs + (int64_t)k * 32;
                oos[u] = (int64_t)b * T.o_bs + (int64_t)m * T.o_rs + (int64_t)k * 32;
            }
            v[u][0] = ld_stream_v4(T.q + io);
            v[u][1] = ld_stream_v4(T.q + io + 16);
            sc[u] = __ldg(T.s + ((int64_t)b * T.tm + (m >> 7)) * T.tn + (k >> 2));
        }
#pragma unroll
        for (int u = 0; u < (int)kMxBlocksPerLane; ++u) {
            if (bis[u] >= T.chunks) continue;
            const uint4 v0 = v[u][0], v1 = v[u][1];
            uint32_t lanes = __vmaxu2(e4m3_maxmag_lanes(make_uint2(v0.x, v0.y)),
                                      e4m3_maxmag_lanes(make_uint2(v0.z, v0.w)));
            lanes = __vmaxu2(lanes, __vmaxu2(e4m3_maxmag_lanes(make_uint2(v1.x, v1.y)),
                                             e4m3_maxmag_lanes(make_uint2(v1.z, v1.w))));
            const int e = ue8m0_exponent(fp8_amax_bits16(e4m3_maxmag_fin(lanes), sc[u]));
            const float inv = exp2i(-e);   // exact power of two
            const uint2 o0 = mx_encode8(fp8_dequant8(make_uint2(v0.x, v0.y), sc[u]), inv);
            const uint2 o1 = mx_encode8(fp8_dequant8(make_uint2(v0.z, v0.w), sc[u]), inv);
            const uint2 o2 = mx_encode8(fp8_dequant8(make_uint2(v1.x, v1.y), sc[u]), inv);
            const uint2 o3 = mx_encode8(fp8_dequant8(make_uint2(v1.z, v1.w), sc[u]), inv);
            st_v4(T.q2 + oos[u], make_uint4(o0.x, o0.y, o1.x, o1.y));
            st_v4(T.q2 + oos[u] + 16, make_uint4(o2.x, o2.y, o3.x, o3.y));
            T.e[bis[u]] = (uint8_t)(e + 127);
        }
    }
}

}  // namespace

cudaError_t launch_fp8_requant_fp8(const RequantJob* jobs, int n, cudaStream_t st) {
    if (fp8_requant_tma_ok(jobs, n)) return launch_fp8_requant_tma(jobs, n, st);
    for (int j0 = 0; j0 < n;) {
        TileArgs a;
        a.n = 0;
        uint32_t tiles = 0;
        for (; j0 + a.n < n && a.n < kMaxLaunchTensors; ++a.n) {
            const RequantJob& J = jobs[j0 + a.n];
            const uint32_t tm = (uint32_t)((J.in.rows + kTile - 1) / kTile);
            const uint32_t tn = (uint32_t)((J.in.cols + kTile - 1) / kTile);
            const uint64_t count = (uint64_t)J.in.batch * tm * tn;
            if (a.n > 0 && tiles + count > (uint64_t(1) << 31)) break;
            RqTensor& T = a.t[a.n];
            T.q = J.in.ptr;
            T.q2 = J.out.ptr;
            T.q_bs = J.in.bstride;
            T.q_rs = J.in.rstride;
            T.o_bs = J.out.bstride;
            T.o_rs = J.out.rstride;
            T.s = static_cast<const float*>(J.scale_in);
            T.s2 = static_cast<float*>(J.scale_out);
            T.rows = (int)J.in.rows;
            T.cols = (int)J.in.cols;
            T.tile_begin = tiles;
            T.tiles_n = make_fastdiv(tn);
            T.tiles_mn = make_fastdiv(tm * tn);
            tiles += (uint32_t)count;
        }
        j0 += a.n;
        a.total_tiles = tiles;
        if (tiles == 0) continue;
        fp8_requant_fp8_kernel<<<persistent_grid(tiles, 3), kThreads, 0, st>>>(a);
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

namespace {

bool aligned16(const View& v) {
    return (uintptr_t)v.ptr % 16 == 0 && v.rstride % 16 == 0 && (v.batch <= 1 || v.bstride % 16 == 0);
}

cudaError_t launch_mx8(const RequantJob& J, cudaStream_t st) {
    const View& q = J.in;
    const View& q2 = J.out;
    MxArgs a;
    a.q = q.ptr;
    a.q2 = q2.ptr;
    a.q_bs = q.bstride;
    a.q_rs = q.rstride;
    a.o_bs = q2.bstride;
    a.o_rs = q2.rstride;
    a.s = static_cast<const float*>(J.scale_in);
    a.e = static_cast<uint8_t*>(J.scale_out);
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

}  // namespace

cudaError_t launch_fp8_requant_mxfp8(const RequantJob* jobs, int n, cudaStream_t st) {
    bool all16 = true;
    for (int i = 0; i < n; ++i) all16 = all16 && aligned16(jobs[i].in) && aligned16(jobs[i].out);
    if (!all16) {   // 8-byte code rows: one launch per tensor with 8-code chunks
        for (int i = 0; i < n; ++i) {
            cudaError_t e = launch_mx8(jobs[i], st);
            if (e != cudaSuccess) return e;
        }
        return cudaSuccess;
    }
    const uint64_t kMaxSlots = uint64_t(1) << 31;
    for (int j0 = 0; j0 < n;) {
        MxBlkArgs a;
        a.n = 0;
        uint32_t slots = 0;
        for (; j0 + a.n < n && a.n < kMaxLaunchTensors; ++a.n) {
            const RequantJob& J = jobs[j0 + a.n];
            const View& q = J.in;
            const View& q2 = J.out;
            const uint64_t chunks = (uint64_t)(q.batch * q.rows * (q.cols / 32));
            const uint64_t span = 32u * kMxBlocksPerLane;
            const uint64_t padded = (chunks + span - 1) / span * span;
            if (a.n > 0 && slots + padded > kMaxSlots) break;
            MxBlkTensor& T = a.t[a.n];
            T.q = q.ptr;
            T.q2 = q2.ptr;
            T.q_bs = q.bstride;
            T.q_rs = q.rstride;
            T.o_bs = q2.bstride;
            T.o_rs = q2.rstride;
            T.s = static_cast<const float*>(J.scale_in);
            T.e = static_cast<uint8_t*>(J.scale_out);
            T.chunks = (uint32_t)chunks;
            T.slot_begin = slots;
            T.tm = (uint32_t)((q.rows + kTile - 1) / kTile);
            T.tn = (uint32_t)((q.cols + kTile - 1) / kTile);
            T.cpr = make_fastdiv((uint32_t)std::max<int64_t>(1, q.cols / 32));
            T.rows = make_fastdiv((uint32_t)std::max<int64_t>(1, q.rows));
            T.dense = q.rstride == q.cols && q2.rstride == q2.cols &&
                      (q.batch == 1 || (q.bstride == q.rows * q.cols && q2.bstride == q2.rows * q2.cols));
            slots += (uint32_t)padded;
        }
        j0 += a.n;
        a.total_slots = slots;
        if (slots == 0) continue;
        const int grid = persistent_grid((slots + kThreads * kMxBlocksPerLane - 1) / (kThreads * kMxBlocksPerLane), kMxGridPerSm);
        fp8_requant_mxfp8_block_kernel<<<grid, kThreads, 0, st>>>(a);
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

}  // namespace pwq
