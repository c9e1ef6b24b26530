// mxfp8.cu -- MXFP8 quantise / dequantise (1x32 blocks, UE8M0 scale byte,
// E4M3 codes).  Source: "Low Precision RL", "Choose a precision" table and
// "Modes" 3 (MXFP8: 1x32 blocks, power-of-two UE8M0 scales packed as uint8,
// float8_e4m3fn weights).
//
// HBM-bound elementwise kernels over a list of up to kMaxLaunchTensors
// tensors per launch, walked by a persistent grid in warp-sized spans; every
// tensor's range is padded to a whole number of spans so a span never
// straddles two tensors.  The scale is a power of two, so x * 2^-e is an
// exact multiply and no division is needed.
//
// Quantise: one thread per 32-element block (64 bytes of BF16 in, 32 codes
// and one scale byte out), so the block amax needs no lane exchange and the
// exponent is found once per block; each lane loads kQBlocksPerLane blocks
// (a warp span apart) before encoding any, 256 bytes in flight per lane
// (one block per lane measured 1.88 ms per 36-layer sweep, two 1.79, four
// 1.70).  Dequantise: when every code tensor of the call has 16-byte
// aligned rows, 16-element chunks (16 code bytes in, 32 bytes of BF16 out
// in one 256-bit store), eight per lane in flight; otherwise 8-element
// chunks (8 code bytes in, 16 bytes out), kUnroll in flight.  Each chunk
// reads its block's scale byte.
#include <algorithm>

#include "pwq_internal.h"

namespace pwq {
namespace {

constexpr int kThreads = 256;
constexpr int kUnroll = 2;
constexpr uint32_t kSpan = 32u * kUnroll;   // chunks per warp span

struct ChunkTensor {
    const char* in;
    char* out;
    int64_t in_bs, in_rs, out_bs, out_rs;   // bytes
    uint8_t* e;            // dense [B][M][N/32] scale bytes
    uint32_t chunks;       // B * M * N / 8
    uint32_t slot_begin;   // first chunk slot of this tensor (multiple of kSpan)
    FastDiv cpr;           // chunks per row (N / 8)
    FastDiv rows;          // M
    int dense;             // both operands dense: chunk c at in + c*in_chunk, out + c*out_chunk
};

struct ChunkArgs {
    ChunkTensor t[kMaxLaunchTensors];
    int n;
    uint32_t total_slots;
};

__device__ __forceinline__ int span_tensor(const ChunkArgs& a, uint32_t slot) {
    int i = 0;
    for (int k = 1; k < a.n; ++k)
        if (slot >= a.t[k].slot_begin) i = k;
    return i;
}

// Byte offsets of chunk c of T (input chunk in_chunk bytes, output out_chunk).
__device__ __forceinline__ void chunk_offsets(const ChunkTensor& T, uint32_t c, int in_chunk, int out_chunk,
                                              int64_t& io, int64_t& oo) {
    if (T.dense) {
        io = (int64_t)c * in_chunk;
        oo = (int64_t)c * out_chunk;
    } else {
        const uint32_t r = fdiv(c, T.cpr);           // row over all batches
        const uint32_t k = c - r * T.cpr.d;
        const uint32_t b = fdiv(r, T.rows);
        const uint32_t m = r - b * T.rows.d;
        io = (int64_t)b * T.in_bs + (int64_t)m * T.in_rs + (int64_t)k * in_chunk;
        oo = (int64_t)b * T.out_bs + (int64_t)m * T.out_rs + (int64_t)k * out_chunk;
    }
}

__global__ void __launch_bounds__(kThreads) mxfp8_dequant_kernel(const __grid_constant__ ChunkArgs a) {
    const uint32_t lane = threadIdx.x & 31u;
    const uint32_t gwarp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const uint32_t nwarps = (gridDim.x * blockDim.x) >> 5;
    for (uint32_t slot = gwarp * kSpan; slot < a.total_slots; slot += nwarps * kSpan) {
        const ChunkTensor& T = a.t[span_tensor(a, slot)];
        const uint32_t base = slot - T.slot_begin;
        uint2 v[kUnroll];
        uint32_t eb[kUnroll];
        int64_t yo[kUnroll];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const uint32_t c = base + u * 32u + lane;
            int64_t qo;
            chunk_offsets(T, c, 8, 16, qo, yo[u]);
            v[u] = make_uint2(0u, 0u);
            eb[u] = 127u;
            if (c < T.chunks) {
                v[u] = ld_stream_v2(T.in + qo);
                eb[u] = __ldg(T.e + (c >> 2));
            }
        }
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const uint32_t c = base + u * 32u + lane;
            const float p2 = exp2i((int)eb[u] - 127);
            uint4 out;
            float2 f;
            f = e4m3x2_decode(v[u].x & 0xffffu);
            out.x = pack_bf16x2(__fmul_rn(f.x, p2), __fmul_rn(f.y, p2));
            f = e4m3x2_decode(v[u].x >> 16);
            out.y = pack_bf16x2(__fmul_rn(f.x, p2), __fmul_rn(f.y, p2));
            f = e4m3x2_decode(v[u].y & 0xffffu);
            out.z = pack_bf16x2(__fmul_rn(f.x, p2), __fmul_rn(f.y, p2));
            f = e4m3x2_decode(v[u].y >> 16);
            out.w = pack_bf16x2(__fmul_rn(f.x, p2), __fmul_rn(f.y, p2));
            if (c < T.chunks) st_v4(T.out + yo[u], out);
        }
    }
}

// Dequantise with 16-code chunks (code rows 16-byte aligned): a chunk lies in
// one 1x32 block, so one scale byte serves it; 16 code bytes in, 32 bytes of
// BF16 out in one 256-bit store when the BF16 rows are 32-byte aligned.  A
// lane loads kDq16Unroll chunks, a warp span apart, before storing any.
// Streams that write twice what they read run far below the copy rate with
// 16-byte stores; 32-byte stores and more loads in flight close the gap.
struct Chunk16Tensor {
    const char* in;
    char* out;
    int64_t in_bs, in_rs, out_bs, out_rs;   // bytes
    uint8_t* e;            // dense [B][M][N/32] scale bytes
    uint32_t chunks;       // B * M * N / 16
    uint32_t slot_begin;   // first chunk slot of this tensor (multiple of kSpan16)
    FastDiv cpr;           // chunks per row (N / 16)
    FastDiv rows;          // M
    int dense;             // both operands dense
    int out32;             // BF16 base, row and slab strides multiples of 32 bytes
};

struct Chunk16Args {
    Chunk16Tensor t[kMaxLaunchTensors];
    int n;
    uint32_t total_slots;
};

constexpr int kDq16Unroll = 8;
constexpr uint32_t kSpan16 = 32u * kDq16Unroll;

__global__ void __launch_bounds__(kThreads) mxfp8_dequant16_kernel(const __grid_constant__ Chunk16Args a) {
    const uint32_t lane = threadIdx.x & 31u;
    const uint32_t gwarp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const uint32_t nwarps = (gridDim.x * blockDim.x) >> 5;
    for (uint32_t slot = gwarp * kSpan16; slot < a.total_slots; slot += nwarps * kSpan16) {
        int ti = 0;
        for (int k = 1; k < a.n; ++k)
            if (slot >= a.t[k].slot_begin) ti = k;
        const Chunk16Tensor& T = a.t[ti];
        const uint32_t base = slot - T.slot_begin;
        uint4 v[kDq16Unroll];
        uint32_t eb[kDq16Unroll];
        int64_t yo[kDq16Unroll];
#pragma unroll
        for (int u = 0; u < kDq16Unroll; ++u) {
            const uint32_t c = base + u * 32u + lane;
            int64_t qo;
            if (T.dense) {
                qo = (int64_t)c * 16;
                yo[u] = (int64_t)c * 32;
            } else {
                const uint32_t r = fdiv(c, T.cpr);           // row over all batches
                const uint32_t k = c - r * T.cpr.d;
                const uint32_t b = fdiv(r, T.rows);
                const uint32_t m = r - b * T.rows.d;
                qo = (int64_t)b * T.in_bs + (int64_t)m * T.in_rs + (int64_t)k * 16;
                yo[u] = (int64_t)b * T.out_bs + (int64_t)m * T.out_rs + (int64_t)k * 32;
            }
            v[u] = make_uint4(0u, 0u, 0u, 0u);
            eb[u] = 127u;
            if (c < T.chunks) {
                v[u] = ld_stream_v4(T.in + qo);
                eb[u] = __ldg(T.e + (c >> 1));
            }
        }
#pragma unroll
        for (int u = 0; u < kDq16Unroll; ++u) {
            const uint32_t c = base + u * 32u + lane;
            if (c >= T.chunks) continue;
            const float p2 = exp2i((int)eb[u] - 127);
            const uint32_t w[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
            uint32_t o[8];
#pragma unroll
            for (int h = 0; h < 8; ++h) {
                const float2 f = e4m3x2_decode((w[h >> 1] >> (16 * (h & 1))) & 0xffffu);
                o[h] = pack_bf16x2(__fmul_rn(f.x, p2), __fmul_rn(f.y, p2));
            }
            const uint4 y0 = make_uint4(o[0], o[1], o[2], o[3]), y1 = make_uint4(o[4], o[5], o[6], o[7]);
            if (T.out32) {
                st_v8(T.out + yo[u], y0, y1);
            } else {
                st_v4(T.out + yo[u], y0);
                st_v4(T.out + yo[u] + 16, y1);
            }
        }
    }
}

bool dense_view(const View& v, int64_t row_bytes) {
    return v.rstride == row_bytes && (v.batch == 1 || v.bstride == v.rows * v.rstride);
}

// ---------------------------------------------------------------- quantise: one thread per block
//
// Each thread owns whole 32-element blocks: 64 bytes of BF16 in (two
// 256-bit loads when the rows are 32-byte aligned, else four 128-bit ones),
// one block amax, one scale exponent, 32 codes and one scale byte out.  No
// lane exchange, and the per-block work is paid once per 32 elements.
constexpr uint32_t kQBlocksPerLane = 4;           // blocks a lane loads before encoding any
constexpr uint32_t kBSpan = 32u * kQBlocksPerLane;  // blocks per warp span

struct BlockTensor {
    const char* in;
    char* out;
    int64_t in_bs, in_rs, out_bs, out_rs;   // bytes
    uint8_t* e;            // scale bytes: dense [B][M][N/32], or the tensor-core tile layout
    uint32_t blocks;       // B * M * N / 32
    uint32_t slot_begin;   // first block slot of this tensor (multiple of kBSpan)
    FastDiv bpr;           // blocks per row (N / 32)
    FastDiv rows;          // M
    int dense;             // both operands dense
    int in32, out32;       // BF16 rows / code rows (and slabs) 32-byte aligned
    int sf_mma;            // scales in the tile layout: sf_ct column tiles, sf_slab bytes per batch slab
    uint32_t sf_ct;
    int64_t sf_slab;
};

struct BlockArgs {
    BlockTensor t[kMaxLaunchTensors];
    int n;
    uint32_t total_slots;
};

__device__ __forceinline__ int block_span_tensor(const BlockArgs& a, uint32_t slot) {
    int i = 0;
    for (int k = 1; k < a.n; ++k)
        if (slot >= a.t[k].slot_begin) i = k;
    return i;
}

__global__ void __launch_bounds__(kThreads) mxfp8_quant_block_kernel(const __grid_constant__ BlockArgs a) {
    const uint32_t lane = threadIdx.x & 31u;
    const uint32_t gwarp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const uint32_t nwarps = (gridDim.x * blockDim.x) >> 5;
    for (uint32_t slot = gwarp * kBSpan; slot < a.total_slots; slot += nwarps * kBSpan) {
        const BlockTensor& T = a.t[block_span_tensor(a, slot)];
        uint4 v[kQBlocksPerLane][4];
        int64_t oo[kQBlocksPerLane];
        uint32_t bis[kQBlocksPerLane];
#pragma unroll
        for (int u = 0; u < (int)kQBlocksPerLane; ++u) {
            const uint32_t bi = slot - T.slot_begin + lane + 32u * u;
            bis[u] = bi;
            oo[u] = 0;
#pragma unroll
            for (int h = 0; h < 4; ++h) v[u][h] = make_uint4(0u, 0u, 0u, 0u);
            if (bi >= T.blocks) continue;
            int64_t io;
            if (T.dense) {
                io = (int64_t)bi * 64;
                oo[u] = (int64_t)bi * 32;
            } else {
                const uint32_t r = fdiv(bi, T.bpr);          // row over all batches
                const uint32_t k = bi - r * T.bpr.d;
                const uint32_t b = fdiv(r, T.rows);
                const uint32_t m = r - b * T.rows.d;
                io = (int64_t)b * T.in_bs + (int64_t)m * T.in_rs + (int64_t)k * 64;
                oo[u] = (int64_t)b * T.out_bs + (int64_t)m * T.out_rs + (int64_t)k * 32;
            }
            if (T.in32) {
                ld_nc_v8(T.in + io, v[u][0], v[u][1]);
                ld_nc_v8(T.in + io + 32, v[u][2], v[u][3]);
            } else {
#pragma unroll
                for (int h = 0; h < 4; ++h) v[u][h] = ld_stream_v4(T.in + io + 16 * h);
            }
        }
#pragma unroll
        for (int u = 0; u < (int)kQBlocksPerLane; ++u) {
            if (bis[u] >= T.blocks) continue;
            const uint32_t mw = hmax_abs(hmax_abs(amax_word8(v[u][0]), amax_word8(v[u][1])),
                                         hmax_abs(amax_word8(v[u][2]), amax_word8(v[u][3]))) & 0x7fff7fffu;
            const int e = ue8m0_exponent(max(mw & 0xffffu, mw >> 16));
            const uint64_t inv2 = f32x2(exp2i(-e), exp2i(-e));   // exact power of two
            uint32_t q[8];
#pragma unroll
            for (int h = 0; h < 4; ++h) {
                // x * 2^-e two at a time (f32x2); the low BF16 widened by a
                // multiply (FMA pipe), the high one by a mask
                const uint32_t wv[4] = {v[u][h].x, v[u][h].y, v[u][h].z, v[u][h].w};
                float2 p[4];
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    uint32_t lo;
                    asm("mul.lo.u32 %0, %1, 0x10000;" : "=r"(lo) : "r"(wv[k]));
                    p[k] = f32x2_split(mul_f32x2(f32x2_bits(lo, wv[k] & 0xffff0000u), inv2));
                }
                q[2 * h] = e4m3x4(p[0].x, p[0].y, p[1].x, p[1].y);
                q[2 * h + 1] = e4m3x4(p[2].x, p[2].y, p[3].x, p[3].y);
            }
            char* dst = T.out + oo[u];
            if (T.out32) {
                st_v8(dst, make_uint4(q[0], q[1], q[2], q[3]), make_uint4(q[4], q[5], q[6], q[7]));
            } else {
#pragma unroll
                for (int h = 0; h < 4; ++h) st_v2(dst + 8 * h, make_uint2(q[2 * h], q[2 * h + 1]));
            }
            if (T.sf_mma) {
                const uint32_t r = fdiv(bis[u], T.bpr);          // row over all batches
                const uint32_t b = fdiv(r, T.rows);
                const uint32_t m = r - b * T.rows.d;
                T.e[(int64_t)b * T.sf_slab + mma_scale_offset(m, bis[u] - r * T.bpr.d, T.sf_ct)] = (uint8_t)(e + 127);
            } else {
                T.e[bis[u]] = (uint8_t)(e + 127);
            }
        }
    }
}

// Base, row and slab strides all multiples of 32 bytes (256-bit accesses).
bool aligned32(const View& v) {
    return (uintptr_t)v.ptr % 32 == 0 && v.rstride % 32 == 0 && (v.batch == 1 || v.bstride % 32 == 0);
}

cudaError_t launch_mx_quant_blocks(const Job* jobs, int n, cudaStream_t s) {
    const uint64_t kMaxSlots = uint64_t(1) << 31;   // block indices stay 32-bit
    for (int j0 = 0; j0 < n;) {
        BlockArgs a;
        a.n = 0;
        uint32_t slots = 0;
        for (; j0 + a.n < n && a.n < kMaxLaunchTensors; ++a.n) {
            const Job& j = jobs[j0 + a.n];
            const View& x = j.in;    // BF16
            const View& q = j.out;   // codes
            const uint64_t padded = ((uint64_t)(x.batch * x.rows * (x.cols / 32)) + kBSpan - 1) / kBSpan * kBSpan;
            if (a.n > 0 && slots + padded > kMaxSlots) break;
            BlockTensor& T = a.t[a.n];
            T.in = j.in.ptr;
            T.out = j.out.ptr;
            T.in_bs = j.in.bstride;
            T.in_rs = j.in.rstride;
            T.out_bs = j.out.bstride;
            T.out_rs = j.out.rstride;
            T.e = static_cast<uint8_t*>(j.scale);
            T.blocks = (uint32_t)(x.batch * x.rows * (x.cols / 32));
            T.slot_begin = slots;
            T.bpr = make_fastdiv((uint32_t)std::max<int64_t>(1, x.cols / 32));
            T.rows = make_fastdiv((uint32_t)std::max<int64_t>(1, x.rows));
            T.dense = dense_view(x, x.cols * 2) && dense_view(q, q.cols);
            T.in32 = aligned32(j.in);
            T.out32 = aligned32(j.out);
            T.sf_mma = j.scale_mma;
            T.sf_ct = (uint32_t)mma_scale_col_tiles(x.cols / 32);
            T.sf_slab = mma_scale_slab_bytes(x.rows, x.cols / 32);
            slots += (uint32_t)padded;
        }
        j0 += a.n;
        a.total_slots = slots;
        if (slots == 0) continue;
        const int grid = persistent_grid((slots + kThreads * kQBlocksPerLane - 1) / (kThreads * kQBlocksPerLane), 8);
        mxfp8_quant_block_kernel<<<grid, kThreads, 0, s>>>(a);
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}


// in = codes, out = BF16 y
bool aligned16_view(const View& v) {
    return (uintptr_t)v.ptr % 16 == 0 && v.rstride % 16 == 0 && (v.batch == 1 || v.bstride % 16 == 0);
}

cudaError_t launch_mx_dequant16(const Job* jobs, int n, cudaStream_t s) {
    const uint64_t kMaxSlots = uint64_t(1) << 31;   // chunk indices stay 32-bit
    for (int j0 = 0; j0 < n;) {
        Chunk16Args a;
        a.n = 0;
        uint32_t slots = 0;
        for (; j0 + a.n < n && a.n < kMaxLaunchTensors; ++a.n) {
            const Job& j = jobs[j0 + a.n];
            const View& x = j.out;   // the BF16 side
            const View& q = j.in;    // the code side
            const uint64_t chunks = (uint64_t)(x.batch * x.rows * (x.cols / 16));
            const uint64_t padded = (chunks + kSpan16 - 1) / kSpan16 * kSpan16;
            if (a.n > 0 && slots + padded > kMaxSlots) break;
            Chunk16Tensor& T = a.t[a.n];
            T.in = q.ptr;
            T.out = x.ptr;
            T.in_bs = q.bstride;
            T.in_rs = q.rstride;
            T.out_bs = x.bstride;
            T.out_rs = x.rstride;
            T.e = static_cast<uint8_t*>(j.scale);
            T.chunks = (uint32_t)chunks;
            T.slot_begin = slots;
            T.cpr = make_fastdiv((uint32_t)std::max<int64_t>(1, x.cols / 16));
            T.rows = make_fastdiv((uint32_t)std::max<int64_t>(1, x.rows));
            T.dense = dense_view(x, x.cols * 2) && dense_view(q, q.cols);
            T.out32 = aligned32(x);
            slots += (uint32_t)padded;
        }
        j0 += a.n;
        a.total_slots = slots;
        if (slots == 0) continue;
        const int grid = persistent_grid((slots + kThreads * kDq16Unroll - 1) / (kThreads * kDq16Unroll), 8);
        mxfp8_dequant16_kernel<<<grid, kThreads, 0, s>>>(a);
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

cudaError_t launch_mx_dequant(const Job* jobs, int n, cudaStream_t s) {
    bool all16 = true;
    for (int i = 0; i < n; ++i) all16 = all16 && aligned16_view(jobs[i].in);
    if (all16) return launch_mx_dequant16(jobs, n, s);
    const uint64_t kMaxSlots = uint64_t(1) << 31;   // chunk indices stay 32-bit
    for (int j0 = 0; j0 < n;) {
        ChunkArgs a;
        a.n = 0;
        uint32_t slots = 0;
        for (; j0 + a.n < n && a.n < kMaxLaunchTensors; ++a.n) {
            const Job& j = jobs[j0 + a.n];
            const View& xv = j.out;
            const uint64_t padded = ((uint64_t)(xv.batch * xv.rows * (xv.cols / 8)) + kSpan - 1) / kSpan * kSpan;
            if (a.n > 0 && slots + padded > kMaxSlots) break;
            ChunkTensor& T = a.t[a.n];
            const View& x = j.out;   // the BF16 side
            const View& q = j.in;    // the code side
            T.in = j.in.ptr;
            T.out = j.out.ptr;
            T.in_bs = j.in.bstride;
            T.in_rs = j.in.rstride;
            T.out_bs = j.out.bstride;
            T.out_rs = j.out.rstride;
            T.e = static_cast<uint8_t*>(j.scale);
            T.chunks = (uint32_t)(x.batch * x.rows * (x.cols / 8));
            T.slot_begin = slots;
            T.cpr = make_fastdiv((uint32_t)std::max<int64_t>(1, x.cols / 8));
            T.rows = make_fastdiv((uint32_t)std::max<int64_t>(1, x.rows));
            T.dense = dense_view(x, x.cols * 2) && dense_view(q, q.cols);
            slots += (uint32_t)padded;
        }
        j0 += a.n;
        a.total_slots = slots;
        if (slots == 0) continue;
        const int grid = persistent_grid((slots + kThreads * kUnroll - 1) / (kThreads * kUnroll), 8);
        mxfp8_dequant_kernel<<<grid, kThreads, 0, s>>>(a);
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

}  // namespace

cudaError_t launch_mxfp8_quant(const Job* jobs, int n, cudaStream_t s) { return launch_mx_quant_blocks(jobs, n, s); }

cudaError_t launch_mxfp8_dequant(const Job* jobs, int n, cudaStream_t s) { return launch_mx_dequant(jobs, n, s); }

}  // namespace pwq
