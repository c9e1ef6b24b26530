// mxfp8.cu -- MXFP8 quantise / dequantise (1x32 blocks, UE8M0 scale byte,
// E4M3 codes).  Source: "Low Precision RL", "Choose a precision" table and
// "Modes" 3 (MXFP8: 1x32 blocks, power-of-two UE8M0 scales packed as uint8,
// float8_e4m3fn weights).
//
// HBM-bound elementwise kernels over a list of up to kMaxLaunchTensors
// tensors per launch.  Each thread owns 8-element chunks (16 B of BF16, one
// 128-bit load); four consecutive lanes form one 32-element block and
// combine their amax with two butterfly shuffles.  The scale is a power of
// two, so x * 2^-e is an exact multiply and no division is needed.  A
// persistent grid walks the concatenated chunk ranges in warp-sized spans of
// kUnroll * 32 chunks (kUnroll independent 128-bit loads in flight per
// thread); every tensor's range is padded to a whole number of spans so a
// span never straddles two tensors.
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

__global__ void __launch_bounds__(kThreads) mxfp8_quant_kernel(const __grid_constant__ ChunkArgs a) {
    const uint32_t lane = threadIdx.x & 31u;
    const uint32_t gwarp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const uint32_t nwarps = (gridDim.x * blockDim.x) >> 5;
    for (uint32_t slot = gwarp * kSpan; slot < a.total_slots; slot += nwarps * kSpan) {
        const ChunkTensor& T = a.t[span_tensor(a, slot)];
        const uint32_t base = slot - T.slot_begin;
        uint4 v[kUnroll];
        int64_t qo[kUnroll];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const uint32_t c = base + u * 32u + lane;
            int64_t xo;
            chunk_offsets(T, c, 16, 8, xo, qo[u]);
            v[u] = make_uint4(0u, 0u, 0u, 0u);
            if (c < T.chunks) v[u] = ld_stream_v4(T.in + xo);
        }
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const uint32_t c = base + u * 32u + lane;
            uint32_t m = amax_bits8_int(v[u]);
            m = max(m, __shfl_xor_sync(0xffffffffu, m, 1));
            m = max(m, __shfl_xor_sync(0xffffffffu, m, 2));
            const int e = ue8m0_exponent(m);
            const float inv = exp2i(-e);  // exact power of two
            uint2 out;
            // x * 2^-e two at a time (f32x2); the low BF16 widened by a
            // multiply (FMA pipe), the high one by a mask
            const uint64_t inv2 = f32x2(inv, inv);
            const uint32_t wv[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
            float2 p[4];
#pragma unroll
            for (int h = 0; h < 4; ++h) {
                uint32_t lo;
                asm("mul.lo.u32 %0, %1, 0x10000;" : "=r"(lo) : "r"(wv[h]));
                p[h] = f32x2_split(mul_f32x2(f32x2_bits(lo, wv[h] & 0xffff0000u), inv2));
            }
            out.x = e4m3x4(p[0].x, p[0].y, p[1].x, p[1].y);
            out.y = e4m3x4(p[2].x, p[2].y, p[3].x, p[3].y);
            if (c < T.chunks) {
                st_v2(T.out + qo[u], out);
                if ((lane & 3u) == 0u) T.e[c >> 2] = (uint8_t)(e + 127);
            }
        }
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

bool dense_view(const View& v, int64_t row_bytes) {
    return v.rstride == row_bytes && (v.batch == 1 || v.bstride == v.rows * v.rstride);
}

// quant: in = BF16 x, out = codes; dequant: in = codes, out = BF16 y
template <bool kQuant>
cudaError_t launch_mx(const Job* jobs, int n, cudaStream_t s) {
    const uint64_t kMaxSlots = uint64_t(1) << 31;   // chunk indices stay 32-bit
    for (int j0 = 0; j0 < n;) {
        ChunkArgs a;
        a.n = 0;
        uint32_t slots = 0;
        for (; j0 + a.n < n && a.n < kMaxLaunchTensors; ++a.n) {
            const Job& j = jobs[j0 + a.n];
            const View& xv = kQuant ? j.in : j.out;
            const uint64_t padded = ((uint64_t)(xv.batch * xv.rows * (xv.cols / 8)) + kSpan - 1) / kSpan * kSpan;
            if (a.n > 0 && slots + padded > kMaxSlots) break;
            ChunkTensor& T = a.t[a.n];
            const View& x = kQuant ? j.in : j.out;   // the BF16 side
            const View& q = kQuant ? j.out : j.in;   // the code side
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
        if (kQuant)
            mxfp8_quant_kernel<<<grid, kThreads, 0, s>>>(a);
        else
            mxfp8_dequant_kernel<<<grid, kThreads, 0, s>>>(a);
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

}  // namespace

cudaError_t launch_mxfp8_quant(const Job* jobs, int n, cudaStream_t s) { return launch_mx<true>(jobs, n, s); }

cudaError_t launch_mxfp8_dequant(const Job* jobs, int n, cudaStream_t s) { return launch_mx<false>(jobs, n, s); }

}  // namespace pwq
