// mxfp8.cu -- MXFP8 quantise / dequantise (1x32 blocks, UE8M0 scale byte,
// E4M3 codes).  Source: "Low Precision RL", "Choose a precision" table and
// "Modes" 3 (MXFP8: 1x32 blocks, power-of-two UE8M0 scales packed as uint8,
// float8_e4m3fn weights).
//
// HBM-bound elementwise kernels: each thread owns 8-element chunks (16 B of
// BF16, one 128-bit load), four consecutive lanes form one 32-element block
// and combine their amax with two butterfly shuffles.  The scale is a power
// of two, so x * 2^-e is an exact multiply and no division is needed.
// Persistent grids (a few CTAs per SM) walk the tensor in warp-sized spans
// with U independent 128-bit loads in flight per thread.
#include "pwq_internal.h"

namespace pwq {
namespace {

constexpr int kThreads = 256;
constexpr int kUnroll = 4;

struct Rows {
    int64_t bstride, rstride;
    FastDiv per_batch;  // rows per batch matrix (M)
    __device__ __forceinline__ int64_t offset(uint32_t r) const {
        uint32_t b = fdiv(r, per_batch);
        return (int64_t)b * bstride + (int64_t)(r - b * per_batch.d) * rstride;
    }
};

struct MxQuantArgs {
    const char* x;
    char* q;
    uint8_t* e;            // dense [rows][N/32]
    Rows xr, qr;
    FastDiv cpr;           // 8-element chunks per row (N / 8)
    uint32_t total;        // chunks in this launch
    int dense;             // x and q both dense: chunk c lives at x + 16c, q + 8c
};

__global__ void __launch_bounds__(kThreads) mxfp8_quant_kernel(const MxQuantArgs a) {
    const uint32_t lane = threadIdx.x & 31u;
    const uint32_t gwarp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const uint32_t nwarps = (gridDim.x * blockDim.x) >> 5;
    for (uint32_t base = gwarp * 32u * kUnroll; base < a.total; base += nwarps * 32u * kUnroll) {
        uint4 v[kUnroll];
        int64_t xo[kUnroll], qo[kUnroll];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const uint32_t c = base + u * 32u + lane;
            if (a.dense) {
                xo[u] = (int64_t)c * 16;
                qo[u] = (int64_t)c * 8;
            } else {
                const uint32_t r = fdiv(c, a.cpr);
                const uint32_t k = c - r * a.cpr.d;
                xo[u] = a.xr.offset(r) + (int64_t)k * 16;
                qo[u] = a.qr.offset(r) + (int64_t)k * 8;
            }
            v[u] = make_uint4(0u, 0u, 0u, 0u);
            if (c < a.total) v[u] = ld_stream_v4(a.x + xo[u]);
        }
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const uint32_t c = base + u * 32u + lane;
            uint32_t m = amax_bits8(v[u]);
            m = max(m, __shfl_xor_sync(0xffffffffu, m, 1));
            m = max(m, __shfl_xor_sync(0xffffffffu, m, 2));
            const int e = ue8m0_exponent(m);
            const float inv = exp2i(-e);  // exact power of two
            uint2 out;
            out.x = e4m3x4(__fmul_rn(bf16_lo(v[u].x), inv), __fmul_rn(bf16_hi(v[u].x), inv),
                           __fmul_rn(bf16_lo(v[u].y), inv), __fmul_rn(bf16_hi(v[u].y), inv));
            out.y = e4m3x4(__fmul_rn(bf16_lo(v[u].z), inv), __fmul_rn(bf16_hi(v[u].z), inv),
                           __fmul_rn(bf16_lo(v[u].w), inv), __fmul_rn(bf16_hi(v[u].w), inv));
            if (c < a.total) {
                st_v2(a.q + qo[u], out);
                if ((lane & 3u) == 0u) a.e[c >> 2] = (uint8_t)(e + 127);
            }
        }
    }
}

struct MxDequantArgs {
    const char* q;
    char* y;
    const uint8_t* e;      // dense [rows][N/32]
    Rows qr, yr;
    FastDiv cpr;
    uint32_t total;
    int dense;
};

__global__ void __launch_bounds__(kThreads) mxfp8_dequant_kernel(const MxDequantArgs a) {
    const uint32_t stride = gridDim.x * blockDim.x;
    uint32_t c0 = blockIdx.x * blockDim.x + threadIdx.x;
    for (uint32_t base = c0; base < a.total; base += stride * kUnroll) {
        uint2 v[kUnroll];
        uint32_t eb[kUnroll];
        int64_t yo[kUnroll];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const uint32_t c = base + u * stride;
            int64_t qo;
            if (a.dense) {
                qo = (int64_t)c * 8;
                yo[u] = (int64_t)c * 16;
            } else {
                const uint32_t r = fdiv(c, a.cpr);
                const uint32_t k = c - r * a.cpr.d;
                qo = a.qr.offset(r) + (int64_t)k * 8;
                yo[u] = a.yr.offset(r) + (int64_t)k * 16;
            }
            v[u] = make_uint2(0u, 0u);
            eb[u] = 127u;
            if (c < a.total) {
                v[u] = ld_stream_v2(a.q + qo);
                eb[u] = __ldg(a.e + (c >> 2));
            }
        }
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const uint32_t c = base + u * stride;
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
            if (c < a.total) st_v4(a.y + yo[u], out);
        }
    }
}

bool dense_view(const View& v, int64_t elem_bytes_per_row) {
    return v.rstride == elem_bytes_per_row && (v.batch == 1 || v.bstride == v.rows * v.rstride);
}

// Splits a launch over whole batch matrices so that each launch has fewer
// than 2^31 chunks (chunk indices stay 32-bit).
template <class F>
cudaError_t for_batch_ranges(int64_t batch, int64_t chunks_per_batch, F&& f) {
    const int64_t cap = (int64_t(1) << 31) - 1;
    const int64_t per = chunks_per_batch > 0 ? std::max<int64_t>(1, cap / chunks_per_batch) : batch;
    for (int64_t b0 = 0; b0 < batch; b0 += per) {
        cudaError_t err = f(b0, std::min(batch, b0 + per));
        if (err != cudaSuccess) return err;
    }
    return cudaSuccess;
}

}  // namespace

cudaError_t launch_mxfp8_quant(const View& x, const View& q, uint8_t* scale, cudaStream_t s) {
    const int64_t cpr = x.cols / 8;
    const bool dense = dense_view(x, x.cols * 2) && dense_view(q, q.cols);
    return for_batch_ranges(x.batch, x.rows * cpr, [&](int64_t b0, int64_t b1) {
        MxQuantArgs a;
        a.x = x.ptr + b0 * x.bstride;
        a.q = q.ptr + b0 * q.bstride;
        a.e = scale + b0 * x.rows * (x.cols / 32);
        a.xr = Rows{x.bstride, x.rstride, make_fastdiv((uint32_t)x.rows)};
        a.qr = Rows{q.bstride, q.rstride, make_fastdiv((uint32_t)x.rows)};
        a.cpr = make_fastdiv((uint32_t)cpr);
        a.total = (uint32_t)((b1 - b0) * x.rows * cpr);
        a.dense = dense;
        const int64_t span = int64_t(kThreads) * kUnroll;
        const int grid = persistent_grid((a.total + span - 1) / span, 8);
        mxfp8_quant_kernel<<<grid, kThreads, 0, s>>>(a);
        return cudaGetLastError();
    });
}

cudaError_t launch_mxfp8_dequant(const View& q, const uint8_t* scale, const View& y, cudaStream_t s) {
    const int64_t cpr = q.cols / 8;
    const bool dense = dense_view(q, q.cols) && dense_view(y, y.cols * 2);
    return for_batch_ranges(q.batch, q.rows * cpr, [&](int64_t b0, int64_t b1) {
        MxDequantArgs a;
        a.q = q.ptr + b0 * q.bstride;
        a.y = y.ptr + b0 * y.bstride;
        a.e = scale + b0 * q.rows * (q.cols / 32);
        a.qr = Rows{q.bstride, q.rstride, make_fastdiv((uint32_t)q.rows)};
        a.yr = Rows{y.bstride, y.rstride, make_fastdiv((uint32_t)q.rows)};
        a.cpr = make_fastdiv((uint32_t)cpr);
        a.total = (uint32_t)((b1 - b0) * q.rows * cpr);
        a.dense = dense;
        const int64_t span = int64_t(kThreads) * kUnroll;
        const int grid = persistent_grid((a.total + span - 1) / span, 8);
        mxfp8_dequant_kernel<<<grid, kThreads, 0, s>>>(a);
        return cudaGetLastError();
    });
}

}  // namespace pwq
