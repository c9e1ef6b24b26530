// observer.cu -- W4A4 activation observers: the running extremes of an
// activation tensor and its NVFP4 global scale (input_global_scale).
// Source: verl NVFP4 QAT article, 2.2 and 3.1 (W4A4 mode keeps an
// input_global_scale buffer filled by an activation observer:
// static_minmax by default, memoryless_minmax or minmax).  The pages name
// the observers only; the readings implemented here:
//   state (lo, hi) = binary32 minimum and maximum of the observed values,
//     empty = (+inf, -inf); values are ordered numerically with -0 < +0;
//   memoryless_minmax: (lo, hi) = (min x, max x) of this tensor;
//   static_minmax:     (lo, hi) = (min(lo, min x), max(hi, max x));
//   minmax:            moving average with constant c: an empty state takes
//                      (min x, max x), otherwise
//                      lo = fl(fl(fl(1 - c) * lo) + fl(c * min x)), hi alike;
//   A = max(|lo|, |hi|), input_global_scale = fl(A / 2688).
//
// Two launches after a memset of two words: a grid-stride reduction of the
// tensor's extremes as order-preserving 16-bit keys of the BF16 values
// (integer min / max, 16-byte loads), published with two atomicMax (the
// minimum as the complement of its key), then one thread applies the
// observer rule and writes the state and the scales.
#include <algorithm>

#include "pwq_internal.h"

namespace pwq {
namespace {

constexpr int kThreads = 256;
constexpr int kUnroll = 4;

// Two BF16 values -> two 16-bit keys in the order of the values (-0 < +0):
// a negative value maps to its complement, a non-negative one gets bit 15.
__device__ __forceinline__ uint32_t bf16x2_keys(uint32_t w) {
    const uint32_t neg = (w >> 15) & 0x00010001u;   // 1 in each half whose sign is set
    return w ^ (0x80008000u | (neg * 0x7fffu));
}

__device__ __forceinline__ uint32_t key_to_bf16(uint32_t k) {
    return (k & 0x8000u) ? (k & 0x7fffu) : ((~k) & 0xffffu);
}

struct ObsArgs {
    const char* x;
    int64_t bs, rs;        // bytes
    uint32_t chunks;       // B * M * N / 8
    FastDiv cpr, rows;     // chunks per row, M
    int dense;
    uint32_t* words;       // [0] = max of ~min key, [1] = max key
};

__global__ void __launch_bounds__(kThreads) observe_reduce_kernel(const __grid_constant__ ObsArgs a) {
    __shared__ uint32_t red[2][kThreads / 32];
    const uint32_t stride = gridDim.x * blockDim.x;
    uint32_t kmin = 0xffffffffu, kmax = 0u;   // two 16-bit lanes each
    for (uint32_t c0 = blockIdx.x * blockDim.x + threadIdx.x; c0 < a.chunks; c0 += stride * kUnroll) {
        uint4 v[kUnroll];
        bool ok[kUnroll];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const uint32_t c = c0 + u * stride;
            ok[u] = c < a.chunks;
            v[u] = make_uint4(0u, 0u, 0u, 0u);
            if (ok[u]) {
                int64_t off;
                if (a.dense) {
                    off = (int64_t)c * 16;
                } else {
                    const uint32_t R = fdiv(c, a.cpr);
                    const uint32_t k = c - R * a.cpr.d;
                    const uint32_t b = fdiv(R, a.rows);
                    off = (int64_t)b * a.bs + (int64_t)(R - b * a.rows.d) * a.rs + (int64_t)k * 16;
                }
                v[u] = ld_stream_v4(a.x + off);
            }
        }
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            if (!ok[u]) continue;
            const uint32_t k0 = bf16x2_keys(v[u].x), k1 = bf16x2_keys(v[u].y);
            const uint32_t k2 = bf16x2_keys(v[u].z), k3 = bf16x2_keys(v[u].w);
            kmin = __vminu2(kmin, __vminu2(__vminu2(k0, k1), __vminu2(k2, k3)));
            kmax = __vmaxu2(kmax, __vmaxu2(__vmaxu2(k0, k1), __vmaxu2(k2, k3)));
        }
    }
    uint32_t nmin = (~min(kmin & 0xffffu, kmin >> 16)) & 0xffffu;   // complement: larger = smaller value
    uint32_t mx = max(kmax & 0xffffu, kmax >> 16);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        nmin = max(nmin, __shfl_xor_sync(0xffffffffu, nmin, o));
        mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    }
    if ((threadIdx.x & 31u) == 0u) {
        red[0][threadIdx.x >> 5] = nmin;
        red[1][threadIdx.x >> 5] = mx;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        for (int w = 1; w < kThreads / 32; ++w) {
            nmin = max(nmin, red[0][w]);
            mx = max(mx, red[1][w]);
        }
        atomicMax(a.words, nmin);
        atomicMax(a.words + 1, mx);
    }
}

__device__ __forceinline__ float min_signed(float a, float b) {   // -0 < +0
    if (a == b) return signbit(a) ? a : b;
    return a < b ? a : b;
}
__device__ __forceinline__ float max_signed(float a, float b) {
    if (a == b) return signbit(a) ? b : a;
    return a > b ? a : b;
}

__global__ void observe_finish_kernel(const uint32_t* words, int kind, float c, float* state, float* amax_out,
                                      float* gs_out) {
    const float mn = __uint_as_float(key_to_bf16((~words[0]) & 0xffffu) << 16);
    const float mx = __uint_as_float(key_to_bf16(words[1]) << 16);
    float lo = state[0], hi = state[1];
    const bool empty = lo > hi;
    if (kind == 0 || (kind == 2 && empty)) {
        lo = mn;
        hi = mx;
    } else if (kind == 1) {
        lo = min_signed(lo, mn);
        hi = max_signed(hi, mx);
    } else {
        const float w = __fsub_rn(1.0f, c);
        lo = __fadd_rn(__fmul_rn(w, lo), __fmul_rn(c, mn));
        hi = __fadd_rn(__fmul_rn(w, hi), __fmul_rn(c, mx));
    }
    state[0] = lo;
    state[1] = hi;
    const float A = fmaxf(fabsf(lo), fabsf(hi));
    if (amax_out) *amax_out = A;
    if (gs_out) *gs_out = __fdiv_rn(A, 2688.0f);
}

}  // namespace

cudaError_t launch_activation_observe(const View& x, int kind, float c, float* state, float* amax_out,
                                      float* gs_out, uint32_t* words, cudaStream_t s) {
    cudaError_t e = cudaMemsetAsync(words, 0, 2 * sizeof(uint32_t), s);
    if (e != cudaSuccess) return e;
    ObsArgs a;
    a.x = x.ptr;
    a.bs = x.bstride;
    a.rs = x.rstride;
    a.chunks = (uint32_t)(x.batch * x.rows * (x.cols / 8));
    a.cpr = make_fastdiv((uint32_t)std::max<int64_t>(1, x.cols / 8));
    a.rows = make_fastdiv((uint32_t)std::max<int64_t>(1, x.rows));
    a.dense = x.rstride == x.cols * 2 && (x.batch == 1 || x.bstride == x.rows * x.rstride);
    a.words = words;
    const int grid = persistent_grid((a.chunks + kThreads * kUnroll - 1) / (kThreads * kUnroll), 4);
    observe_reduce_kernel<<<grid, kThreads, 0, s>>>(a);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    observe_finish_kernel<<<1, 1, 0, s>>>(words, kind, c, state, amax_out, gs_out);
    return cudaGetLastError();
}

}  // namespace pwq
