// selftest.cu -- exhaustive checks of the device arithmetic the kernels use.
//
// Division: the quantisers replace the per-element IEEE division by one
// correctly rounded reciprocal per tile/block and an FMA residual correction
// (pwq_device.cuh).  The numerators are BF16 values and the divisors come
// from small finite sets (FP8 block-wise: fl(a / 448); NVFP4:
// fl(dec(sb) * fl(a / 2688)) and fl(6 * fl(a / 2688)); the 4over6 variant
// adds fl(a / 1536) for the global scale and 4 for the block-scale
// multiplier; a a positive BF16, sb a non-zero E4M3 code), so
// every (numerator, divisor) pair can be enumerated and compared with CUDA's
// IEEE division __fdiv_rn in well under a second.
//
// Codecs: writes the hardware conversions of a range of binary32 inputs so
// the host can compare them with the CPU oracle.
//
// Rewrites: the BF16 magnitude max by the bf16x2 abs-max instruction and
// the NVFP4 dequantisation through an exact binary16 product are compared
// with their plain forms over every input they can see.
#include "pwq_internal.h"

namespace pwq {
namespace {

constexpr int kThreads = 256;

__device__ __forceinline__ bool bf16_is_finite(uint32_t b) { return ((b >> 7) & 0xffu) != 0xffu; }

// One divisor per CTA; every finite BF16 numerator the format can pair with
// it:
//   kKind 0  FP8 block-wise code divisor s = fl(a / 448), |x| <= a (x is in
//            the tile whose amax is a);
//   kKind 1  NVFP4 code divisor d = fl(dec(sb) * fl(a / kDen)), |x| <= 16 d
//            (x / d stays below 6 / (1 - 2^-4) for an E4M3-normal block
//            scale and below 9.1 for a subnormal one; the 4over6 candidate
//            of 4 stays lower);
//   kKind 2  NVFP4 block-scale divisor fl(kMul * fl(a / kDen)), |x| <= a
//            (the block amax never exceeds the group amax a).
// kDen = 6 E: 2688 for NVFP4, 1536 for 4over6 with E = 256; kMul = 6, or 4
// for the 4over6 candidate.  The kernels' path (reciprocal or IEEE, chosen
// by the divisor) is compared with __fdiv_rn: codes for every pair, binary32
// quotients where |x| >= 2^-100 and the IEEE quotient is normal.
template <int kKind, int kDen = 2688, int kMul = 6>
__global__ void __launch_bounds__(kThreads) selftest_division_kernel(unsigned long long* counts) {
    const uint32_t a = blockIdx.x + 1u;                // positive finite BF16 0x0001..0x7f7f
    const float av = __uint_as_float(a << 16);
    float d, xmax;
    if (kKind == 0) {
        d = __fdiv_rn(av, 448.0f);
        xmax = av;
    } else if (kKind == 1) {
        const uint32_t sb = blockIdx.y + 1u;           // E4M3 0x01..0x7e
        d = __fmul_rn(e4m3_decode(sb), __fdiv_rn(av, (float)kDen));
        xmax = __fmul_rn(16.0f, d);
    } else {
        d = __fmul_rn((float)kMul, __fdiv_rn(av, (float)kDen));
        xmax = av;
    }
    const float r = __frcp_rn(d);
    const bool fast = div_fast_ok(d);
    unsigned long long n = 0, code_bad = 0, quot_bad = 0, slow = 0;
    // numerators in BF16 pairs, through the same functions the kernels call:
    // the packed pair path for code divisors, the scalar one for fl(6 gs)
    for (uint32_t wi = threadIdx.x; wi < 32768u; wi += kThreads) {
        const uint32_t w = (2u * wi) | ((2u * wi + 1u) << 16);
        float2 qp;
        if (kKind == 2) {
            qp.x = fast ? quotient<true>(bf16_lo(w), d, r) : quotient<false>(bf16_lo(w), d, r);
            qp.y = fast ? quotient<true>(bf16_hi(w), d, r) : quotient<false>(bf16_hi(w), d, r);
        } else {
            qp = fast ? quotient_bf16x2<true>(w, d, r) : quotient_bf16x2<false>(w, d, r);
        }
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const uint32_t xb = 2u * wi + (uint32_t)h;
            if (!bf16_is_finite(xb)) continue;
            const float x = __uint_as_float(xb << 16);
            if (!(fabsf(x) <= xmax)) continue;
            const float qf = h ? qp.y : qp.x;
            const float qr = (d == 0.0f) ? __uint_as_float((xb << 16) & 0x80000000u) : __fdiv_rn(x, d);
            ++n;
            slow += !fast;
            if (kKind == 1)
                code_bad += (e2m1x2(qf, 0.0f) & 0xfu) != (e2m1x2(qr, 0.0f) & 0xfu);
            else
                code_bad += (e4m3x2(qf, 0.0f) & 0xffu) != (e4m3x2(qr, 0.0f) & 0xffu);
            const uint32_t ef = (__float_as_uint(qr) >> 23) & 0xffu;
            if (ef != 0u && fabsf(x) >= 0x1p-100f) quot_bad += __float_as_uint(qf) != __float_as_uint(qr);
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        n += __shfl_xor_sync(0xffffffffu, n, o);
        code_bad += __shfl_xor_sync(0xffffffffu, code_bad, o);
        quot_bad += __shfl_xor_sync(0xffffffffu, quot_bad, o);
        slow += __shfl_xor_sync(0xffffffffu, slow, o);
    }
    if ((threadIdx.x & 31u) == 0u) {
        atomicAdd(counts + 0, n);
        atomicAdd(counts + 1, code_bad);
        atomicAdd(counts + 2, quot_bad);
        atomicAdd(counts + 3, slow);
    }
}

// FP8 tile scale: fp8_tile_scale(a) against fl(a / 448) for every finite
// non-negative BF16 a.
__global__ void __launch_bounds__(kThreads) selftest_tile_scale_kernel(unsigned long long* counts) {
    unsigned long long n = 0, bad = 0, slow = 0;
    for (uint32_t ab = blockIdx.x * blockDim.x + threadIdx.x; ab < 0x7f80u; ab += gridDim.x * blockDim.x) {
        const float a = __uint_as_float(ab << 16);
        ++n;
        bad += __float_as_uint(fp8_tile_scale(a)) != __float_as_uint(__fdiv_rn(a, 448.0f));
        slow += !(a >= 0x1p-100f);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        n += __shfl_xor_sync(0xffffffffu, n, o);
        bad += __shfl_xor_sync(0xffffffffu, bad, o);
        slow += __shfl_xor_sync(0xffffffffu, slow, o);
    }
    if ((threadIdx.x & 31u) == 0u) {
        atomicAdd(counts + 0, n);
        atomicAdd(counts + 1, bad);
        atomicAdd(counts + 2, bad);
        atomicAdd(counts + 3, slow);
    }
}

// BF16 magnitude max: hmax_abs against the integer max of the magnitude
// bits, for every ordered pair (a, b) of finite BF16 values, in both halves
// of the word (a low in one operand, high in the other).  One CTA per a.
__global__ void __launch_bounds__(kThreads) selftest_absmax_kernel(unsigned long long* counts) {
    const uint32_t a = blockIdx.x;
    unsigned long long n = 0, bad = 0;
    if (bf16_is_finite(a)) {
        for (uint32_t b = threadIdx.x; b < 0x10000u; b += blockDim.x) {
            if (!bf16_is_finite(b)) continue;
            const uint32_t want = max(a & 0x7fffu, b & 0x7fffu);
            const uint32_t got = hmax_abs(a | (b << 16), b | (a << 16)) & 0x7fff7fffu;
            ++n;
            bad += (got & 0xffffu) != want || (got >> 16) != want;
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        n += __shfl_xor_sync(0xffffffffu, n, o);
        bad += __shfl_xor_sync(0xffffffffu, bad, o);
    }
    if ((threadIdx.x & 31u) == 0u && n != 0) {
        atomicAdd(counts + 0, n);
        atomicAdd(counts + 1, bad);
    }
}

// NVFP4 dequantisation, binary16-product form (dequant_half_h) against the
// binary32 form (dequant_half): every byte of two E2M1 codes, every block
// scale code 0..126, every global scale gs = fl(a / 2688) with a = 0 or a
// positive finite BF16 (one CTA per a).  Counts code pairs.
__global__ void __launch_bounds__(kThreads) selftest_fp4_dequant_kernel(unsigned long long* counts) {
    const float gs = __fdiv_rn(__uint_as_float(blockIdx.x << 16), 2688.0f);
    const uint64_t gs2 = f32x2(gs, gs);
    unsigned long long n = 0, bad = 0;
    for (uint32_t i = threadIdx.x; i < 127u * 64u; i += blockDim.x) {
        const uint32_t sb = i >> 6, w = (i & 63u) * 4u;
        const uint32_t codes = w | ((w + 1u) << 8) | ((w + 2u) << 16) | ((w + 3u) << 24);
        const uint4 want = dequant_half(codes, e4m3_decode(sb), gs);
        const uint4 got = dequant_half_h(codes, e4m3x2_f16x2(sb * 0x101u), gs2);
        n += 4;
        bad += (got.x != want.x) + (got.y != want.y) + (got.z != want.z) + (got.w != want.w);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        n += __shfl_xor_sync(0xffffffffu, n, o);
        bad += __shfl_xor_sync(0xffffffffu, bad, o);
    }
    if ((threadIdx.x & 31u) == 0u) {
        atomicAdd(counts + 0, n);
        atomicAdd(counts + 1, bad);
    }
}

__global__ void __launch_bounds__(kThreads)
selftest_codecs_kernel(uint32_t first, uint32_t count, uint8_t* e4m3, uint8_t* e2m1, uint16_t* bf16) {
    const uint32_t stride = gridDim.x * blockDim.x;
    for (uint32_t i = blockIdx.x * blockDim.x + threadIdx.x; i < count; i += stride) {
        const float f = __uint_as_float(first + i);
        if (e4m3) e4m3[i] = (uint8_t)(e4m3x2(f, 0.0f) & 0xffu);
        if (e2m1) e2m1[i] = (uint8_t)(e2m1x2(f, 0.0f) & 0xfu);
        if (bf16) bf16[i] = (uint16_t)(pack_bf16x2(f, 0.0f) & 0xffffu);
    }
}

}  // namespace

cudaError_t launch_selftest_division(int which, unsigned long long* counts, cudaStream_t s) {
    cudaError_t e = cudaMemsetAsync(counts, 0, 4 * sizeof(unsigned long long), s);
    if (e != cudaSuccess) return e;
    if (which == 0)
        selftest_division_kernel<0><<<dim3(0x7f7f), kThreads, 0, s>>>(counts);
    else if (which == 1)
        selftest_division_kernel<1><<<dim3(0x7f7f, 0x7e), kThreads, 0, s>>>(counts);
    else if (which == 2)
        selftest_division_kernel<2><<<dim3(0x7f7f), kThreads, 0, s>>>(counts);
    else if (which == 3)
        selftest_tile_scale_kernel<<<dim3(64), kThreads, 0, s>>>(counts);
    else if (which == 4)
        selftest_absmax_kernel<<<dim3(0x10000), kThreads, 0, s>>>(counts);
    else if (which == 5)
        selftest_fp4_dequant_kernel<<<dim3(0x7f80), kThreads, 0, s>>>(counts);
    else if (which == 6)
        selftest_division_kernel<1, 1536><<<dim3(0x7f7f, 0x7e), kThreads, 0, s>>>(counts);
    else if (which == 7)
        selftest_division_kernel<2, 1536, 6><<<dim3(0x7f7f), kThreads, 0, s>>>(counts);
    else if (which == 8)
        selftest_division_kernel<2, 1536, 4><<<dim3(0x7f7f), kThreads, 0, s>>>(counts);
    else
        selftest_division_kernel<2, 2688, 4><<<dim3(0x7f7f), kThreads, 0, s>>>(counts);
    return cudaGetLastError();
}

cudaError_t launch_selftest_codecs(uint32_t first, uint32_t count, uint8_t* e4m3, uint8_t* e2m1,
                                   uint16_t* bf16, cudaStream_t s) {
    if (count == 0) return cudaSuccess;
    const int grid = persistent_grid((count + kThreads - 1) / kThreads, 8);
    selftest_codecs_kernel<<<grid, kThreads, 0, s>>>(first, count, e4m3, e2m1, bf16);
    return cudaGetLastError();
}

}  // namespace pwq
