// pwq_device.cuh -- device helpers shared by the libpwq kernels (sm_100a).
//
// Conversions use the sm_100a hardware converters:
//   cvt.rn.satfinite.e4m3x2.f32   binary32 pair -> two E4M3 bytes (RNE, saturating)
//   cvt.rn.satfinite.e2m1x2.f32   binary32 pair -> two E2M1 nibbles (RNE, saturating)
//   cvt.rn.f16x2.e4m3x2 / .e2m1x2 exact decode to binary16
//   cvt.rn.bf16x2.f32             binary32 pair -> BF16 pair (RNE, subnormals kept)
// Their rounding, saturation and sign-of-zero behaviour is checked against
// the CPU oracle over whole input ranges by the codec self-test.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

namespace pwq {

// ---------------------------------------------------------------- BF16 lanes

// Low / high BF16 of a packed 32-bit word, widened exactly to binary32.
__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// Per half of two BF16 pairs: the larger magnitude, exactly (finite values,
// subnormals kept), with the sign bit set to the XOR of the inputs' signs.
// One instruction per pair instead of a mask and an integer max; callers
// clear the sign bits once at the end.  pwq_selftest_division(4) checks it
// against the integer magnitude max for every pair of finite BF16 values.
__device__ __forceinline__ uint32_t hmax_abs(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("max.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}
// Per half: the largest magnitude of the four BF16 values of that half of
// a 16-byte chunk (sign bits not meaningful).
__device__ __forceinline__ uint32_t amax_word8(uint4 v) {
    return hmax_abs(hmax_abs(v.x, v.y), hmax_abs(v.z, v.w));
}

// Max of |x| over the 8 BF16 values of a 16-byte chunk, as BF16 magnitude
// bits (for finite values the magnitude order is the unsigned order of the
// low 15 bits).
__device__ __forceinline__ uint32_t amax_bits8(uint4 v) {
    const uint32_t c = amax_word8(v) & 0x7fff7fffu;
    return max(c & 0xffffu, c >> 16);
}

// Pack two binary32 into a BF16x2 word (lo in bits 0..15), RNE.
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

// ---------------------------------------------------------------- E4M3

// Two binary32 -> two E4M3 codes in a 16-bit value (lo in bits 0..7).
__device__ __forceinline__ uint32_t e4m3x2(float lo, float hi) {
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
    return r;
}

// Four binary32 -> four E4M3 codes in a 32-bit word (element 0 in byte 0).
__device__ __forceinline__ uint32_t e4m3x4(float a, float b, float c, float d) {
    uint32_t r;
    asm("{\n\t.reg .b16 lo, hi;\n\t"
        "cvt.rn.satfinite.e4m3x2.f32 lo, %2, %1;\n\t"
        "cvt.rn.satfinite.e4m3x2.f32 hi, %4, %3;\n\t"
        "mov.b32 %0, {lo, hi};\n\t}"
        : "=r"(r) : "f"(a), "f"(b), "f"(c), "f"(d));
    return r;
}

// Two E4M3 codes (lo in bits 0..7) -> exact binary32 values.
__device__ __forceinline__ float2 e4m3x2_decode(uint32_t codes16) {
    uint32_t h2;
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"((uint16_t)codes16));
    float2 f;
    asm("cvt.f32.f16 %0, %1;" : "=f"(f.x) : "h"((unsigned short)(h2 & 0xffffu)));
    asm("cvt.f32.f16 %0, %1;" : "=f"(f.y) : "h"((unsigned short)(h2 >> 16)));
    return f;
}

// One E4M3 code -> exact binary32 value.
__device__ __forceinline__ float e4m3_decode(uint32_t code) { return e4m3x2_decode(code & 0xffu).x; }

// Largest magnitude byte (bits 0..6) among E4M3 codes; positive E4M3 codes
// order like their values.  A per-byte SIMD max has no single instruction
// on this target (it is emulated with several), so the bytes are compared
// as the high bytes of 16-bit lanes: the masked words themselves (bytes 1
// and 3 high) and the words shifted up by 8 (bytes 0 and 2 high).  The lane
// form accumulates over chunks with __vmaxu2; e4m3_maxmag_fin reads the
// maximum out once.
__device__ __forceinline__ uint32_t e4m3_maxmag_lanes(uint2 c) {
    const uint32_t a = c.x & 0x7f7f7f7fu, b = c.y & 0x7f7f7f7fu;
    return __vmaxu2(__vmaxu2(a, b), __vmaxu2(a << 8, b << 8));
}
__device__ __forceinline__ uint32_t e4m3_maxmag_fin(uint32_t lanes) {
    return max(lanes >> 24, (lanes >> 8) & 0xffu);
}
__device__ __forceinline__ uint32_t e4m3_maxmag8(uint2 c) { return e4m3_maxmag_fin(e4m3_maxmag_lanes(c)); }

// BF16 magnitude bits of max |y| over FP8 codes of one scale s whose largest
// magnitude byte is mc: rounding is monotone and symmetric in sign, so the
// max of bf16(fl(dec(q) * s)) in magnitude is bf16(fl(dec(mc) * |s|)).
__device__ __forceinline__ uint32_t fp8_amax_bits16(uint32_t mc, float s) {
    return pack_bf16x2(__fmul_rn(e4m3_decode(mc), fabsf(s)), 0.0f) & 0xffffu;
}

// ---------------------------------------------------------------- E2M1

// Two binary32 -> one byte of two E2M1 codes (lo element in bits 0..3).
__device__ __forceinline__ uint32_t e2m1x2(float lo, float hi) {
    uint32_t r;
    asm("{\n\t.reg .b8 t;\n\tcvt.rn.satfinite.e2m1x2.f32 t, %1, %2;\n\tcvt.u32.u8 %0, t;\n\t}"
        : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

// Eight binary32 -> eight E2M1 codes in a 32-bit word (element 0 in bits
// 0..3, element 2j in the low nibble of byte j).
__device__ __forceinline__ uint32_t e2m1x8(const float (&q)[8]) {
    uint32_t r;
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
        "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
        : "=r"(r)
        : "f"(q[0]), "f"(q[1]), "f"(q[2]), "f"(q[3]), "f"(q[4]), "f"(q[5]), "f"(q[6]), "f"(q[7]));
    return r;
}

// Byte of two E2M1 codes -> two exact binary32 values (lo nibble first).
__device__ __forceinline__ float2 e2m1x2_decode(uint32_t byte) {
    uint32_t h2;
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\tmov.b32 {b0, b1, b2, b3}, %1;\n\t"
        "cvt.rn.f16x2.e2m1x2 %0, b0;\n\t}" : "=r"(h2) : "r"(byte));
    float2 f;
    asm("cvt.f32.f16 %0, %1;" : "=f"(f.x) : "h"((unsigned short)(h2 & 0xffffu)));
    asm("cvt.f32.f16 %0, %1;" : "=f"(f.y) : "h"((unsigned short)(h2 >> 16)));
    return f;
}

// ---------------------------------------------------------------- division

// Quotient x / s for a positive block divisor s, from the correctly rounded
// reciprocal r = RN(1/s): one product and one residual correction with
// fused multiply-adds (Markstein's correction step; P. Markstein,
// "Computation of elementary functions on the IBM RISC System/6000
// processor", IBM J. Res. Dev. 34(1), 1990).
//
// It is used for a whole tile or block when 2^-64 <= s <= 2^126 (then s and
// r are normal).  Within that range:
//   |x| >= 2^-100: the residual x - q0*s is exact and the result is the IEEE
//                  quotient, bit for bit;
//   |x| <  2^-100: |x / s| < 2^-36 and every intermediate stays below 2^-30,
//                  so the E4M3 / E2M1 code is +-0 exactly as with IEEE
//                  division (the binary32 quotient itself may differ in its
//                  last subnormal bits, and is never stored).
// pwq_selftest_division checks both statements over every BF16 numerator
// and every divisor the formats produce, against __fdiv_rn.
//
// Written with the negated numerator nx = -x and negated reciprocal nr = -r:
//   q0 = nx * nr (= x * r),  e = q0 * s + nx (= q0 * s - x, exact),
//   q  = e * nr + q0 (= q0 - e * r),
// the same roundings as q0 + (x - q0 * s) * r, but the final product
// (+0) * nr = -0 carries the sign of zero through: -0 / s gives -0 and +0 / s
// gives +0 with no extra instruction.
__device__ __forceinline__ float div_fast(float x, float s, float r) {
    const float nx = -x, nr = -r;
    const float q0 = __fmul_rn(nx, nr);
    const float e = __fmaf_rn(q0, s, nx);
    return __fmaf_rn(e, nr, q0);
}

__device__ __forceinline__ bool div_fast_ok(float s) { return s >= 0x1p-64f && s <= 0x1p126f; }

// Packed binary32 pairs (sm_100 f32x2 arithmetic: one instruction, two lanes).
__device__ __forceinline__ uint64_t f32x2_bits(uint32_t lo, uint32_t hi) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "r"(lo), "r"(hi));
    return r;
}
__device__ __forceinline__ uint64_t f32x2(float lo, float hi) {
    return f32x2_bits(__float_as_uint(lo), __float_as_uint(hi));
}
__device__ __forceinline__ float2 f32x2_split(uint64_t v) {
    float2 f;
    asm("mov.b64 {%0, %1}, %2;" : "=f"(f.x), "=f"(f.y) : "l"(v));
    return f;
}
__device__ __forceinline__ uint64_t mul_f32x2(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ uint64_t fma_f32x2(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}

// y = bf16(fl((dec(c) * dec(sb)) * gs)) for the 8 codes of a half block.
__device__ __forceinline__ uint4 dequant_half(uint32_t codes, float sbv, float gs) {
    uint32_t w[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const float2 c = e2m1x2_decode((codes >> (8 * j)) & 0xffu);
        w[j] = pack_bf16x2(__fmul_rn(__fmul_rn(c.x, sbv), gs), __fmul_rn(__fmul_rn(c.y, sbv), gs));
    }
    return make_uint4(w[0], w[1], w[2], w[3]);
}

// Two E4M3 codes (16 bits, code 0 low) -> their exact binary16 values.
__device__ __forceinline__ uint32_t e4m3x2_f16x2(uint32_t codes16) {
    uint32_t h2;
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"((uint16_t)codes16));
    return h2;
}

// dequant_half with dec(c) * dec(sb) taken as binary16 pairs, then times
// gs as binary32 pairs.  The binary16 product is exact: dec(c) has at most
// 2 significant bits and dec(sb) at most 4, and every non-zero product lies
// in [2^-10, 2688], inside binary16's normal range; so the one rounding is
// still fl(. * gs), then bf16.  sb2 = {dec(sb), dec(sb)} in binary16, gs2 =
// {gs, gs}.  Each byte is shifted out before its decode (decoding straight
// from a packed byte lane gave wrong results on the fast path).
// pwq_selftest_division(5) compares it with dequant_half for every code
// byte, every block scale and every global scale fl(a / 2688).
__device__ __forceinline__ uint4 dequant_half_h(uint32_t codes, uint32_t sb2, uint64_t gs2) {
    uint32_t h[4];
#pragma unroll
    for (int j = 0; j < 4; ++j)
        asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\tmov.b32 {b0, b1, b2, b3}, %1;\n\t"
            "cvt.rn.f16x2.e2m1x2 %0, b0;\n\t}" : "=r"(h[j]) : "r"((codes >> (8 * j)) & 0xffu));
    uint32_t w[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        uint32_t p2;
        asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(p2) : "r"(h[j]), "r"(sb2));
        float lo, hi;
        asm("cvt.f32.f16 %0, %1;" : "=f"(lo) : "h"((uint16_t)(p2 & 0xffffu)));
        asm("cvt.f32.f16 %0, %1;" : "=f"(hi) : "h"((uint16_t)(p2 >> 16)));
        const float2 y = f32x2_split(mul_f32x2(f32x2(lo, hi), gs2));
        w[j] = pack_bf16x2(y.x, y.y);
    }
    return make_uint4(w[0], w[1], w[2], w[3]);
}

// FP8 block-wise dequantisation of 8 codes (code 0 in bits 0..7 of c.x):
// BF16 bits of y = bf16(fl(dec(q) * s)), element 0 in the low half of .x.
// The products are taken two at a time (f32x2).
__device__ __forceinline__ uint4 fp8_dequant8(uint2 c, float s) {
    const uint64_t s2 = f32x2(s, s);
    uint32_t w[4];
#pragma unroll
    for (int h = 0; h < 4; ++h) {
        const uint32_t pair = ((h < 2 ? c.x : c.y) >> (16 * (h & 1))) & 0xffffu;
        const float2 f = e4m3x2_decode(pair);
        const float2 p = f32x2_split(mul_f32x2(f32x2(f.x, f.y), s2));
        w[h] = pack_bf16x2(p.x, p.y);
    }
    return make_uint4(w[0], w[1], w[2], w[3]);
}

// div_fast on the two BF16 values of a packed word w (low half first):
// s2 = {s, s}, nr2 = {-r, -r}.  The negated numerators come straight from
// the BF16 bits (widening and sign flip in one integer operation each; the
// low one as a multiply-add, w * 2^16 + 2^31, which issues on the FMA pipe
// and leaves the busier integer pipe to the rest).
__device__ __forceinline__ float2 div_fast_bf16x2(uint32_t w, uint64_t s2, uint64_t nr2) {
    uint32_t lo;
    asm("mad.lo.u32 %0, %1, 0x10000, 0x80000000;" : "=r"(lo) : "r"(w));
    const uint64_t nx = f32x2_bits(lo, (w & 0xffff0000u) ^ 0x80000000u);
    const uint64_t q0 = mul_f32x2(nx, nr2);
    const uint64_t e = fma_f32x2(q0, s2, nx);
    return f32x2_split(fma_f32x2(e, nr2, q0));
}

// Outside that range: IEEE division, with the zero-scale reading (s == 0
// gives a zero of x's sign).
__device__ __forceinline__ float div_slow(float x, float s) {
    if (s == 0.0f) return __uint_as_float(__float_as_uint(x) & 0x80000000u);
    return __fdiv_rn(x, s);
}

template <bool kFast>
__device__ __forceinline__ float quotient(float x, float s, float r) {
    return kFast ? div_fast(x, s, r) : div_slow(x, s);
}

// FP8 block-wise tile scale s = fl(amax / 448).  The divisor is the
// constant 448, so its reciprocal RN(1/448) = 0x3b124925 is exact input to
// the reciprocal path, which gives the IEEE quotient for amax >= 2^-100;
// smaller (BF16-subnormal-range) amax use IEEE division.  s is stored, so
// pwq_selftest_division checks it bit for bit for every BF16 amax.
__device__ __forceinline__ float fp8_tile_scale(float amax) {
    return amax >= 0x1p-100f ? div_fast(amax, 448.0f, __uint_as_float(0x3b124925u))
                             : __fdiv_rn(amax, 448.0f);
}

// The quotients of the two BF16 values of a packed word.
template <bool kFast>
__device__ __forceinline__ float2 quotient_bf16x2(uint32_t w, float s, float r) {
    if (kFast) return div_fast_bf16x2(w, f32x2(s, s), f32x2(-r, -r));
    return make_float2(div_slow(bf16_lo(w), s), div_slow(bf16_hi(w), s));
}

// The 8 quotients of a 16-byte BF16 chunk.
template <bool kFast>
__device__ __forceinline__ void quotients8(uint4 v, float s, float r, float q[8]) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 p = quotient_bf16x2<kFast>(w[i], s, r);
        q[2 * i] = p.x;
        q[2 * i + 1] = p.y;
    }
}

// FP8 block-wise re-quantisation of 8 codes: the codes of the dequantised
// values y = bf16(fl(dec(q) * s)) against the new tile scale s2 (r2 =
// RN(1/s2) on the reciprocal path, kFast).
template <bool kFast>
__device__ __forceinline__ uint2 fp8_requant8(uint2 c, float s, float s2, float r2) {
    const uint4 y = fp8_dequant8(c, s);
    float q[8];
    quotients8<kFast>(y, s2, r2, q);
    return make_uint2(e4m3x4(q[0], q[1], q[2], q[3]), e4m3x4(q[4], q[5], q[6], q[7]));
}

// ---------------------------------------------------------------- UE8M0

// e = min{k : amax <= 448 * 2^k} from the BF16 magnitude bits of amax,
// clamped to [-127, 127] (amax = 0 gives -127).  With amax = sig * 2^(E-msb)
// and sig an integer whose top bit is bit msb: 448 * 2^(E-8) = 1.75 * 2^E,
// so e = E - 8 when sig <= 1.75 * 2^msb and E - 7 otherwise.
__device__ __forceinline__ int ue8m0_exponent(uint32_t amax_bits16) {
    if (amax_bits16 == 0u) return -127;
    uint32_t ef = amax_bits16 >> 7, mant = amax_bits16 & 0x7fu;
    uint32_t sig = ef ? (0x80u | mant) : mant;
    int msb = 31 - __clz(sig);
    int E = (int)(ef ? ef : 1u) - 127 - 7 + msb;
    int e = E - 8 + ((4u * sig <= (7u << msb)) ? 0 : 1);
    return max(-127, min(127, e));
}

// 2^k as binary32 for k in [-127, 127] (2^-127 is subnormal).
__device__ __forceinline__ float exp2i(int k) {
    return k >= -126 ? __uint_as_float((uint32_t)(k + 127) << 23) : __uint_as_float(0x00400000u);
}

// ---------------------------------------------------------------- loads / stores

__device__ __forceinline__ uint4 ld_stream_v4(const void* p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
    return v;
}
__device__ __forceinline__ uint2 ld_stream_v2(const void* p) {
    uint2 v;
    asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0, %1}, [%2];"
                 : "=r"(v.x), "=r"(v.y) : "l"(p));
    return v;
}
// L2 eviction-priority policies for loads and stores that carry a cache hint.
__device__ __forceinline__ uint64_t l2_policy_evict_last() {
    uint64_t p;
    asm("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
    return p;
}
__device__ __forceinline__ uint64_t l2_policy_evict_first() {
    uint64_t p;
    asm("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
    return p;
}
__device__ __forceinline__ uint4 ld_hint_v4(const void* p, uint64_t pol) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.L2::cache_hint.v4.u32 {%0, %1, %2, %3}, [%4], %5;"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p), "l"(pol));
    return v;
}
__device__ __forceinline__ void st_hint_v4(void* p, uint4 v, uint64_t pol) {
    asm volatile("st.global.L2::cache_hint.v4.u32 [%0], {%1, %2, %3, %4}, %5;"
                 :: "l"(p), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w), "l"(pol) : "memory");
}

__device__ __forceinline__ void st_hint_v2(void* p, uint32_t a, uint32_t b, uint64_t pol) {
    asm volatile("st.global.L2::cache_hint.v2.u32 [%0], {%1, %2}, %3;" :: "l"(p), "r"(a), "r"(b), "l"(pol) : "memory");
}
// 32-byte store (sm_100 256-bit vector): p must be 32-byte aligned.
__device__ __forceinline__ void st_hint_v8(void* p, uint4 a, uint4 b, uint64_t pol) {
    asm volatile("st.global.L2::cache_hint.v8.u32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8}, %9;"
                 :: "l"(p), "r"(a.x), "r"(a.y), "r"(a.z), "r"(a.w), "r"(b.x), "r"(b.y), "r"(b.z), "r"(b.w), "l"(pol)
                 : "memory");
}

// 256-bit (32-byte) load / store, sm_100: p must be 32-byte aligned.
__device__ __forceinline__ void ld_nc_v8(const void* p, uint4& a, uint4& b) {
    asm volatile("ld.global.nc.L1::no_allocate.v8.u32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
                 : "=r"(a.x), "=r"(a.y), "=r"(a.z), "=r"(a.w), "=r"(b.x), "=r"(b.y), "=r"(b.z), "=r"(b.w)
                 : "l"(p));
}
__device__ __forceinline__ void st_v8(void* p, uint4 a, uint4 b) {
    asm volatile("st.global.v8.u32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};"
                 :: "l"(p), "r"(a.x), "r"(a.y), "r"(a.z), "r"(a.w), "r"(b.x), "r"(b.y), "r"(b.z), "r"(b.w)
                 : "memory");
}

__device__ __forceinline__ void st_v4(void* p, uint4 v) {
    asm volatile("st.global.v4.u32 [%0], {%1, %2, %3, %4};"
                 :: "l"(p), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w) : "memory");
}
__device__ __forceinline__ void st_v2(void* p, uint2 v) {
    asm volatile("st.global.v2.u32 [%0], {%1, %2};" :: "l"(p), "r"(v.x), "r"(v.y) : "memory");
}
__device__ __forceinline__ void st_u32(void* p, uint32_t v) {
    asm volatile("st.global.u32 [%0], %1;" :: "l"(p), "r"(v) : "memory");
}

// ---------------------------------------------------------------- fast division by a constant

// Unsigned 32-bit division by a runtime constant d >= 1 (round-up magic
// multiplier; T. Granlund and P. Montgomery, "Division by invariant integers
// using multiplication", PLDI 1994): q = (umulhi(n, m) + n) >> l with
// l = ceil(log2 d), m = floor(2^32 (2^l - d) / d) + 1.
struct FastDiv {
    uint32_t d, m, l;
};

inline FastDiv make_fastdiv(uint32_t d) {
    FastDiv f;
    f.d = d;
    uint32_t l = 0;
    while ((1ull << l) < d) ++l;
    f.l = l;
    f.m = (uint32_t)((((1ull << l) - d) << 32) / d + 1);
    return f;
}

__device__ __forceinline__ uint32_t fdiv(uint32_t n, const FastDiv& f) {
    uint32_t t = __umulhi(n, f.m);
    return (uint32_t)(((uint64_t)t + n) >> f.l);
}

// ---------------------------------------------------------------- device error word

// Bits of the device error word set by kernels whose bounded waits give up.
constexpr uint32_t kErrTmaTimeout = 1u;

__device__ __forceinline__ uint64_t globaltimer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
    return t;
}

// ---------------------------------------------------------------- mbarrier / TMA

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
    return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" :: "r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;"
                 :: "r"(bar), "r"(bytes) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t done;
    asm volatile("{\n\t.reg .pred p;\n\t"
                 "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
                 "selp.u32 %0, 1, 0, p;\n\t}"
                 : "=r"(done) : "r"(bar), "r"(parity) : "memory");
    return done != 0;
}

// Waits for the phase with the given parity to complete; gives up after
// `limit_ns` nanoseconds of wall time and returns false.
__device__ __forceinline__ bool mbar_wait_bounded(uint32_t bar, uint32_t parity, uint64_t limit_ns) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    for (;;) {
        for (int i = 0; i < 64; ++i)
            if (mbar_try_wait(bar, parity)) return true;
        if (globaltimer_ns() - t0 > limit_ns) return false;
    }
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" :: "r"(bar) : "memory");
}

// 1-D bulk async copy (no multicast) of `bytes` (a multiple of 16; both
// addresses 16-byte aligned) from global to shared memory, completing
// `bar`'s transaction count, with an L2 eviction-priority hint.
__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar,
                                          uint64_t pol) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1], %2, [%3], %4;"
        :: "r"(dst), "l"(src), "r"(bytes), "r"(bar), "l"(pol) : "memory");
}

// 3-D tiled TMA load (no multicast) of the box at (x, y, z) into shared
// memory, completing `bar`'s transaction count.
__device__ __forceinline__ void tma_load_3d(uint32_t dst, const void* tmap, uint32_t bar,
                                           int x, int y, int z) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4, %5}], [%2];"
        :: "r"(dst), "l"(tmap), "r"(bar), "r"(x), "r"(y), "r"(z) : "memory");
}

}  // namespace pwq
