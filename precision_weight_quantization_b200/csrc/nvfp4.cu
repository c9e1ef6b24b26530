// nvfp4.cu -- NVFP4 (E2M1 codes, 1x16 blocks, E4M3 block scale, FP32 global
// scale) group amax, quantise, fake-quantise and dequantise.
// Source: verl NVFP4 QAT article, section 2.3 (global scale =
// amax / (6 * 448), E4M3 block scale per 16 elements, nearest E2M1 value on
// {0, 0.5, 1, 1.5, 2, 3, 4, 6}, multiply back), 2.4 (q/k/v and gate/up
// siblings share the group's maximum amax), 3.3 (weight_scale_2 =
// amax / (6.0 * 448.0)); "Low Precision RL", "Choose a precision" table.
//
// Quantise and fake-quantise run as one single-pass launch per call
// (nvfp4_flow_kernel, described at its queue below): amax items and encode
// items of every group of the call share one work queue, and an encode
// item re-reads its data while it is still in L2.  Calls whose every
// instance is small run one thread-block cluster per instance instead
// (nvfp4_cluster_kernel).  Calls whose amax is given (amax_in, or the words
// of an amax launch: the entry point without allocation) run one streaming
// encode over the blocks of all their instances (nvfp4_units_kernel); the
// group amax alone (nvfp4_group_amax) is nvfp4_amax_kernel: every CTA
// reduces a slice of one group to a max and publishes it with one atomicMax
// on the group's word (the float bit patterns of non-negative values order
// like unsigned integers).  The NVFP4 "4over6" variant has its own pair of
// kernels over the same block space.
// The kernels also take an FP8 block-wise source (E4M3 codes with tile
// scales, dequantised in registers) for the re-quantisation calls.
// Dequantise is a grouped walk over 16-element blocks (8 packed bytes and a
// block-scale byte in, 32 bytes of BF16 out), eight blocks per lane in
// flight.
// Division: a group has at most 127 distinct code divisors d = fl(dec(sb) *
// gs), so each CTA tabulates d and RN(1/d) for every block-scale code in
// shared memory once; the block scale itself divides by fl(6 gs), whose
// reciprocal is also formed once.  Per element the quotient is the
// reciprocal product plus one FMA residual correction (pwq_device.cuh),
// which the self-test proves to give IEEE division's codes over every BF16
// numerator and every reachable divisor.
#include <algorithm>
#include <mutex>

#include <cooperative_groups.h>

#include "pwq_internal.h"

namespace pwq {
namespace {

constexpr int kThreads = 256;
constexpr int kUnroll = 8;
constexpr int kMaxSib = 8;

// One sibling of a group set, addressed per batch slab.  The source is BF16
// or, for the FP8 block re-quantisation, E4M3 codes with one FP32 scale per
// 128x128 tile (the kernels then see y = bf16(fl(dec(q) * s))).
struct Sib {
    const char* x;        // BF16, or E4M3 codes
    int64_t x_bs, x_rs;   // bytes
    const float* ts;      // FP8 source: tile scales [B][TM][TN]
    int64_t ts_bs;        // FP8 source: TM * TN
    uint32_t tn;          // FP8 source: TN
    char* out;            // packed codes (quant) or BF16 (fake); unused by amax
    int64_t o_bs, o_rs;   // bytes
    uint8_t* sb;          // dense [B][M][N/16] (quant only)
    uint32_t chunks;      // 8-element chunks per batch slab (M * N / 8)
    FastDiv cpr;          // chunks per row (N / 8)
    int dense_x, dense_o; // slab rows are contiguous
    int vec16_x;          // FP8 source: every block's 16 codes start on a 16-byte boundary
    int vec32_x, vec32_o; // BF16 source / fake-quant output: every block's 32 bytes on a 32-byte boundary
};

// The 32 bytes of a 16-element BF16 block at byte offset xo of a member's
// source: one 256-bit load when the member's blocks are 32-byte aligned
// (the two halves then leave L2 as one request), else two 128-bit loads.
__device__ __forceinline__ void ld_block32(const char* p, int vec32, uint4& lo, uint4& hi) {
    if (vec32) {
        ld_nc_v8(p, lo, hi);
    } else {
        lo = ld_stream_v4(p);
        hi = ld_stream_v4(p + 16);
    }
}
// The 32 bytes of a fake-quantised block at p.
__device__ __forceinline__ void st_block32(char* p, int vec32, uint4 y0, uint4 y1) {
    if (vec32) {
        st_v8(p, y0, y1);
    } else {
        st_v4(p, y0);
        st_v4(p + 16, y1);
    }
}

struct AmaxArgs {
    Sib s[kMaxSib];
    int n;
    uint32_t* amax_bits;  // [B]
};

__device__ __forceinline__ uint32_t block_max_u32(uint32_t m) {
    __shared__ uint32_t red[kThreads / 32];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, o));
    if ((threadIdx.x & 31u) == 0u) red[threadIdx.x >> 5] = m;
    __syncthreads();
    if (threadIdx.x < 32u) {
        m = threadIdx.x < (kThreads / 32) ? red[threadIdx.x] : 0u;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, o));
    }
    return m;
}

// Chunk c of an FP8-source slab: its 8 codes and its tile scale.
__device__ __forceinline__ uint2 fp8_chunk(const Sib& S, const char* base, const float* tsb, uint32_t c,
                                           float& s) {
    const uint32_t r = fdiv(c, S.cpr);
    const uint32_t k = c - r * S.cpr.d;
    const int64_t off = S.dense_x ? (int64_t)c * 8 : (int64_t)r * S.x_rs + (int64_t)k * 8;
    s = __ldg(tsb + (r >> 7) * S.tn + (k >> 4));
    return ld_stream_v2(base + off);
}

template <bool kFp8>
__global__ void __launch_bounds__(kThreads) nvfp4_amax_kernel(const AmaxArgs a) {
    const uint32_t b = blockIdx.y;
    const uint32_t stride = gridDim.x * blockDim.x;
    const uint32_t t0 = blockIdx.x * blockDim.x + threadIdx.x;
    uint32_t m = 0u;
    for (int i = 0; i < a.n; ++i) {
        const Sib& S = a.s[i];
        const char* base = S.x + (int64_t)b * S.x_bs;
        if constexpr (kFp8) {
            const float* tsb = S.ts + (int64_t)b * S.ts_bs;
            for (uint32_t c0 = t0; c0 < S.chunks; c0 += stride * kUnroll) {
                uint2 v[kUnroll];
                float sc[kUnroll];
#pragma unroll
                for (int u = 0; u < kUnroll; ++u) {
                    const uint32_t c = c0 + u * stride;
                    v[u] = make_uint2(0u, 0u);
                    sc[u] = 0.0f;
                    if (c < S.chunks) v[u] = fp8_chunk(S, base, tsb, c, sc[u]);
                }
#pragma unroll
                for (int u = 0; u < kUnroll; ++u) m = max(m, fp8_amax_bits16(e4m3_maxmag8(v[u]), sc[u]));
            }
        } else {
            for (uint32_t c0 = t0; c0 < S.chunks; c0 += stride * kUnroll) {
                uint4 v[kUnroll];
#pragma unroll
                for (int u = 0; u < kUnroll; ++u) {
                    const uint32_t c = c0 + u * stride;
                    v[u] = make_uint4(0u, 0u, 0u, 0u);
                    if (c < S.chunks) {
                        int64_t off;
                        if (S.dense_x) {
                            off = (int64_t)c * 16;
                        } else {
                            const uint32_t r = fdiv(c, S.cpr);
                            off = (int64_t)r * S.x_rs + (int64_t)(c - r * S.cpr.d) * 16;
                        }
                        v[u] = ld_stream_v4(base + off);
                    }
                }
#pragma unroll
                for (int u = 0; u < kUnroll; ++u) m = max(m, amax_bits8(v[u]));
            }
        }
    }
    m = block_max_u32(m);
    if (threadIdx.x == 0 && m != 0u) atomicMax(a.amax_bits + b, m << 16);
}

// Per-group constants of the encode pass, for every E4M3 block-scale code
// k: d_k = fl(dec(k) * gs) (the code divisor), r_k = RN(1/d_k) when d_k is
// in the reciprocal path's range (else 0: IEEE division), and dec(k).
struct ScaleTable {
    float2 e[128];   // {d_k, RN(1 / d_k)}, or {d_k, 0} off the reciprocal path
};

__device__ __forceinline__ void fill_scale_table(ScaleTable& t, float gs) {
    for (uint32_t k = threadIdx.x; k < 128u; k += blockDim.x) {
        const float dec = e4m3_decode(k);  // k = 0x7f (NaN) is never produced
        const float d = __fmul_rn(dec, gs);
        t.e[k] = make_float2(d, div_fast_ok(d) ? __frcp_rn(d) : 0.0f);
    }
}

// Per block-scale code k, the dequantised magnitudes y(m) =
// bf16(fl(fl(dec(m) dec(k)) gs)) of the 8 E2M1 magnitude codes m, as
// dequant_half_h computes them, in byte planes for byte permutes: {low
// bytes of y(0..3), low bytes of y(4..7), high bytes of y(0..3), high
// bytes of y(4..7)}.  A fake-quantised block then looks its values up
// instead of decoding and multiplying each one.
struct DeqTable {
    uint4 e[128];
};

__device__ __forceinline__ void fill_deq_table(DeqTable& t, uint64_t gs2) {
    for (uint32_t k = threadIdx.x; k < 128u; k += blockDim.x) {
        const uint4 w = dequant_half_h(0x76543210u, e4m3x2_f16x2(k * 0x101u), gs2);   // y(0), y(1), ..., y(7)
        t.e[k] = make_uint4(__byte_perm(w.x, w.y, 0x6420u), __byte_perm(w.z, w.w, 0x6420u),
                            __byte_perm(w.x, w.y, 0x7531u), __byte_perm(w.z, w.w, 0x7531u));
    }
}

// The BF16 values of the 8 E2M1 codes of a half block (element 0 in bits
// 0..3) from the block's DeqTable entry tb, each with the sign of its input
// value in x: with a positive divisor a code carries its input's sign,
// signed zeros included, and rounding is symmetric in sign, so y(-m) is
// -y(m).  Byte permutes pick the magnitude bytes (3-bit indices), then
// interleave the low and high bytes into BF16 pairs.
__device__ __forceinline__ uint4 dequant_lookup8(uint32_t codes, uint4 tb, uint4 x) {
    const uint32_t s0 = codes & 0x7777u, s1 = (codes >> 16) & 0x7777u;
    const uint32_t l0 = __byte_perm(tb.x, tb.y, s0), h0 = __byte_perm(tb.z, tb.w, s0);
    const uint32_t l1 = __byte_perm(tb.x, tb.y, s1), h1 = __byte_perm(tb.z, tb.w, s1);
    return make_uint4(__byte_perm(l0, h0, 0x5140u) | (x.x & 0x80008000u),
                      __byte_perm(l0, h0, 0x7362u) | (x.y & 0x80008000u),
                      __byte_perm(l1, h1, 0x5140u) | (x.z & 0x80008000u),
                      __byte_perm(l1, h1, 0x7362u) | (x.w & 0x80008000u));
}

// E2M1 codes of one 8-element half block (element 0 in bits 0..3).
__device__ __forceinline__ uint32_t codes_half(uint4 v, float d, float r) {
    float q[8];
    if (r != 0.0f)
        quotients8<true>(v, d, r, q);
    else
        quotients8<false>(v, d, r, q);
    return e2m1x2(q[0], q[1]) | (e2m1x2(q[2], q[3]) << 8) | (e2m1x2(q[4], q[5]) << 16) |
           (e2m1x2(q[6], q[7]) << 24);
}

// NVFP4 "4over6" (vime pull request #503, NVFP4 QDQ config thread:
// NVTE_NVFP4_4OVER6 and NVTE_NVFP4_4OVER6_E4M3_USE_256).  The global scale
// leaves room for a larger block scale, gs = fl(A / (6 E)) with E = 256 (or
// 448); every block is encoded twice, its amax mapped to 6 (the NVFP4 rule)
// and to 4, and keeps the candidate whose dequantised values have the
// smaller sum of squared errors -- fl(fl(x - y)^2) added left to right in
// binary32, ties keeping 6.  The output is plain NVFP4 (nvfp4_dequant reads
// it).
//
// Work units are 16-element blocks.  The units of a launch (up to 16
// members in up to 16 sibling groups) form one index space: group after
// group, batch index (instance) after batch index, member after member, row
// after row.  Each persistent CTA takes one contiguous range of it, so a
// 256-expert batch fills every SM as well as one large tensor does.  Two
// launches: the amax kernel reduces each instance piece of a range to one
// atomicMax on the instance's word; the encode kernel walks its range
// backwards, one instance piece at a time (the scale table depends on the
// instance's gs), so that the data its own amax pass read last -- still in
// L2 -- comes first.  The error sum is one chain over a block, so a thread
// owns whole blocks (two 16-byte chunks); neighbouring threads take
// neighbouring blocks.
struct FourSixGroup {
    uint64_t unit0;         // first unit of the group in the launch
    uint32_t units;         // units per instance: sum of the members' blocks
    uint32_t inst0;         // first amax word of the group
    uint32_t batch;         // instances
    int m0, nm;             // members m0 .. m0 + nm - 1
    const float* amax_in;   // [batch] or null
    float* gs_out;          // [batch] or null
    float* amax_out;        // [batch] or null
};

struct FourSixArgs {
    Sib m[kMaxLaunchTensors];
    uint32_t mblk0[kMaxLaunchTensors];   // first unit of each member inside its instance
    FourSixGroup g[kMaxLaunchTensors];
    int n_groups;
    uint64_t total;                      // units of the launch
    uint32_t* amax_bits;                 // one word per instance
    float six_e;                         // 6 E: 2688 or 1536
};

// The CTA's contiguous range of units.
__device__ __forceinline__ void four_six_range(const FourSixArgs& a, uint64_t& lo, uint64_t& hi) {
    const uint64_t per = (a.total + gridDim.x - 1) / gridDim.x;
    lo = min(a.total, (uint64_t)blockIdx.x * per);
    hi = min(a.total, lo + per);
}

// Group, instance and the instance's first unit of unit u.
__device__ __forceinline__ void four_six_locate(const FourSixArgs& a, uint64_t u, int& gi, uint32_t& b,
                                                uint64_t& inst_lo) {
    gi = 0;
    while (gi + 1 < a.n_groups && u >= a.g[gi + 1].unit0) ++gi;
    const FourSixGroup& G = a.g[gi];
    b = (uint32_t)((u - G.unit0) / G.units);
    inst_lo = G.unit0 + (uint64_t)b * G.units;
}

// Member, and the byte offsets of a block's input and output (and its
// block-scale index), for unit r of an instance of group G.
__device__ __forceinline__ int four_six_member(const FourSixArgs& a, const FourSixGroup& G, uint32_t r) {
    int i = G.m0 + G.nm - 1;
    while (r < a.mblk0[i]) --i;
    return i;
}

template <bool kFake>
__device__ __forceinline__ void four_six_offsets(const Sib& S, uint32_t b, uint32_t j, int64_t& xo, int64_t& oo) {
    const uint32_t c = 2u * j;   // the block's first chunk; c + 1 is in the same row
    if (S.dense_x && S.dense_o) {
        xo = (int64_t)c * 16;
        oo = (int64_t)c * (kFake ? 16 : 4);
    } else {
        const uint32_t r = fdiv(c, S.cpr);
        const uint32_t k = c - r * S.cpr.d;
        xo = S.dense_x ? (int64_t)c * 16 : (int64_t)r * S.x_rs + (int64_t)k * 16;
        oo = S.dense_o ? (int64_t)c * (kFake ? 16 : 4) : (int64_t)r * S.o_rs + (int64_t)k * (kFake ? 16 : 4);
    }
    xo += (int64_t)b * S.x_bs;
    oo += (int64_t)b * S.o_bs;
}

// The BF16 pairs of a chunk widened to binary32 pairs (element 0 first).
__device__ __forceinline__ void widen8(uint4 v, uint64_t (&w)[4]) {
    const uint32_t a[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) w[i] = f32x2_bits(a[i] << 16, a[i] & 0xffff0000u);
}

// err + sum of fl(fl(x_j - y_j)^2) over the 8 elements of a chunk, one
// rounding per operation, element 0 first.  fl(x - y) is taken as
// fma(y, -1, x): the product is exact, so the one rounding is the
// difference's.
__device__ __forceinline__ float sse8(const uint64_t (&x)[4], uint4 y, float err) {
    uint64_t yw[4];
    widen8(y, yw);
    const uint64_t m1 = f32x2(-1.0f, -1.0f);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const uint64_t d = fma_f32x2(yw[i], m1, x[i]);
        const float2 sq = f32x2_split(mul_f32x2(d, d));
        err = __fadd_rn(err, sq.x);
        err = __fadd_rn(err, sq.y);
    }
    return err;
}

// E2M1 codes of 8 values widened to binary32 pairs, divided by d on the
// reciprocal path (nr2 = {-r, -r}, r = RN(1/d)).  The quotient is formed
// negated -- q0 = x (-r), e = q0 d + x, q = e (-r) + q0, one rounding each
// -- which is exactly the negation of div_fast's quotient (every step is
// the same operation with all signs flipped, and rounding to nearest is
// symmetric in sign), so flipping the sign bit of each code gives the codes
// of the quotient itself, signed zeros included.
__device__ __forceinline__ uint32_t codes_neg8(const uint64_t (&x)[4], uint64_t d2, uint64_t nr2) {
    float q[8];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const uint64_t q0 = mul_f32x2(x[i], nr2);
        const uint64_t e = fma_f32x2(q0, d2, x[i]);
        const float2 qn = f32x2_split(fma_f32x2(e, nr2, q0));
        q[2 * i] = qn.x;
        q[2 * i + 1] = qn.y;
    }
    return e2m1x8(q) ^ 0x88888888u;
}

// One candidate of a block: the block scale code for the amax divided by
// t_gs = fl(t gs), the codes of its two chunks, and the error of their
// dequantised values.
__device__ __forceinline__ float four_six_candidate(uint4 lo, uint4 hi, const uint64_t (&xl)[4],
                                                    const uint64_t (&xh)[4], float amax_b, float t_gs, float rt,
                                                    bool fast_t, const ScaleTable& tab, const DeqTable& dtab,
                                                    uint64_t gs2, uint32_t& sb, uint32_t& c0, uint32_t& c1,
                                                    uint4& y0, uint4& y1) {
    const float ratio = fast_t ? div_fast(amax_b, t_gs, rt) : div_slow(amax_b, t_gs);
    sb = e4m3x2(ratio, 0.0f) & 0x7fu;   // ratio >= 0
    const float2 e = tab.e[sb];
    if (e.y != 0.0f) {   // d > 0 finite, so gs is: the table holds the values
        const uint64_t d2 = f32x2(e.x, e.x), nr2 = f32x2(-e.y, -e.y);
        c0 = codes_neg8(xl, d2, nr2);
        c1 = codes_neg8(xh, d2, nr2);
        const uint4 tb = dtab.e[sb];
        y0 = dequant_lookup8(c0, tb, lo);
        y1 = dequant_lookup8(c1, tb, hi);
    } else {
        c0 = codes_half(lo, e.x, e.y);
        c1 = codes_half(hi, e.x, e.y);
        const uint32_t sb2 = e4m3x2_f16x2(sb * 0x101u);
        y0 = dequant_half_h(c0, sb2, gs2);
        y1 = dequant_half_h(c1, sb2, gs2);
    }
    return sse8(xh, y1, sse8(xl, y0, 0.0f));
}

constexpr int kFourSixCtasPerSm = 3;
constexpr int kFourSixAmaxUnroll = 4;

__global__ void __launch_bounds__(kThreads) nvfp4_4over6_amax_kernel(const FourSixArgs a) {
    __shared__ uint32_t red[kThreads / 32];
    uint64_t lo, hi;
    four_six_range(a, lo, hi);
    for (uint64_t u = lo; u < hi;) {
        int gi;
        uint32_t b;
        uint64_t inst_lo;
        four_six_locate(a, u, gi, b, inst_lo);
        const FourSixGroup& G = a.g[gi];
        const uint64_t end = min(hi, inst_lo + G.units);   // this instance's piece of the range
        if (!G.amax_in) {
            uint32_t m = 0u;
            const uint32_t r0 = (uint32_t)(u - inst_lo), r1 = (uint32_t)(end - inst_lo);
            for (uint32_t r = r0 + threadIdx.x; r < r1; r += kThreads * kFourSixAmaxUnroll) {
                uint4 v[2 * kFourSixAmaxUnroll];
#pragma unroll
                for (int k = 0; k < kFourSixAmaxUnroll; ++k) {
                    const uint32_t rk = r + (uint32_t)k * kThreads;
                    v[2 * k] = v[2 * k + 1] = make_uint4(0u, 0u, 0u, 0u);
                    if (rk < r1) {
                        const int i = four_six_member(a, G, rk);
                        int64_t xo, oo;
                        four_six_offsets<true>(a.m[i], b, rk - a.mblk0[i], xo, oo);
                        v[2 * k] = ld_stream_v4(a.m[i].x + xo);
                        v[2 * k + 1] = ld_stream_v4(a.m[i].x + xo + 16);
                    }
                }
#pragma unroll
                for (int k = 0; k < 2 * kFourSixAmaxUnroll; ++k) m = max(m, amax_bits8(v[k]));
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, o));
            if ((threadIdx.x & 31u) == 0u) red[threadIdx.x >> 5] = m;
            __syncthreads();
            if (threadIdx.x == 0) {
                for (int w = 1; w < kThreads / 32; ++w) m = max(m, red[w]);
                if (m != 0u) atomicMax(a.amax_bits + G.inst0 + b, m << 16);
            }
            __syncthreads();   // red is reused by the next piece
        }
        u = end;
    }
}

template <bool kFake>
__global__ void __launch_bounds__(kThreads, kFourSixCtasPerSm) nvfp4_4over6_kernel(const FourSixArgs a) {
    __shared__ ScaleTable tab;
    __shared__ DeqTable dtab;
    uint64_t lo, hi;
    four_six_range(a, lo, hi);
    for (uint64_t u = hi; u > lo;) {
        int gi;
        uint32_t b;
        uint64_t inst_lo;
        four_six_locate(a, u - 1, gi, b, inst_lo);
        const FourSixGroup& G = a.g[gi];
        const uint64_t start = max(lo, inst_lo);   // this instance's piece of the range: [start, u)
        const float A = G.amax_in ? G.amax_in[b] : __uint_as_float(a.amax_bits[G.inst0 + b]);
        const float gs = __fdiv_rn(A, a.six_e);
        const float g6 = __fmul_rn(6.0f, gs), g4 = __fmul_rn(4.0f, gs);
        const float r6 = __frcp_rn(g6), r4 = __frcp_rn(g4);
        const bool fast6 = div_fast_ok(g6), fast4 = div_fast_ok(g4);
        const uint64_t gs2 = f32x2(gs, gs);
        __syncthreads();   // the previous piece's table reads are done
        fill_scale_table(tab, gs);
        fill_deq_table(dtab, gs2);
        if (start == inst_lo && threadIdx.x == 0) {   // the one CTA that holds the instance's first unit
            if (G.gs_out) G.gs_out[b] = gs;
            if (G.amax_out) G.amax_out[b] = A;
        }
        __syncthreads();
        // the piece's member segments, last first (member i holds units
        // [mblk0[i], mblk0[i + 1]) of the instance); per segment the
        // member's values are CTA-uniform and read once; its blocks
        // j = jh - 1 - k, k = tid, tid + kThreads, ..., the next block's two
        // loads issued before the current one is encoded
        const uint32_t rs = (uint32_t)(start - inst_lo), re = (uint32_t)(u - inst_lo);
        int i = four_six_member(a, G, re - 1u);
        for (uint32_t se = re; se > rs; --i) {
            const Sib& S = a.m[i];
            const uint32_t m0 = a.mblk0[i];
            const uint32_t ss = max(rs, m0);
            const uint32_t jh = se - m0, n = se - ss;
            se = ss;
            const char* xb = S.x + (int64_t)b * S.x_bs;
            char* ob = S.out + (int64_t)b * S.o_bs;
            uint8_t* sbb = kFake ? nullptr : S.sb + (int64_t)b * (S.chunks >> 1);
            const bool dense_x = S.dense_x, dense_o = S.dense_o;
            const FastDiv cpr = S.cpr;
            const int64_t x_rs = S.x_rs, o_rs = S.o_rs;
            auto fetch = [&](uint32_t j, uint4& flo, uint4& fhi, int64_t& foo) {
                const uint32_t c = 2u * j;   // the block's first chunk; c + 1 is in the same row
                uint32_t r = 0u, kc = 0u;
                if (!dense_x || !dense_o) {
                    r = fdiv(c, cpr);
                    kc = c - r * cpr.d;
                }
                constexpr uint32_t kOb = kFake ? 16u : 4u;   // output bytes per chunk
                const char* p = xb + (dense_x ? (int64_t)c * 16 : (int64_t)r * x_rs + (int64_t)kc * 16);
                foo = dense_o ? (int64_t)c * kOb : (int64_t)r * o_rs + (int64_t)kc * kOb;
                flo = ld_stream_v4(p);
                fhi = ld_stream_v4(p + 16);
            };
            uint4 nlo = make_uint4(0u, 0u, 0u, 0u), nhi = nlo;
            int64_t noo = 0;
            if (threadIdx.x < n) fetch(jh - 1u - threadIdx.x, nlo, nhi, noo);
            for (uint32_t k = threadIdx.x; k < n; k += kThreads) {
                const uint4 lo4 = nlo, hi4 = nhi;
                const int64_t ooc = noo;
                const uint32_t jc = jh - 1u - k;
                if (k + kThreads < n) fetch(jc - kThreads, nlo, nhi, noo);
                const uint32_t mw = hmax_abs(amax_word8(lo4), amax_word8(hi4)) & 0x7fff7fffu;
                const float amax_b = __uint_as_float(max(mw & 0xffffu, mw >> 16) << 16);
                uint64_t xl[4], xh[4];
                widen8(lo4, xl);
                widen8(hi4, xh);
                uint32_t sb6, a0, a1, sb4, b0, b1;
                uint4 ya0, ya1, yb0, yb1;
                const float e6 = four_six_candidate(lo4, hi4, xl, xh, amax_b, g6, r6, fast6, tab, dtab, gs2, sb6, a0, a1,
                                                    ya0, ya1);
                const float e4 = four_six_candidate(lo4, hi4, xl, xh, amax_b, g4, r4, fast4, tab, dtab, gs2, sb4, b0, b1,
                                                    yb0, yb1);
                const bool four = e4 < e6;
                if (kFake) {
                    st_v4(ob + ooc, four ? yb0 : ya0);
                    st_v4(ob + ooc + 16, four ? yb1 : ya1);
                } else {
                    st_v2(ob + ooc, make_uint2(four ? b0 : a0, four ? b1 : a1));   // 8-byte aligned: 2 jc even
                    sbb[jc] = (uint8_t)(four ? sb4 : sb6);
                }
            }
        }
        u = start;
    }
}

// ---------------------------------------------------------------- plain NVFP4 with a given amax
//
// Quantise / fake-quantise when every instance's amax is known before the
// launch (amax_in: a cached or all-reduced value; or the words an amax
// launch has just written): one streaming pass over the unit space of the
// 4over6 kernels, each persistent CTA walking its contiguous range
// backwards one instance piece at a time (the scale table belongs to the
// instance's gs), one thread per 16-element block, the next block's loads
// issued before the current one is encoded.  kFp8: an FP8 block-wise source
// whose codes are dequantised in registers, y = bf16(fl(dec(q) s)).  Four
// CTAs per SM (at most 64 registers a thread): a block's 32 bytes are one
// 256-bit access where aligned, and more blocks in flight per thread
// measured no faster than the fourth CTA.

constexpr int kUnitCtasPerSm = 4;
template <bool kFake, bool kFp8>
__global__ void __launch_bounds__(kThreads, kUnitCtasPerSm) nvfp4_units_kernel(const FourSixArgs a) {
    __shared__ ScaleTable tab;
    uint64_t lo, hi;
    four_six_range(a, lo, hi);
    for (uint64_t u = hi; u > lo;) {
        int gi;
        uint32_t b;
        uint64_t inst_lo;
        four_six_locate(a, u - 1, gi, b, inst_lo);
        const FourSixGroup& G = a.g[gi];
        const uint64_t start = max(lo, inst_lo);   // this instance's piece of the range: [start, u)
        const float A = G.amax_in ? G.amax_in[b] : __uint_as_float(a.amax_bits[G.inst0 + b]);
        const float gs = __fdiv_rn(A, 2688.0f);
        const float six_gs = __fmul_rn(6.0f, gs);
        const float r6 = __frcp_rn(six_gs);
        const bool fast6 = div_fast_ok(six_gs);
        // every non-zero block scale gives dec(sb) * gs in [2^-9 gs, 448 gs]
        const bool all_fast = fast6 && __fmul_rn(0x1p-9f, gs) >= 0x1p-64f && __fmul_rn(448.0f, gs) <= 0x1p126f;
        const uint64_t gs2 = f32x2(gs, gs);
        __syncthreads();   // the previous piece's table reads are done
        fill_scale_table(tab, gs);
        if (start == inst_lo && threadIdx.x == 0) {   // the one CTA that holds the instance's first unit
            if (G.gs_out) G.gs_out[b] = gs;
            if (G.amax_out) G.amax_out[b] = A;
        }
        __syncthreads();
        const uint32_t rs = (uint32_t)(start - inst_lo), re = (uint32_t)(u - inst_lo);
        // the piece's member segments, last first: member i holds units
        // [mblk0[i], mblk0[i + 1]) of the instance.  Per segment the
        // member's values are CTA-uniform and read once; its blocks
        // j = jh - 1 - k, k = tid, tid + kThreads, ..., the next block's
        // loads issued before the current one is encoded.
        int i = four_six_member(a, G, re - 1u);
        for (uint32_t se = re; se > rs; --i) {
            const Sib& S = a.m[i];
            const uint32_t m0 = a.mblk0[i];
            const uint32_t ss = max(rs, m0);
            const uint32_t jh = se - m0, n = se - ss;
            se = ss;
            const char* xb = S.x + (int64_t)b * S.x_bs;
            char* ob = S.out + (int64_t)b * S.o_bs;
            uint8_t* sbb = kFake ? nullptr : S.sb + (int64_t)b * (S.chunks >> 1);
            const float* tsb = kFp8 ? S.ts + (int64_t)b * S.ts_bs : nullptr;
            const bool dense_x = S.dense_x, dense_o = S.dense_o;
            const int vec_x = kFp8 ? S.vec16_x : S.vec32_x, vec_o = S.vec32_o;
            const FastDiv cpr = S.cpr;
            const int64_t x_rs = S.x_rs, o_rs = S.o_rs;
            const uint32_t tn = S.tn;
            // block j: its source bytes (and, FP8, its tile scale) and its output offset
            auto fetch = [&](uint32_t j, uint4& flo, uint4& fhi, float& fsc, int64_t& foo) {
                const uint32_t c = 2u * j;   // the block's first chunk; c + 1 is in the same row
                uint32_t r = 0u, kc = 0u;
                if (kFp8 || !dense_x || !dense_o) {
                    r = fdiv(c, cpr);
                    kc = c - r * cpr.d;
                }
                constexpr uint32_t kXb = kFp8 ? 8u : 16u, kOb = kFake ? 16u : 4u;   // bytes per chunk
                const char* p = xb + (dense_x ? (int64_t)c * kXb : (int64_t)r * x_rs + (int64_t)kc * kXb);
                foo = dense_o ? (int64_t)c * kOb : (int64_t)r * o_rs + (int64_t)kc * kOb;
                if (kFp8) {
                    fsc = __ldg(tsb + (r >> 7) * tn + (kc >> 4));
                    if (vec_x) {
                        flo = ld_stream_v4(p);
                    } else {
                        const uint2 c0 = ld_stream_v2(p), c1 = ld_stream_v2(p + 8);
                        flo = make_uint4(c0.x, c0.y, c1.x, c1.y);
                    }
                } else {
                    ld_block32(p, vec_x, flo, fhi);
                }
            };
            uint4 nlo = make_uint4(0u, 0u, 0u, 0u), nhi = nlo;
            float nsc = 0.0f;
            int64_t noo = 0;
            if (threadIdx.x < n) fetch(jh - 1u - threadIdx.x, nlo, nhi, nsc, noo);
            for (uint32_t k = threadIdx.x; k < n; k += kThreads) {
                uint4 lo4 = nlo, hi4 = nhi;
                const float sc = nsc;
                const int64_t ooc = noo;
                const uint32_t jc = jh - 1u - k;
                if (k + kThreads < n) fetch(jc - kThreads, nlo, nhi, nsc, noo);
                if (kFp8) {
                    hi4 = fp8_dequant8(make_uint2(lo4.z, lo4.w), sc);
                    lo4 = fp8_dequant8(make_uint2(lo4.x, lo4.y), sc);
                }
                const uint32_t mw = hmax_abs(amax_word8(lo4), amax_word8(hi4)) & 0x7fff7fffu;
                const float amax_b = __uint_as_float(max(mw & 0xffffu, mw >> 16) << 16);
                const float ratio = fast6 ? div_fast(amax_b, six_gs, r6) : div_slow(amax_b, six_gs);
                const uint32_t sb = e4m3x2(ratio, 0.0f) & 0x7fu;   // ratio >= 0
                const float2 e = tab.e[sb];
                uint32_t c0, c1;
                if (all_fast) {
                    float q[8];
                    quotients8<true>(lo4, e.x, e.y, q);
                    c0 = e2m1x8(q);
                    quotients8<true>(hi4, e.x, e.y, q);
                    c1 = e2m1x8(q);
                } else {
                    c0 = codes_half(lo4, e.x, e.y);
                    c1 = codes_half(hi4, e.x, e.y);
                }
                if (kFake) {
                    const uint32_t sb2 = e4m3x2_f16x2(sb * 0x101u);
                    st_block32(ob + ooc, vec_o, dequant_half_h(c0, sb2, gs2), dequant_half_h(c1, sb2, gs2));
                } else {
                    st_v2(ob + ooc, make_uint2(c0, c1));   // 8-byte aligned: 2 jc even
                    sbb[jc] = (uint8_t)sb;
                }
            }
        }
        u = start;
    }
}

// ---------------------------------------------------------------- small instances, one cluster each
//
// When every instance (batch index of a sibling group) of a call has at most
// kClusterUnits 16-element blocks, one thread-block cluster of up to
// kMaxCluster CTAs owns each instance: every thread holds up to
// kClusterUnitsPerThread blocks in registers, the CTA maxima meet across the
// cluster in distributed shared memory (barrier.cluster orders them), and
// the blocks are encoded from the registers.  One launch, one read of the
// input, no workspace and no global atomics -- for the small tensors whose
// time the single pass's queue, amax handshake and workspace clear would
// dominate.  The units of an instance are numbered as for the 4over6 kernels
// (member after member, row after row); CTA r of a cluster takes the r-th
// contiguous share of them.
namespace cg = cooperative_groups;

constexpr int kClusterUnitsPerThread = 4;
constexpr int kClusterCtaUnits = kThreads * kClusterUnitsPerThread;   // 1024 blocks per CTA
constexpr int kMaxCluster = 8;                                         // portable cluster size
constexpr uint32_t kClusterUnits = kMaxCluster * kClusterCtaUnits;     // 131072 elements

template <bool kFake>
__global__ void __launch_bounds__(kThreads) nvfp4_cluster_kernel(const FourSixArgs a) {
    __shared__ ScaleTable tab;
    __shared__ uint32_t red[kThreads / 32];
    __shared__ uint32_t cta_max, s_amax;
    const cg::cluster_group cluster = cg::this_cluster();
    const uint32_t cs = cluster.num_blocks(), rank = cluster.block_rank();
    const uint32_t inst = blockIdx.x / cs;
    int gi = 0;
    while (gi + 1 < a.n_groups && inst >= a.g[gi + 1].inst0) ++gi;
    const FourSixGroup& G = a.g[gi];
    const uint32_t b = inst - G.inst0;
    const uint32_t per = (G.units + cs - 1) / cs;
    const uint32_t u0 = min(G.units, rank * per), u1 = min(G.units, u0 + per);

    // ---- the CTA's blocks into registers, and their maximum
    uint4 lo[kClusterUnitsPerThread], hi[kClusterUnitsPerThread];
    uint32_t m = 0u;
#pragma unroll
    for (int k = 0; k < kClusterUnitsPerThread; ++k) {
        const uint32_t r = u0 + threadIdx.x + (uint32_t)k * kThreads;
        lo[k] = hi[k] = make_uint4(0u, 0u, 0u, 0u);
        if (r < u1) {
            const int i = four_six_member(a, G, r);
            int64_t xo, oo;
            four_six_offsets<kFake>(a.m[i], b, r - a.mblk0[i], xo, oo);
            ld_block32(a.m[i].x + xo, a.m[i].vec32_x, lo[k], hi[k]);
        }
        m = max(m, max(amax_bits8(lo[k]), amax_bits8(hi[k])));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, o));
    if ((threadIdx.x & 31u) == 0u) red[threadIdx.x >> 5] = m;
    __syncthreads();
    if (threadIdx.x == 0) {
        for (int w = 1; w < kThreads / 32; ++w) m = max(m, red[w]);
        cta_max = m;
    }
    // ---- the group amax: every CTA reads every CTA's maximum of the cluster
    cluster.sync();
    if (threadIdx.x < 32u) {
        uint32_t v = threadIdx.x < cs ? *cluster.map_shared_rank(&cta_max, threadIdx.x) : 0u;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) v = max(v, __shfl_xor_sync(0xffffffffu, v, o));
        if (threadIdx.x == 0) s_amax = v;
    }
    // no CTA may leave while another still reads its cta_max: arrive now,
    // wait before the end
    cluster.barrier_arrive();
    __syncthreads();
    const float A = G.amax_in ? G.amax_in[b] : __uint_as_float(s_amax << 16);
    const float gs = __fdiv_rn(A, 2688.0f);
    const float six_gs = __fmul_rn(6.0f, gs);
    const float r6 = __frcp_rn(six_gs);
    const bool fast6 = div_fast_ok(six_gs);
    const uint64_t gs2 = f32x2(gs, gs);
    fill_scale_table(tab, gs);
    if (rank == 0 && threadIdx.x == 0) {
        if (G.gs_out) G.gs_out[b] = gs;
        if (G.amax_out) G.amax_out[b] = A;
    }
    __syncthreads();

    // ---- encode from the registers
#pragma unroll
    for (int k = 0; k < kClusterUnitsPerThread; ++k) {
        const uint32_t r = u0 + threadIdx.x + (uint32_t)k * kThreads;
        if (r < u1) {
            const int i = four_six_member(a, G, r);
            const Sib& S = a.m[i];
            const uint32_t j = r - a.mblk0[i];
            int64_t xo, oo;
            four_six_offsets<kFake>(S, b, j, xo, oo);
            const uint32_t mw = hmax_abs(amax_word8(lo[k]), amax_word8(hi[k])) & 0x7fff7fffu;
            const float amax_b = __uint_as_float(max(mw & 0xffffu, mw >> 16) << 16);
            const float ratio = fast6 ? div_fast(amax_b, six_gs, r6) : div_slow(amax_b, six_gs);
            const uint32_t sb = e4m3x2(ratio, 0.0f) & 0x7fu;   // ratio >= 0
            const float2 e = tab.e[sb];
            const uint32_t c0 = codes_half(lo[k], e.x, e.y), c1 = codes_half(hi[k], e.x, e.y);
            if (kFake) {
                const uint32_t sb2 = e4m3x2_f16x2(sb * 0x101u);
                st_block32(S.out + oo, S.vec32_o, dequant_half_h(c0, sb2, gs2), dequant_half_h(c1, sb2, gs2));
            } else {
                st_v2(S.out + oo, make_uint2(c0, c1));   // 8-byte aligned: 2 j even
                S.sb[(int64_t)b * (S.chunks >> 1) + j] = (uint8_t)sb;
            }
        }
    }
    cluster.barrier_wait();
}

// Dequantise: a grouped walk over 16-element blocks like MXFP8's.  Per
// block: 8 packed bytes in, 32 bytes of BF16 out (one 256-bit store when the
// BF16 rows are 32-byte aligned); the block scale and the batch index's
// global scale are cached loads.  A lane loads kDqUnroll blocks, a warp span
// apart, before storing any: streams that write twice what they read run
// far below the copy rate with 16-byte stores, and 32-byte stores with more
// loads in flight close the gap.
constexpr int kDqUnroll = 8;
constexpr uint32_t kSpan = 32u * kDqUnroll;   // blocks per warp span

struct DqTensor {
    const char* q;        // packed codes
    char* y;              // BF16
    int64_t q_bs, q_rs, y_bs, y_rs;
    const uint8_t* sb;    // dense [B][M][N/16]
    const float* gs;      // [B]
    uint32_t blocks;      // B * M * N / 16
    uint32_t slot_begin;  // multiple of kSpan
    FastDiv bpr;          // blocks per row (N / 16)
    FastDiv per_batch;    // blocks per batch matrix (M * N / 16)
    FastDiv rows;         // M
    int dense;
    int y32;              // BF16 base, row and slab strides multiples of 32 bytes
};

struct DequantArgs {
    DqTensor t[kMaxLaunchTensors];
    int n;
    uint32_t total_slots;
};

__global__ void __launch_bounds__(kThreads) nvfp4_dequant_kernel(const __grid_constant__ DequantArgs a) {
    const uint32_t lane = threadIdx.x & 31u;
    const uint32_t gwarp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const uint32_t nwarps = (gridDim.x * blockDim.x) >> 5;
    for (uint32_t slot = gwarp * kSpan; slot < a.total_slots; slot += nwarps * kSpan) {
        int ti = 0;
        for (int k = 1; k < a.n; ++k)
            if (slot >= a.t[k].slot_begin) ti = k;
        const DqTensor& T = a.t[ti];
        const uint32_t base = slot - T.slot_begin;
        uint2 codes[kDqUnroll];
        uint32_t sbyte[kDqUnroll], bidx[kDqUnroll];
        int64_t yo[kDqUnroll];
#pragma unroll
        for (int u = 0; u < kDqUnroll; ++u) {
            const uint32_t c = base + u * 32u + lane;   // block
            const uint32_t b = fdiv(c, T.per_batch);
            int64_t qo;
            if (T.dense) {
                qo = (int64_t)c * 8;
                yo[u] = (int64_t)c * 32;
            } else {
                const uint32_t r = fdiv(c, T.bpr);          // row over all batches
                const uint32_t k = c - r * T.bpr.d;
                const uint32_t mrow = r - b * T.rows.d;
                qo = (int64_t)b * T.q_bs + (int64_t)mrow * T.q_rs + (int64_t)k * 8;
                yo[u] = (int64_t)b * T.y_bs + (int64_t)mrow * T.y_rs + (int64_t)k * 32;
            }
            bidx[u] = b;
            codes[u] = make_uint2(0u, 0u);
            sbyte[u] = 0u;
            if (c < T.blocks) {
                codes[u] = ld_stream_v2(T.q + qo);
                sbyte[u] = __ldg(T.sb + c);
            }
        }
#pragma unroll
        for (int u = 0; u < kDqUnroll; ++u) {
            const uint32_t c = base + u * 32u + lane;
            if (c >= T.blocks) continue;
            const float gs = __ldg(T.gs + bidx[u]);
            const float sbv = e4m3_decode(sbyte[u]);
            const uint4 y0 = dequant_half(codes[u].x, sbv, gs), y1 = dequant_half(codes[u].y, sbv, gs);
            if (T.y32) {
                st_v8(T.y + yo[u], y0, y1);
            } else {
                st_v4(T.y + yo[u], y0);
                st_v4(T.y + yo[u] + 16, y1);
            }
        }
    }
}

// ---------------------------------------------------------------- single-pass quantise / fake-quantise
//
// One launch covers up to kMaxLaunchTensors members in up to as many sibling
// groups, every batch index of a group being one "instance" with its own
// amax.  The work is a queue of items of one member's batch slab -- 32 KB of
// data, one stage: kItemChunks chunks of BF16, or kItemChunksFp8 chunks of
// E4M3 codes for an FP8 block-wise source, worked in two halves -- amax
// items A(i, k) and encode items E(i, k) of instance i.  The
// encode items of instance i follow its amax items after a lead of L amax
// items of instance i+1 (the order is set out at flow_decode), so that they
// re-read the instance while it is still in L2, and a CTA that takes one
// seldom waits: the lead covers the amax items still in flight.  CTAs take
// items from a global atomic counter.  An encode item waits (bounded) until
// all amax items of its instance are done; those items all sit earlier in
// the queue, were taken by running CTAs that never wait on later items, and
// so finish: there is no deadlock whatever the number of resident CTAs.  An
// amax item publishes its max with atomicMax and then counts itself done
// (fence + atomicAdd); the waiting side reads the count with acquire
// semantics before it reads the amax.
constexpr int kFlowThreads = 256;
constexpr uint32_t kItemChunks = 2048;                        // 16384 elements
constexpr uint32_t kItemChunksFp8 = 2 * kItemChunks;          // FP8 source: 32 KB of codes, two halves
constexpr int kItemChunksPerThread = kItemChunks / kFlowThreads;   // 8
constexpr int kFlowMaxInst = 512;                             // instances per launch
constexpr uint64_t kFlowWaitNs = kFlowWaitLimitNs;             // 2 s
constexpr uint32_t kFlowLeadPerCta = 4;                       // L = kFlowLeadPerCta * grid
constexpr int kFlowStages = 2;
constexpr int kFlowCtasPerSm = 3;
constexpr uint32_t kFlowStageBytes = kItemChunks * 16u;   // 32 KB
constexpr uint32_t kErrFlowTimeout = 2u;

struct FlowMember {
    const char* x;        // BF16, at this launch's first batch index
    int64_t x_bs, x_rs;
    char* out;            // packed codes (quant) or BF16 (fake)
    int64_t o_bs, o_rs;
    uint8_t* sb;          // quant: dense [B][M][N/16], at the first batch index
    uint32_t chunks;      // chunks per batch slab (M * N / 8)
    FastDiv cpr;          // chunks per row
    int dense_x, dense_o;
    uint32_t item_off;    // first item of this member inside an instance
    const float* ts;      // FP8 block-wise source: tile scales [B][TM][TN] at the first batch index
    int64_t ts_bs;        // FP8 source: TM * TN
    uint32_t tn;          // FP8 source: TN
    int vec32_o;          // fake-quant output slab and rows 32-byte aligned
    int sf_mma;           // quant: block scales in the tensor-core tile layout (sf_ct column tiles,
    uint32_t sf_ct;       // sf_slab bytes per batch slab) instead of dense [B][M][N/16]
    int64_t sf_slab;
};

struct FlowGroup {
    int m_begin, m_count;
    uint32_t inst_begin, batch;   // instances [inst_begin, inst_begin + batch)
    uint32_t items;               // items per instance
    uint32_t item_begin;          // items of all instances before inst_begin
    float* gs_out;                // [batch] or null, at the first batch index
    float* amax_out;              // [batch] or null
};

struct FlowArgs {
    FlowMember m[kMaxLaunchTensors];
    FlowGroup g[kMaxLaunchTensors];
    int n_groups;
    uint32_t n_inst;
    uint32_t total_items;         // items per pass (A items = E items)
    uint32_t lead;                // amax items of the next instance between A(i) and E(i)
    uint32_t* amax_bits;          // [n_inst]  (workspace, zeroed before launch)
    uint32_t* done;               // [n_inst]  completed amax items
    uint32_t* counter;            // [1]       queue head
    const uint32_t* wait_done;    // the counts an encode item waits on: done (the self-test
                                  // of the bounded wait points it at counts nothing adds to)
    uint64_t wait_ns;             // limit of that wait (kFlowWaitNs; shorter in the self-test)
};

// The launch description in shared memory, so that the per-item decode and
// the member fields cost shared-memory loads only.
struct FlowTables {
    FlowMember m[kMaxLaunchTensors];
    FlowGroup g[kMaxLaunchTensors];
    uint32_t pa[kFlowMaxInst + 1];   // items before instance i; pa[I] = total
    uint32_t se[kFlowMaxInst];       // queue position of the first encode item of instance i
    uint8_t ig[kFlowMaxInst];        // group of instance i
};

__device__ uint32_t g_flow_error = 0u;

__device__ __forceinline__ uint32_t ld_acquire_gpu(const uint32_t* p) {
    uint32_t v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
// Adds v with release semantics at GPU scope: the thread's earlier writes
// (the amax atomicMax) are visible to whoever reads the sum with acquire.
__device__ __forceinline__ void red_add_release_gpu(uint32_t* p, uint32_t v) {
    asm volatile("red.release.gpu.global.add.u32 [%0], %1;" :: "l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ uint32_t ld_relaxed_gpu(const uint32_t* p) {
    uint32_t v;
    asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ int flow_group_of(const FlowArgs& a, uint32_t inst) {
    int g = 0;
    for (int k = 1; k < a.n_groups; ++k)
        if (inst >= a.g[k].inst_begin) g = k;
    return g;
}

// The queue order.  pa[i] = items before instance i (pa[I] = total), n_i =
// pa[i+1] - pa[i].  The amax items of all instances form one stream, in
// instance order; the encode items of instance i form one block, released
// once the amax stream has gone lead(i) = max(min(n_{i+1}, L), Lmin) items
// past the last amax item of instance i (or reached its end):
//     R(i) = min(pa[i+1] + lead(i), total),   se(i) = pa[i] + R(i)
// is the queue position of E(i)'s first item, and an amax item with stream
// index a sits at a + pa[m], m being the number of encode blocks released
// before it.  With instances of at least Lmin items this reads
//     A(0) H(1) E(0) T(1) H(2) E(1) T(2) ... E(I-1),
// H(j) the first min(n_j, L) amax items of instance j: E(i) re-reads
// instance i while the head of the next instance is read, and the data it
// re-reads was read at most n_i + lead(i) items ago.  Lmin (one item per
// CTA of the grid) matters for small instances: releasing E(i) after the
// few items of a small next instance chained them -- a CTA that claimed an
// encode item ahead of its own amax items of a later instance made that
// instance's encode wait on its encode (64 instances of 8 items took 113
// us against 27 with the minimum lead).
//
// A decoding thread takes positions in increasing order, so it keeps in
// `hint` the last encode block it found (se[hint] <= every later q) and
// steps forward from there; a CTA's consecutive positions are about a grid
// apart, a fraction of an instance of the large workloads, so one or two
// steps usually do, and the binary search runs only after four.
__device__ __forceinline__ void flow_decode(const FlowTables& t, uint32_t I, uint32_t q, uint32_t& hint,
                                            bool& is_e, uint32_t& inst, uint32_t& k) {
    uint32_t a = q, lo = 0;
    if (q >= t.se[0]) {
        lo = hint;
        int fwd = 0;
        while (lo + 1 < I && t.se[lo + 1] <= q && fwd < 4) {
            ++lo;
            ++fwd;
        }
        if (fwd == 4) {
            uint32_t hi = I - 1;
            while (lo < hi) {
                const uint32_t mid = (lo + hi + 1) >> 1;
                if (t.se[mid] <= q) lo = mid; else hi = mid - 1;
            }
        }
        hint = lo;
        if (q < t.se[lo] + (t.pa[lo + 1] - t.pa[lo])) {
            is_e = true;
            inst = lo;
            k = q - t.se[lo];
            return;
        }
        a = q - t.pa[lo + 1];   // the encode items of instances 0..lo precede q
        ++lo;                   // and a >= R(lo) >= pa[lo + 1]
    }
    is_e = false;
    // the instance of amax stream index a: with instances of Lmin items or
    // more it is lo or one of the next two, so a few forward steps find it
    // (a second binary search over hundreds of instances would sit on the
    // decoding thread's path every item); smaller instances fall back to
    // the search
    int steps = 0;
    while (lo + 1 < I && t.pa[lo + 1] <= a && steps < 4) {
        ++lo;
        ++steps;
    }
    if (steps == 4) {
        uint32_t hi = I - 1;
        while (lo < hi) {
            const uint32_t mid = (lo + hi + 1) >> 1;
            if (t.pa[mid] <= a) lo = mid; else hi = mid - 1;
        }
    }
    inst = lo;
    k = a - t.pa[lo];
}

// A decoded queue item.  Thread 0 decodes items kFlowStages ahead of the CTA
// and publishes them in a ring of kFlowStages + 1 slots in shared memory.
struct FlowItem {
    uint32_t valid, is_e, inst, k;   // k: item within its instance's pass (encode: reversed)
    int g, m;                        // group, member
    uint32_t b, c0, c1;              // batch index in the group; chunk range of the member slab
};

__device__ __forceinline__ FlowItem flow_item(const FlowTables& t, uint32_t I, uint32_t total, uint32_t q,
                                              uint32_t& hint, uint32_t chunks) {
    FlowItem it{};
    it.valid = q < 2u * total;
    if (!it.valid) return it;
    bool is_e;
    uint32_t inst, k;
    flow_decode(t, I, q, hint, is_e, inst, k);
    const int g = t.ig[inst];
    const FlowGroup& G = t.g[g];
    if (is_e) k = G.items - 1u - k;                    // encode walks the instance backwards
    int mi = G.m_begin;
    for (int u = 1; u < G.m_count; ++u)
        if (k >= t.m[G.m_begin + u].item_off) mi = G.m_begin + u;
    const FlowMember& M = t.m[mi];
    it.is_e = is_e;
    it.inst = inst;
    it.k = k;
    it.g = g;
    it.m = mi;
    it.b = inst - G.inst_begin;
    it.c0 = (k - M.item_off) * chunks;
    it.c1 = min(it.c0 + chunks, M.chunks);
    return it;
}

// Starts the data of item `it` into stage buffer `dst` (thread 0): one bulk
// copy of the item's contiguous bytes when the member slab is dense,
// otherwise a plain arrival (the item is then read straight from global
// memory), so that every stage completes one barrier phase per item.
__device__ __forceinline__ void flow_stage(const FlowMember& M, const FlowItem& it, uint32_t dst, uint32_t bar,
                                           uint64_t pol) {
    if (M.dense_x) {
        const uint32_t cb = M.ts ? 8u : 16u;   // bytes per 8-element chunk: E4M3 codes or BF16
        const uint32_t bytes = (it.c1 - it.c0) * cb;
        mbar_arrive_expect_tx(bar, bytes);
        bulk_load(dst, M.x + (int64_t)it.b * M.x_bs + (int64_t)it.c0 * cb, bytes, bar, pol);
    } else {
        mbar_arrive(bar);
    }
}

// Chunks of an item taken by thread tid: steps 2i and 2i+1 give the two
// chunks of one 16-element block (first chunk flow_blk(i, tid)), so a thread
// holds whole blocks (no exchange for the block amax, one block scale per 16
// elements).  sw = 1 takes the block's second chunk first: a BF16 stage is
// read with sw = bit 2 of the lane, so that the 8 lanes of each quarter-warp
// (one shared-memory wavefront of 16-byte loads) cover the 32 banks once --
// chunks 32 bytes apart in lane order would put two lanes on every bank.
__device__ __forceinline__ uint32_t flow_blk(int i, uint32_t tid) {
    return (uint32_t)i * (2u * kFlowThreads) + 2u * tid;
}
__device__ __forceinline__ uint32_t flow_lc(int j, uint32_t tid, uint32_t sw) {
    return flow_blk(j >> 1, tid) + ((uint32_t)(j & 1) ^ sw);
}

// Encodes the blocks of one item held in registers.  kFast: every block
// divisor of the instance lies in the reciprocal path's range (checked per
// instance), so no per-block branch; a zero block scale then has d = 0 and a
// zero table reciprocal, for which the reciprocal formula yields the signed
// zero the zero-scale reading asks for.  kFull: all kItemChunks chunks of the
// item exist and both operands are dense.
template <bool kFake, bool kFast, bool kFull>
__device__ __forceinline__ void flow_encode(const uint4 (&v)[kItemChunksPerThread], const FlowItem& it,
                                            const FlowMember& M, const ScaleTable& tab, const DeqTable& dtab,
                                            float gs, float six_gs, float r6, bool fast6, uint64_t pol, uint32_t sw,
                                            uint32_t c_off = 0u) {
    const uint32_t tid = threadIdx.x;
    char* ob = M.out + (int64_t)it.b * M.o_bs;
    uint8_t* sbb = kFake ? nullptr : M.sb + (int64_t)it.b * (M.sf_mma ? M.sf_slab : (int64_t)(M.chunks >> 1));
#pragma unroll
    for (int i = 0; i < kItemChunksPerThread / 2; ++i) {
        const uint4 lo = v[2 * i], hi = v[2 * i + 1];
        // c is even (the block's first chunk); rows hold an even number of
        // chunks, so c + 1 is in the same row and c < c1 implies c + 1 < c1
        const uint32_t c = it.c0 + c_off + flow_blk(i, tid);
        const uint32_t mw = hmax_abs(amax_word8(lo), amax_word8(hi)) & 0x7fff7fffu;
        const float amax_b = __uint_as_float(max(mw & 0xffffu, mw >> 16) << 16);
        float ratio;
        if (kFast)
            ratio = div_fast(amax_b, six_gs, r6);
        else
            ratio = fast6 ? div_fast(amax_b, six_gs, r6) : div_slow(amax_b, six_gs);
        const uint32_t sb = e4m3x2(ratio, 0.0f) & 0x7fu;   // ratio >= 0 (a NaN ratio, outside the contract, stays in the table)
        const float2 e = tab.e[sb];
        uint32_t c0, c1;
        if (kFast) {
            float q[8];
            quotients8<true>(lo, e.x, e.y, q);
            c0 = e2m1x8(q);
            quotients8<true>(hi, e.x, e.y, q);
            c1 = e2m1x8(q);
        } else {
            c0 = codes_half(lo, e.x, e.y);
            c1 = codes_half(hi, e.x, e.y);
        }
        uint4 ya, yb;   // fake, fast: the values of the codes of lo and hi
        if (kFake && kFast) {
            const uint4 tb = dtab.e[sb];
            ya = dequant_lookup8(c0, tb, lo);
            yb = dequant_lookup8(c1, tb, hi);
        }
        if (sw) {   // v[2i] held the block's second chunk
            const uint32_t t = c0;
            c0 = c1;
            c1 = t;
        }
        if (kFull || c < it.c1) {
            int64_t oo;
            if (kFull || M.dense_o) {
                oo = (int64_t)c * (kFake ? 16 : 4);
            } else {
                const uint32_t r = fdiv(c, M.cpr);
                oo = (int64_t)r * M.o_rs + (int64_t)(c - r * M.cpr.d) * (kFake ? 16 : 4);
            }
            if (kFake) {
                uint4 y0, y1;
                if (kFast) {
                    y0 = sw ? yb : ya;
                    y1 = sw ? ya : yb;
                } else {
                    const uint32_t sb2 = e4m3x2_f16x2(sb * 0x101u);
                    const uint64_t gs2 = f32x2(gs, gs);
                    y0 = dequant_half_h(c0, sb2, gs2);
                    y1 = dequant_half_h(c1, sb2, gs2);
                }
                if (M.vec32_o) {
                    st_hint_v8(ob + oo, y0, y1, pol);
                } else {
                    st_hint_v4(ob + oo, y0, pol);
                    st_hint_v4(ob + oo + 16, y1, pol);
                }
            } else {
                st_hint_v2(ob + oo, c0, c1, pol);   // 8-byte aligned: c even, packed rows 8-byte aligned
                if (M.sf_mma) {
                    const uint32_t r = fdiv(c, M.cpr);
                    sbb[mma_scale_offset(r, (c - r * M.cpr.d) >> 1, M.sf_ct)] = (uint8_t)sb;
                } else {
                    sbb[c >> 1] = (uint8_t)sb;
                }
            }
        }
    }
}

// Chunk c of an FP8 block-wise member: the BF16 values of its 8 codes.
__device__ __forceinline__ uint4 flow_fp8_chunk(const FlowMember& M, const FlowItem& it, uint2 codes, uint32_t c) {
    const uint32_t r = fdiv(c, M.cpr);
    const uint32_t k = c - r * M.cpr.d;
    const float s = __ldg(M.ts + (int64_t)it.b * M.ts_bs + (r >> 7) * M.tn + (k >> 4));
    return fp8_dequant8(codes, s);
}

// kFp8: the members are FP8 block-wise (E4M3 codes + tile scales) and the
// values quantised are their dequantised BF16 values.
// L2 policy of an item's staged load: the encode pass streams; of an
// instance's amax items only the last kKeepItems (32 MB of BF16; 16 MB of
// codes for an FP8 block-wise source, whose time does not depend on it;
// those its backward encode walk reaches first) are marked evict-last, the
// earlier ones
// stream like the encode pass: they would be evicted before their encode
// anyway, and as evict-last they pushed out the data the encode pass of the
// previous instance was about to re-read.  Measured (ms per 36-layer sweep,
// quantise / fake-quantise): every amax item kept 2.86 / 3.39, the last
// 3072 items 2.87 / 3.39, 2048 2.82 / 3.33, 1024 2.82 / 3.30, 512 2.82 /
// 3.35, 256 2.82 / 3.46, none 2.95 / 3.50.
constexpr uint32_t kKeepItems = 1024;
__device__ __forceinline__ uint64_t flow_amax_policy(const FlowTables& t, const FlowItem& it, uint64_t keep,
                                                     uint64_t stream) {
    if (it.is_e) return stream;
    return t.g[it.g].items - it.k <= kKeepItems ? keep : stream;
}

template <bool kFake, bool kFp8>
__global__ void __launch_bounds__(kFlowThreads, kFlowCtasPerSm) nvfp4_flow_kernel(const __grid_constant__ FlowArgs a) {
    extern __shared__ __align__(128) unsigned char flow_smem[];
    __shared__ FlowTables t;
    __shared__ ScaleTable tab;
    __shared__ DeqTable dtab;   // fake-quantise only
    __shared__ FlowItem items[kFlowStages + 1];   // item n in slot n % (kFlowStages + 1)
    __shared__ __align__(8) uint64_t bars[kFlowStages];
    __shared__ uint32_t s_amax[2];
    __shared__ uint32_t red[2][kFlowThreads / 32];
    __shared__ uint32_t s_q[kFlowStages + 1];
    // Thread 0 waits for amax values, starts the stage copies and publishes
    // amax runs; thread kQueueThread (another warp) takes queue positions and
    // decodes items, so the two chains overlap within an item.
    constexpr uint32_t kQueueThread = 32;
    // FP8 source: items of two halves of kItemChunks chunks (32 KB of codes)
    constexpr uint32_t kChunks = kFp8 ? kItemChunksFp8 : kItemChunks;
    constexpr int kHalves = kFp8 ? 2 : 1;
    const uint32_t tid = threadIdx.x;
    const uint32_t sw = kFp8 ? 0u : (tid >> 2) & 1u;   // chunk order within a block (flow_lc)
    const uint32_t stage0 = smem_addr(flow_smem);
    const uint32_t I = a.n_inst, L = a.lead, total = a.total_items;

    // the amax pass keeps its data in L2 for the encode pass; the encode
    // pass and every store stream through
    const uint64_t keep = l2_policy_evict_last();
    const uint64_t stream = l2_policy_evict_first();

    for (uint32_t i = tid; i < (uint32_t)kMaxLaunchTensors; i += blockDim.x) {
        t.m[i] = a.m[i];
        t.g[i] = a.g[i];
    }
    for (uint32_t i = tid; i <= I; i += blockDim.x) {
        uint32_t v = total;
        if (i < I) {
            const int g = flow_group_of(a, i);
            const FlowGroup& G = a.g[g];
            v = G.item_begin + (i - G.inst_begin) * G.items;
            t.ig[i] = (uint8_t)g;
        }
        t.pa[i] = v;
    }
    if (tid == 0) {
        for (int s = 0; s < kFlowStages; ++s) mbar_init(smem_addr(&bars[s]), 1);
        fence_mbar_init();
        for (int s = 0; s <= kFlowStages; ++s) s_q[s] = atomicAdd(a.counter, 1u);
    }
    __syncthreads();
    for (uint32_t i = tid; i < I; i += blockDim.x) {
        const uint32_t next_n = i + 1 < I ? t.pa[i + 2] - t.pa[i + 1] : 0u;
        t.se[i] = t.pa[i] + min(t.pa[i + 1] + max(min(next_n, L), gridDim.x), total);
    }
    __syncthreads();
    if (tid == 0) {
        uint32_t hint0 = 0u;
        for (int s = 0; s < kFlowStages; ++s) {
            items[s] = flow_item(t, I, total, s_q[s], hint0, kChunks);
            if (items[s].valid)
                flow_stage(t.m[items[s].m], items[s], stage0 + s * kFlowStageBytes, smem_addr(&bars[s]),
                           flow_amax_policy(t, items[s], keep, stream));
        }
    }
    __syncthreads();
    // thread kQueueThread: queue position of the item kFlowStages ahead
    uint32_t pend = s_q[kFlowStages];
    uint32_t hint = 0u;   // thread kQueueThread: its last encode block (flow_decode)

    uint32_t cached = 0xffffffffu;
    float gs = 0.0f, six_gs = 0.0f, r6 = 0.0f;
    bool fast6 = false, all_fast = false;
    // thread 0: the current run of consecutive amax items of one instance;
    // its max and count are published when the run ends, before the CTA
    // takes any encode item, so no CTA waits while it holds unpublished work
    uint32_t run_max = 0u, run_count = 0u;
    // thread 0: the last instance whose amax this CTA has seen final
    uint32_t known_inst = 0xffffffffu, known_amax = 0u;
    for (uint32_t k = 0;; ++k) {
        const uint32_t slot = k % (kFlowStages + 1u), st = k % kFlowStages, par = (k / kFlowStages) & 1u;
        const uint32_t ahead = (k + kFlowStages) % (kFlowStages + 1u);   // slot of item k + kFlowStages
        const FlowItem it = items[slot];
        if (!it.valid) break;
        uint32_t next_q = 0u;
        if (tid == kQueueThread) next_q = atomicAdd(a.counter, 1u);   // decoded at the next item
        const FlowMember& M = t.m[it.m];

        // ---- the item's data
        if (!mbar_wait_bounded(smem_addr(&bars[st]), par, kFlowWaitNs)) atomicOr(&g_flow_error, kErrFlowTimeout);
        const unsigned char* buf = flow_smem + st * kFlowStageBytes;
        const bool full = (it.c1 - it.c0 == kChunks) && M.dense_x && M.dense_o;
        // the chunks of half h into registers (BF16 values; FP8 codes dequantised)
        auto load_half = [&](int h, uint4 (&v)[kItemChunksPerThread]) {
            const uint32_t hoff = (uint32_t)h * kItemChunks;
            if (full) {
                if (kFp8) {
#pragma unroll
                    for (int j = 0; j < kItemChunksPerThread; j += 2) {
                        // lc even: the block's two chunks lie in one row and one
                        // tile, so one row / column step and one tile-scale load
                        const uint32_t lc = hoff + flow_blk(j >> 1, tid);
                        const uint4 cc = *reinterpret_cast<const uint4*>(buf + lc * 8u);
                        const uint32_t c = it.c0 + lc;
                        const uint32_t r = fdiv(c, M.cpr);
                        const uint32_t k = c - r * M.cpr.d;
                        const float sc = __ldg(M.ts + (int64_t)it.b * M.ts_bs + (r >> 7) * M.tn + (k >> 4));
                        v[j] = fp8_dequant8(make_uint2(cc.x, cc.y), sc);
                        v[j + 1] = fp8_dequant8(make_uint2(cc.z, cc.w), sc);
                    }
                } else {
#pragma unroll
                    for (int j = 0; j < kItemChunksPerThread; ++j)
                        v[j] = *reinterpret_cast<const uint4*>(buf + flow_lc(j, tid, sw) * 16u);
                }
            } else {
                const char* xb = M.x + (int64_t)it.b * M.x_bs;
#pragma unroll
                for (int j = 0; j < kItemChunksPerThread; ++j) {
                    const uint32_t lc = hoff + flow_lc(j, tid, sw);   // chunk within the item
                    const uint32_t c = it.c0 + lc;
                    v[j] = make_uint4(0u, 0u, 0u, 0u);
                    if (c < it.c1) {
                        if (kFp8) {
                            uint2 codes;
                            if (M.dense_x) {
                                codes = *reinterpret_cast<const uint2*>(buf + lc * 8u);
                            } else {
                                const uint32_t r = fdiv(c, M.cpr);
                                codes = ld_stream_v2(xb + (int64_t)r * M.x_rs + (int64_t)(c - r * M.cpr.d) * 8);
                            }
                            v[j] = flow_fp8_chunk(M, it, codes, c);
                        } else if (M.dense_x) {
                            v[j] = *reinterpret_cast<const uint4*>(buf + lc * 16u);
                        } else {
                            const uint32_t r = fdiv(c, M.cpr);
                            v[j] = ld_hint_v4(xb + (int64_t)r * M.x_rs + (int64_t)(c - r * M.cpr.d) * 16,
                                              it.is_e ? stream : keep);
                        }
                    }
                }
            }
        };

        if (!it.is_e) {
            // ---- amax item
            uint32_t m = 0u;
#pragma unroll
            for (int h = 0; h < kHalves; ++h) {
                if (kFp8 && full) {
                    // FP8 source over whole chunk pairs: the block maxima come
                    // from the largest code magnitude of each pair (one tile
                    // scale each), bf16(fl(dec(mc) |s|)) -- rounding is
                    // monotone and symmetric in sign, so that is the largest
                    // |y| of the pair -- without dequantising
#pragma unroll
                    for (int j = 0; j < kItemChunksPerThread; j += 2) {
                        const uint32_t lc = (uint32_t)h * kItemChunks + flow_blk(j >> 1, tid);
                        const uint4 cc = *reinterpret_cast<const uint4*>(buf + lc * 8u);
                        const uint32_t c = it.c0 + lc;
                        const uint32_t r = fdiv(c, M.cpr);
                        const uint32_t k = c - r * M.cpr.d;
                        const float sc = __ldg(M.ts + (int64_t)it.b * M.ts_bs + (r >> 7) * M.tn + (k >> 4));
                        const uint32_t lanes = __vmaxu2(e4m3_maxmag_lanes(make_uint2(cc.x, cc.y)),
                                                        e4m3_maxmag_lanes(make_uint2(cc.z, cc.w)));
                        m = max(m, fp8_amax_bits16(e4m3_maxmag_fin(lanes), sc));
                    }
                } else {
                    uint4 v[kItemChunksPerThread];
                    load_half(h, v);
                    uint32_t mw = 0u;
#pragma unroll
                    for (int j = 0; j < kItemChunksPerThread; ++j) mw = hmax_abs(mw, amax_word8(v[j]));
                    mw &= 0x7fff7fffu;
                    m = max(m, max(mw & 0xffffu, mw >> 16));
                }
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, o));
            if ((tid & 31u) == 0u) red[k & 1u][tid >> 5] = m;
            if (tid == kQueueThread) {
                items[ahead] = flow_item(t, I, total, pend, hint, kChunks);
                pend = next_q;
            }
            __syncthreads();   // stage st is free; red and the new item are published
            if (tid == 0) {
                const FlowItem& nx = items[ahead];
                if (nx.valid)
                    flow_stage(t.m[nx.m], nx, stage0 + st * kFlowStageBytes, smem_addr(&bars[st]),
                               flow_amax_policy(t, nx, keep, stream));
                for (int w = 1; w < kFlowThreads / 32; ++w) m = max(m, red[k & 1u][w]);
                run_max = max(run_max, m);
                ++run_count;
                const FlowItem& nn = items[(k + 1u) % (kFlowStages + 1u)];   // decoded earlier
                if (!nn.valid || nn.is_e || nn.inst != it.inst) {
                    if (run_max != 0u) atomicMax(a.amax_bits + it.inst, run_max << 16);
                    red_add_release_gpu(a.done + it.inst, run_count);   // ordered after the max
                    run_max = 0u;
                    run_count = 0u;
                }
            }
            continue;
        }

        // BF16 source: the item goes to registers and frees its stage at the
        // barrier below; an FP8 item is encoded from the stage, half by half
        uint4 v[kItemChunksPerThread];
        if (!kFp8) load_half(0, v);

        // ---- encode item: wait (bounded) for the instance's amax
        const FlowGroup& G = t.g[it.g];
        if (tid == kQueueThread) {
            items[ahead] = flow_item(t, I, total, pend, hint, kChunks);
            pend = next_q;
        }
        if (tid == 0) {
            if (it.inst != known_inst) {
                if (ld_acquire_gpu(a.wait_done + it.inst) < G.items) {
                    const uint64_t t0 = globaltimer_ns();
                    while (ld_acquire_gpu(a.wait_done + it.inst) < G.items) {
                        if (globaltimer_ns() - t0 > a.wait_ns) {
                            atomicOr(&g_flow_error, kErrFlowTimeout);
                            break;
                        }
                        __nanosleep(100);
                    }
                }
                known_amax = ld_relaxed_gpu(a.amax_bits + it.inst);
                known_inst = it.inst;
            }
            s_amax[k & 1u] = known_amax;
        }
        __syncthreads();   // the amax and the new item are published (BF16: stage st is free)
        if (!kFp8 && tid == 0) {
            const FlowItem& nx = items[ahead];
            if (nx.valid)
                flow_stage(t.m[nx.m], nx, stage0 + st * kFlowStageBytes, smem_addr(&bars[st]),
                           flow_amax_policy(t, nx, keep, stream));
        }
        if (it.inst != cached) {   // CTA-uniform
            gs = __fdiv_rn(__uint_as_float(s_amax[k & 1u]), 2688.0f);
            six_gs = __fmul_rn(6.0f, gs);
            r6 = __frcp_rn(six_gs);
            fast6 = div_fast_ok(six_gs);
            // every non-zero block scale gives dec(sb) * gs in [2^-9 gs, 448 gs]
            all_fast = fast6 && __fmul_rn(0x1p-9f, gs) >= 0x1p-64f && __fmul_rn(448.0f, gs) <= 0x1p126f;
            fill_scale_table(tab, gs);
            if (kFake) fill_deq_table(dtab, f32x2(gs, gs));
            __syncthreads();
            cached = it.inst;
        }
        if (tid == 0 && it.k == 0u) {
            if (G.gs_out) G.gs_out[it.b] = gs;
            if (G.amax_out) G.amax_out[it.b] = __uint_as_float(s_amax[k & 1u]);
        }
        if (!kFp8) {
            if (all_fast && full)
                flow_encode<kFake, true, true>(v, it, M, tab, dtab, gs, six_gs, r6, fast6, stream, sw);
            else
                flow_encode<kFake, false, false>(v, it, M, tab, dtab, gs, six_gs, r6, fast6, stream, sw);
        } else {
#pragma unroll 1
            for (int h = 0; h < kHalves; ++h) {
                load_half(h, v);
                if (all_fast && full)
                    flow_encode<kFake, true, true>(v, it, M, tab, dtab, gs, six_gs, r6, fast6, stream, sw,
                                                   (uint32_t)h * kItemChunks);
                else
                    flow_encode<kFake, false, false>(v, it, M, tab, dtab, gs, six_gs, r6, fast6, stream, sw,
                                                     (uint32_t)h * kItemChunks);
            }
            __syncthreads();   // stage st is free
            if (tid == 0) {
                const FlowItem& nx = items[ahead];
                if (nx.valid)
                    flow_stage(t.m[nx.m], nx, stage0 + st * kFlowStageBytes, smem_addr(&bars[st]),
                               flow_amax_policy(t, nx, keep, stream));
            }
        }
    }
}


bool dense_rows(const View& v, int64_t row_bytes) {
    return v.rstride == row_bytes;
}

// BF16 source (ts null) or E4M3 codes with tile scales ts [B][TM][TN].
void set_source(Sib& S, const View& x, const float* ts) {
    S.ts = ts;
    S.tn = (uint32_t)((x.cols + 127) / 128);
    S.ts_bs = (int64_t)((x.rows + 127) / 128) * S.tn;
    S.dense_x = dense_rows(x, ts ? x.cols : x.cols * 2);
}

}  // namespace

cudaError_t launch_nvfp4_amax(const View* x, int n, uint32_t* amax_bits, cudaStream_t s, const float* const* ts) {
    const int64_t B = x[0].batch;
    cudaError_t err = cudaMemsetAsync(amax_bits, 0, sizeof(uint32_t) * B, s);
    if (err != cudaSuccess) return err;
    AmaxArgs a{};
    a.n = n;
    a.amax_bits = amax_bits;
    int64_t max_chunks = 0;
    for (int i = 0; i < n; ++i) {
        Sib& S = a.s[i];
        S.x = x[i].ptr;
        S.x_bs = x[i].bstride;
        S.x_rs = x[i].rstride;
        S.chunks = (uint32_t)(x[i].rows * (x[i].cols / 8));
        S.cpr = make_fastdiv((uint32_t)std::max<int64_t>(1, x[i].cols / 8));
        set_source(S, x[i], ts ? ts[i] : nullptr);
        max_chunks = std::max<int64_t>(max_chunks, S.chunks);
    }
    const int64_t total_ctas = (max_chunks + int64_t(kThreads) * kUnroll - 1) / (int64_t(kThreads) * kUnroll);
    // spread about 4 resident CTAs per SM over all groups
    const int64_t budget = (int64_t)sm_count(current_device()) * 4;
    int gx = (int)std::max<int64_t>(1, std::min<int64_t>(total_ctas, (budget + B - 1) / B));
    dim3 grid(gx, (unsigned)B);
    if (ts)
        nvfp4_amax_kernel<true><<<grid, kThreads, 0, s>>>(a);
    else
        nvfp4_amax_kernel<false><<<grid, kThreads, 0, s>>>(a);
    return cudaGetLastError();
}

size_t nvfp4_4over6_workspace_bytes(int64_t instances) {
    return (size_t)((std::max<int64_t>(1, instances) * 4 + 255) / 256 * 256);
}

namespace {

// Cuts a list of NVFP4 groups into launches over the unit space (at most
// kMaxLaunchTensors members and groups each) and calls run(args) for each.
// Instance words (amax_bits) are numbered across the whole call.
template <typename Run>
cudaError_t for_unit_launches(const NvGroup* groups, int n_groups, bool fake, uint32_t* words, float six_e,
                              Run run) {
    FourSixArgs a{};
    uint32_t inst = 0;   // amax words used by earlier groups of the call
    int n_members = 0;
    for (int gi = 0; gi < n_groups; ++gi) {
        const NvGroup& G = groups[gi];
        if (n_members + G.n > kMaxLaunchTensors || a.n_groups == kMaxLaunchTensors) {
            cudaError_t e = run(a);
            if (e != cudaSuccess) return e;
            a = FourSixArgs{};
            n_members = 0;
        }
        a.amax_bits = words;
        a.six_e = six_e;
        FourSixGroup& F = a.g[a.n_groups];
        F.unit0 = a.total;
        F.inst0 = inst;
        F.batch = (uint32_t)G.x[0].batch;
        F.m0 = n_members;
        F.nm = G.n;
        F.amax_in = G.amax_in;
        F.gs_out = G.gs_out;
        F.amax_out = G.amax_out;
        uint64_t units = 0;
        for (int i = 0; i < G.n; ++i) {
            Sib& S = a.m[n_members + i];
            const View& x = G.x[i];
            const View& o = G.out[i];
            S.x = x.ptr;
            S.x_bs = x.bstride;
            S.x_rs = x.rstride;
            S.out = o.ptr;
            S.o_bs = o.bstride;
            S.o_rs = o.rstride;
            S.sb = fake ? nullptr : G.sb[i];
            S.chunks = (uint32_t)(x.rows * (x.cols / 8));
            S.cpr = make_fastdiv((uint32_t)std::max<int64_t>(1, x.cols / 8));
            set_source(S, x, G.ts ? G.ts[i] : nullptr);
            S.dense_o = dense_rows(o, fake ? o.cols * 2 : o.cols / 2);
            S.vec16_x = (uintptr_t)x.ptr % 16 == 0 && (x.rows <= 1 || x.rstride % 16 == 0) &&
                        (x.batch <= 1 || x.bstride % 16 == 0);
            S.vec32_x = !G.ts && (uintptr_t)x.ptr % 32 == 0 && (x.rows <= 1 || x.rstride % 32 == 0) &&
                        (x.batch <= 1 || x.bstride % 32 == 0);
            S.vec32_o = fake && (uintptr_t)o.ptr % 32 == 0 && (o.rows <= 1 || o.rstride % 32 == 0) &&
                        (o.batch <= 1 || o.bstride % 32 == 0);
            a.mblk0[n_members + i] = (uint32_t)units;
            units += S.chunks / 2;
        }
        if (units == 0) continue;                               // an empty group: nothing to launch
        if (units > UINT32_MAX) return cudaErrorInvalidValue;   // more than 2^32 blocks per instance
        F.units = (uint32_t)units;
        a.total += units * F.batch;
        inst += F.batch;
        n_members += G.n;
        ++a.n_groups;
    }
    return a.n_groups ? run(a) : cudaSuccess;
}

int unit_grid(const FourSixArgs& a, int ctas_per_sm = kFourSixCtasPerSm) {
    const int cap = sm_count(current_device()) * ctas_per_sm;
    return (int)std::max<int64_t>(1, std::min<int64_t>(cap, (int64_t)((a.total + kThreads - 1) / kThreads)));
}

}  // namespace

cudaError_t launch_nvfp4_4over6(const NvGroup* groups, int n_groups, bool fake, int e4m3_max, void* workspace,
                               cudaStream_t s) {
    uint32_t* words = static_cast<uint32_t*>(workspace);
    return for_unit_launches(groups, n_groups, fake, words, (float)(6 * e4m3_max), [&](const FourSixArgs& a) {
        const int grid = unit_grid(a);
        bool reduce = false;
        uint32_t w0 = UINT32_MAX, w1 = 0;
        for (int g = 0; g < a.n_groups; ++g)
            if (!a.g[g].amax_in) {
                reduce = true;
                w0 = std::min(w0, a.g[g].inst0);
                w1 = std::max(w1, a.g[g].inst0 + a.g[g].batch);
            }
        if (reduce) {
            cudaError_t e = cudaMemsetAsync(words + w0, 0, sizeof(uint32_t) * (w1 - w0), s);
            if (e != cudaSuccess) return e;
            nvfp4_4over6_amax_kernel<<<grid, kThreads, 0, s>>>(a);
            if ((e = cudaGetLastError()) != cudaSuccess) return e;
        }
        if (fake)
            nvfp4_4over6_kernel<true><<<grid, kThreads, 0, s>>>(a);
        else
            nvfp4_4over6_kernel<false><<<grid, kThreads, 0, s>>>(a);
        return cudaGetLastError();
    });
}

cudaError_t launch_nvfp4_units_encode(const NvGroup* groups, int n_groups, bool fake, const uint32_t* amax_bits,
                                      cudaStream_t s) {
    const bool fp8 = n_groups > 0 && groups[0].ts != nullptr;   // every group of a call has the same source
    return for_unit_launches(groups, n_groups, fake, const_cast<uint32_t*>(amax_bits), 2688.0f,
                             [&](const FourSixArgs& a) {
                                 const int grid = unit_grid(a, kUnitCtasPerSm);
                                 if (fp8)
                                     nvfp4_units_kernel<false, true><<<grid, kThreads, 0, s>>>(a);
                                 else if (fake)
                                     nvfp4_units_kernel<true, false><<<grid, kThreads, 0, s>>>(a);
                                 else
                                     nvfp4_units_kernel<false, false><<<grid, kThreads, 0, s>>>(a);
                                 return cudaGetLastError();
                             });
}

bool nvfp4_cluster_ok(const NvGroup* groups, int n_groups) {
    for (int gi = 0; gi < n_groups; ++gi) {
        const NvGroup& G = groups[gi];
        if (G.sb_mma || G.ts) return false;
        int64_t units = 0;
        for (int i = 0; i < G.n; ++i) units += G.x[i].rows * (G.x[i].cols / 16);
        if (units > (int64_t)kClusterUnits) return false;
    }
    return true;
}

cudaError_t launch_nvfp4_cluster(const NvGroup* groups, int n_groups, bool fake, cudaStream_t s) {
    FourSixArgs a{};
    uint32_t max_units = 0;
    int n_members = 0;
    auto flush = [&]() -> cudaError_t {
        if (a.n_groups == 0) return cudaSuccess;
        const uint32_t n_inst = a.g[a.n_groups - 1].inst0 + a.g[a.n_groups - 1].batch;
        const uint32_t cs = std::max<uint32_t>(1, (max_units + kClusterCtaUnits - 1) / kClusterCtaUnits);
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(n_inst * cs);
        cfg.blockDim = dim3(kThreads);
        cfg.stream = s;
        cudaLaunchAttribute at[1];
        at[0].id = cudaLaunchAttributeClusterDimension;
        at[0].val.clusterDim.x = cs;
        at[0].val.clusterDim.y = 1;
        at[0].val.clusterDim.z = 1;
        cfg.attrs = at;
        cfg.numAttrs = 1;
        cudaError_t e = fake ? cudaLaunchKernelEx(&cfg, nvfp4_cluster_kernel<true>, a)
                             : cudaLaunchKernelEx(&cfg, nvfp4_cluster_kernel<false>, a);
        a = FourSixArgs{};
        max_units = 0;
        n_members = 0;
        return e;
    };
    for (int gi = 0; gi < n_groups; ++gi) {
        const NvGroup& G = groups[gi];
        for (int64_t b0 = 0; b0 < G.x[0].batch;) {
            if (n_members + G.n > kMaxLaunchTensors || a.n_groups == kMaxLaunchTensors) {
                cudaError_t e = flush();
                if (e != cudaSuccess) return e;
            }
            // at most 2^16 instances per launch keep the grid within range
            const uint32_t inst0 = a.n_groups ? a.g[a.n_groups - 1].inst0 + a.g[a.n_groups - 1].batch : 0u;
            const uint32_t nb = (uint32_t)std::min<int64_t>(G.x[0].batch - b0, 65536 - (int64_t)inst0);
            if (nb == 0) {
                cudaError_t e = flush();
                if (e != cudaSuccess) return e;
                continue;
            }
            FourSixGroup& F = a.g[a.n_groups];
            F.unit0 = 0;
            F.inst0 = inst0;
            F.batch = nb;
            F.m0 = n_members;
            F.nm = G.n;
            F.amax_in = G.amax_in ? G.amax_in + b0 : nullptr;
            F.gs_out = G.gs_out ? G.gs_out + b0 : nullptr;
            F.amax_out = G.amax_out ? G.amax_out + b0 : nullptr;
            uint32_t units = 0;
            for (int i = 0; i < G.n; ++i) {
                Sib& S = a.m[n_members + i];
                const View& x = G.x[i];
                const View& o = G.out[i];
                S.x = x.ptr + b0 * x.bstride;
                S.x_bs = x.bstride;
                S.x_rs = x.rstride;
                S.out = o.ptr + b0 * o.bstride;
                S.o_bs = o.bstride;
                S.o_rs = o.rstride;
                S.chunks = (uint32_t)(x.rows * (x.cols / 8));
                S.sb = fake ? nullptr : G.sb[i] + b0 * (int64_t)(S.chunks / 2);
                S.cpr = make_fastdiv((uint32_t)std::max<int64_t>(1, x.cols / 8));
                set_source(S, x, nullptr);
                S.dense_o = dense_rows(o, fake ? o.cols * 2 : o.cols / 2);
                a.mblk0[n_members + i] = units;
                units += S.chunks / 2;
            }
            b0 += nb;
            F.units = units;
            max_units = std::max(max_units, units);
            n_members += G.n;
            ++a.n_groups;
        }
    }
    return flush();
}

cudaError_t launch_nvfp4_dequant(const Job* jobs, int n, cudaStream_t s) {
    const uint64_t kMaxSlots = uint64_t(1) << 31;   // chunk indices stay 32-bit
    for (int j0 = 0; j0 < n;) {
        DequantArgs a;
        a.n = 0;
        uint32_t slots = 0;
        for (; j0 + a.n < n && a.n < kMaxLaunchTensors; ++a.n) {
            const Job& j = jobs[j0 + a.n];
            const View& q = j.in;
            const View& y = j.out;
            const uint64_t blocks = (uint64_t)(q.batch * q.rows * (q.cols / 16));
            const uint64_t padded = (blocks + kSpan - 1) / kSpan * kSpan;
            if (a.n > 0 && slots + padded > kMaxSlots) break;
            DqTensor& T = a.t[a.n];
            T.q = q.ptr;
            T.y = y.ptr;
            T.q_bs = q.bstride;
            T.q_rs = q.rstride;
            T.y_bs = y.bstride;
            T.y_rs = y.rstride;
            T.sb = static_cast<const uint8_t*>(j.scale);
            T.gs = j.gs;
            T.blocks = (uint32_t)blocks;
            T.slot_begin = slots;
            const int64_t bpr = std::max<int64_t>(1, q.cols / 16);
            T.bpr = make_fastdiv((uint32_t)bpr);
            T.per_batch = make_fastdiv((uint32_t)std::max<int64_t>(1, q.rows * bpr));
            T.rows = make_fastdiv((uint32_t)std::max<int64_t>(1, q.rows));
            T.dense = q.rstride == q.cols / 2 && y.rstride == y.cols * 2 &&
                      (q.batch == 1 || (q.bstride == q.rows * q.rstride && y.bstride == y.rows * y.rstride));
            T.y32 = (uintptr_t)y.ptr % 32 == 0 && y.rstride % 32 == 0 && (y.batch == 1 || y.bstride % 32 == 0);
            slots += (uint32_t)padded;
        }
        j0 += a.n;
        a.total_slots = slots;
        if (slots == 0) continue;
        const int grid = persistent_grid((slots + kThreads * kDqUnroll - 1) / (kThreads * kDqUnroll), 8);
        nvfp4_dequant_kernel<<<grid, kThreads, 0, s>>>(a);
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

cudaError_t read_and_clear_flow_error(uint32_t* code) {
    uint32_t zero = 0u;
    cudaError_t e = cudaMemcpyFromSymbol(code, g_flow_error, sizeof(uint32_t));
    if (e != cudaSuccess) return e;
    return cudaMemcpyToSymbol(g_flow_error, &zero, sizeof(uint32_t));
}

size_t nvfp4_flow_workspace_bytes(int64_t instances) {
    const int64_t per = std::max<int64_t>(1, std::min<int64_t>(instances, kFlowMaxInst));
    return (size_t)((2 * per + 1) * 4 + 255) / 256 * 256;
}

size_t nvfp4_flow_timeout_selftest_bytes(int64_t instances) {
    const int64_t per = std::max<int64_t>(1, std::min<int64_t>(instances, kFlowMaxInst));
    return (size_t)((3 * per + 1) * 4 + 255) / 256 * 256;
}

cudaError_t launch_nvfp4_flow(const NvGroup* groups, int n_groups, bool fake, void* workspace, cudaStream_t s,
                              uint64_t wait_ns, bool wait_on_idle_counts) {
    const bool fp8 = n_groups > 0 && groups[0].ts != nullptr;   // every group of a call has the same source
    const uint32_t item_chunks = fp8 ? kItemChunksFp8 : kItemChunks;
    uint32_t* words = static_cast<uint32_t*>(workspace);
    const uint64_t kMaxItems = uint64_t(1) << 30;   // queue positions (2 per item) stay 32-bit
    FlowArgs a;
    int n_members = 0;
    auto reset = [&]() {
        a.n_groups = 0;
        a.n_inst = 0;
        a.total_items = 0;
        n_members = 0;
    };
    auto flush = [&]() -> cudaError_t {
        if (a.n_groups == 0) return cudaSuccess;
        a.amax_bits = words;
        a.done = words + a.n_inst;
        a.counter = words + 2 * a.n_inst;
        // the self-test's encode items wait on n_inst zeroed words that no
        // amax item adds to, so every such wait runs out after wait_ns
        a.wait_done = wait_on_idle_counts ? words + 2 * a.n_inst + 1 : a.done;
        a.wait_ns = wait_ns;
        const size_t words_used = (size_t)((wait_on_idle_counts ? 3 : 2) * a.n_inst + 1);
        cudaError_t e = cudaMemsetAsync(words, 0, words_used * 4, s);
        if (e != cudaSuccess) return e;
        const int dev = current_device();
        const size_t smem = (size_t)kFlowStages * kFlowStageBytes;
        static int configured[kMaxDevices] = {0};
        const void* fns[4] = {(const void*)nvfp4_flow_kernel<true, false>, (const void*)nvfp4_flow_kernel<false, false>,
                              (const void*)nvfp4_flow_kernel<true, true>, (const void*)nvfp4_flow_kernel<false, true>};
        e = set_smem_limit_once(configured, fns, 4, (int)smem);
        if (e != cudaSuccess) return e;
        const int grid = (int)std::max<int64_t>(
            1, std::min<int64_t>((int64_t)sm_count(dev) * kFlowCtasPerSm, 2 * (int64_t)a.total_items));
        a.lead = kFlowLeadPerCta * (uint32_t)grid;
        if (fp8)
            fake ? nvfp4_flow_kernel<true, true><<<grid, kFlowThreads, smem, s>>>(a)
                 : nvfp4_flow_kernel<false, true><<<grid, kFlowThreads, smem, s>>>(a);
        else
            fake ? nvfp4_flow_kernel<true, false><<<grid, kFlowThreads, smem, s>>>(a)
                 : nvfp4_flow_kernel<false, false><<<grid, kFlowThreads, smem, s>>>(a);
        e = cudaGetLastError();
        reset();
        return e;
    };
    reset();
    for (int gi = 0; gi < n_groups; ++gi) {
        const NvGroup& G = groups[gi];
        const int64_t B = G.x[0].batch;
        uint32_t items = 0;
        for (int i = 0; i < G.n; ++i)
            items += (uint32_t)((G.x[i].rows * (G.x[i].cols / 8) + item_chunks - 1) / item_chunks);
        if (items == 0 || B == 0) continue;
        for (int64_t b0 = 0; b0 < B;) {
            const int64_t room_inst = kFlowMaxInst - (int64_t)a.n_inst;
            const int64_t room_items = (int64_t)(kMaxItems - a.total_items) / items;
            if (n_members + G.n > kMaxLaunchTensors || a.n_groups == kMaxLaunchTensors || room_inst < 1 ||
                room_items < 1) {
                cudaError_t e = flush();
                if (e != cudaSuccess) return e;
                continue;
            }
            const int64_t take = std::min<int64_t>({B - b0, room_inst, room_items});
            FlowGroup& F = a.g[a.n_groups++];
            F.m_begin = n_members;
            F.m_count = G.n;
            F.inst_begin = a.n_inst;
            F.batch = (uint32_t)take;
            F.items = items;
            F.item_begin = a.total_items;
            F.gs_out = G.gs_out ? G.gs_out + b0 : nullptr;
            F.amax_out = G.amax_out ? G.amax_out + b0 : nullptr;
            uint32_t off = 0;
            for (int i = 0; i < G.n; ++i) {
                const View& x = G.x[i];
                const View& o = G.out[i];
                FlowMember& M = a.m[n_members++];
                M.x = x.ptr + b0 * x.bstride;
                M.x_bs = x.bstride;
                M.x_rs = x.rstride;
                M.out = o.ptr + b0 * o.bstride;
                M.o_bs = o.bstride;
                M.o_rs = o.rstride;
                M.chunks = (uint32_t)(x.rows * (x.cols / 8));
                M.sf_mma = G.sb_mma;
                M.sf_ct = (uint32_t)mma_scale_col_tiles(x.cols / 16);
                M.sf_slab = mma_scale_slab_bytes(x.rows, x.cols / 16);
                M.sb = fake ? nullptr : G.sb[i] + b0 * (G.sb_mma ? M.sf_slab : (int64_t)(M.chunks / 2));
                M.cpr = make_fastdiv((uint32_t)std::max<int64_t>(1, x.cols / 8));
                // the stage copy of a dense slab needs 16-byte aligned addresses;
                // E4M3 code tensors are only checked to 8 bytes, so such a
                // member is read row by row with 8-byte loads instead
                M.dense_x = dense_rows(x, fp8 ? x.cols : x.cols * 2) &&
                            (!fp8 || ((uintptr_t)M.x % 16 == 0 && (take == 1 || x.bstride % 16 == 0)));
                M.dense_o = dense_rows(o, fake ? o.cols * 2 : o.cols / 2);
                M.tn = (uint32_t)((x.cols + 127) / 128);
                M.ts_bs = (int64_t)((x.rows + 127) / 128) * M.tn;
                M.ts = fp8 ? G.ts[i] + b0 * M.ts_bs : nullptr;
                M.item_off = off;
                off += (M.chunks + item_chunks - 1) / item_chunks;
                M.vec32_o = (uintptr_t)M.out % 32 == 0 && o.rstride % 32 == 0 &&
                            (take == 1 || o.bstride % 32 == 0);
            }
            a.n_inst += (uint32_t)take;
            a.total_items += (uint32_t)take * items;
            b0 += take;
        }
    }
    return flush();
}

// ---------------------------------------------------------------- scratch for callers that cannot allocate

// Group-amax scratch of nvfp4_fake_quant_noalloc: one word per group, in a
// file-scope device array.  Every device that loads the library holds these
// kStaticScratchGroups * 4 bytes until the process exits.
__device__ __align__(256) uint32_t g_static_amax[kStaticScratchGroups];

cudaError_t static_amax_scratch(uint32_t** ptr) {
    // In host code g_static_amax names a host-side stand-in, not the device
    // array: the device address is looked up once per device, with that
    // device current, and cached.
    static uint32_t* addr[kMaxDevices] = {};
    static std::mutex mu;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(mu);
    if (addr[dev] == nullptr) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_static_amax);
        if (e != cudaSuccess) return e;
        addr[dev] = static_cast<uint32_t*>(p);
    }
    *ptr = addr[dev];
    return cudaSuccess;
}

}  // namespace pwq
