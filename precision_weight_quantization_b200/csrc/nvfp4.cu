// nvfp4.cu -- NVFP4 (E2M1 codes, 1x16 blocks, E4M3 block scale, FP32 global
// scale) group amax, quantise, fake-quantise and dequantise.
// Source: verl NVFP4 QAT article, section 2.3 (global scale =
// amax / (6 * 448), E4M3 block scale per 16 elements, nearest E2M1 value on
// {0, 0.5, 1, 1.5, 2, 3, 4, 6}, multiply back), 2.4 (q/k/v and gate/up
// siblings share the group's maximum amax), 3.3 (weight_scale_2 =
// amax / (6.0 * 448.0)); "Low Precision RL", "Choose a precision" table.
//
// Two stream-ordered passes, no device-side waiting:
//   1. amax: every CTA reduces a slice of one group to a max and publishes
//      it with one atomicMax on the group's word (the float bit patterns of
//      non-negative values order like unsigned integers);
//   2. encode: every CTA reads its group's amax, forms the global scale and
//      quantises 16-element blocks held by lane pairs (8 elements, one
//      128-bit load each, amax combined with one shuffle).  It walks the
//      tensor in the reverse order of pass 1 so that the most recently read
//      data -- still in the 126 MB L2 -- is consumed first.
// Division: a group has at most 127 distinct code divisors d = fl(dec(sb) *
// gs), so each CTA tabulates d and RN(1/d) for every block-scale code in
// shared memory once; the block scale itself divides by fl(6 gs), whose
// reciprocal is also formed once.  Per element the quotient is the
// reciprocal product plus one FMA residual correction (pwq_device.cuh),
// which the self-test proves to give IEEE division's codes over every BF16
// numerator and every reachable divisor.
#include <algorithm>
#include <mutex>

#include "pwq_internal.h"

namespace pwq {
namespace {

constexpr int kThreads = 256;
constexpr int kUnroll = 4;
constexpr int kMaxSib = 8;

// One sibling of a group set, addressed per batch slab.
struct Sib {
    const char* x;        // BF16
    int64_t x_bs, x_rs;   // bytes
    char* out;            // packed codes (quant) or BF16 (fake); unused by amax
    int64_t o_bs, o_rs;   // bytes
    uint8_t* sb;          // dense [B][M][N/16] (quant only)
    uint32_t chunks;      // 8-element chunks per batch slab (M * N / 8)
    FastDiv cpr;          // chunks per row (N / 8)
    int dense_x, dense_o; // slab rows are contiguous
};

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

__global__ void __launch_bounds__(kThreads) nvfp4_amax_kernel(const AmaxArgs a) {
    const uint32_t b = blockIdx.y;
    const uint32_t stride = gridDim.x * blockDim.x;
    const uint32_t t0 = blockIdx.x * blockDim.x + threadIdx.x;
    uint32_t m = 0u;
    for (int i = 0; i < a.n; ++i) {
        const Sib& S = a.s[i];
        const char* base = S.x + (int64_t)b * S.x_bs;
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
    m = block_max_u32(m);
    if (threadIdx.x == 0 && m != 0u) atomicMax(a.amax_bits + b, m << 16);
}

struct EncodeArgs {
    Sib s[kMaxSib];
    int n;
    const uint32_t* amax_bits;  // [B] or null
    const float* amax_in;       // [B] or null (takes precedence)
    float* gs_out;              // [B] or null
    float* amax_out;            // [B] or null
};

// Per-group constants of the encode pass, for every E4M3 block-scale code
// k: d_k = fl(dec(k) * gs) (the code divisor), r_k = RN(1/d_k) when d_k is
// in the reciprocal path's range (else 0: IEEE division), and dec(k).
struct ScaleTable {
    float4 e[128];
};

__device__ __forceinline__ void fill_scale_table(ScaleTable& t, float gs) {
    for (uint32_t k = threadIdx.x; k < 128u; k += blockDim.x) {
        const float dec = e4m3_decode(k);  // k = 0x7f (NaN) is never produced
        const float d = __fmul_rn(dec, gs);
        t.e[k] = make_float4(d, div_fast_ok(d) ? __frcp_rn(d) : 0.0f, dec, 0.0f);
    }
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

template <bool kFake>
__global__ void __launch_bounds__(kThreads) nvfp4_encode_kernel(const EncodeArgs a) {
    __shared__ ScaleTable tab;
    const uint32_t b = blockIdx.y;
    const float A = a.amax_in ? a.amax_in[b] : __uint_as_float(a.amax_bits[b]);
    const float gs = __fdiv_rn(A, 2688.0f);
    const float six_gs = __fmul_rn(6.0f, gs);
    const float r6 = __frcp_rn(six_gs);
    const bool fast6 = div_fast_ok(six_gs);
    fill_scale_table(tab, gs);
    if (blockIdx.x == 0 && threadIdx.x == 0) {
        if (a.gs_out) a.gs_out[b] = gs;
        if (a.amax_out) a.amax_out[b] = A;
    }
    __syncthreads();
    const uint32_t lane = threadIdx.x & 31u;
    const uint32_t gwarp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const uint32_t nwarps = (gridDim.x * blockDim.x) >> 5;
    // Reverse order: last sibling first, each walked from its end.
    for (int i = a.n - 1; i >= 0; --i) {
        const Sib& S = a.s[i];
        const char* xb = S.x + (int64_t)b * S.x_bs;
        char* ob = S.out + (int64_t)b * S.o_bs;
        uint8_t* sbb = kFake ? nullptr : S.sb + (int64_t)b * (S.chunks >> 1);
        for (uint32_t base = gwarp * 32u * kUnroll; base < S.chunks; base += nwarps * 32u * kUnroll) {
            uint4 v[kUnroll];
            uint32_t cc[kUnroll];
#pragma unroll
            for (int u = 0; u < kUnroll; ++u) {
                const uint32_t j = base + u * 32u + lane;
                // lanes 2k and 2k+1 take the high and low halves of one block
                cc[u] = S.chunks - 1u - j;
                v[u] = make_uint4(0u, 0u, 0u, 0u);
                if (j < S.chunks) {
                    int64_t off;
                    if (S.dense_x) {
                        off = (int64_t)cc[u] * 16;
                    } else {
                        const uint32_t r = fdiv(cc[u], S.cpr);
                        off = (int64_t)r * S.x_rs + (int64_t)(cc[u] - r * S.cpr.d) * 16;
                    }
                    v[u] = ld_stream_v4(xb + off);
                }
            }
#pragma unroll
            for (int u = 0; u < kUnroll; ++u) {
                const uint32_t j = base + u * 32u + lane;
                uint32_t m = amax_bits8(v[u]);
                m = max(m, __shfl_xor_sync(0xffffffffu, m, 1));
                // block scale sb = e4m3(fl(amax_b / fl(6 gs)))
                const float amax_b = __uint_as_float(m << 16);
                const float ratio = fast6 ? div_fast(amax_b, six_gs, r6) : div_slow(amax_b, six_gs);
                const uint32_t sb = e4m3x2(ratio, 0.0f) & 0xffu;
                const float4 e = tab.e[sb];
                const uint32_t codes = codes_half(v[u], e.x, e.y);
                if (j < S.chunks) {
                    const uint32_t c = cc[u];
                    int64_t oo;
                    if (S.dense_o) {
                        oo = (int64_t)c * (kFake ? 16 : 4);
                    } else {
                        const uint32_t r = fdiv(c, S.cpr);
                        oo = (int64_t)r * S.o_rs + (int64_t)(c - r * S.cpr.d) * (kFake ? 16 : 4);
                    }
                    if (kFake) {
                        st_v4(ob + oo, dequant_half(codes, e.z, gs));
                    } else {
                        st_u32(ob + oo, codes);
                        if ((c & 1u) == 0u) sbb[c >> 1] = (uint8_t)sb;
                    }
                }
            }
        }
    }
}

struct DequantArgs {
    const char* q;        // packed codes
    char* y;              // BF16
    const uint8_t* sb;    // dense [B][M][N/16]
    const float* gs;      // [B]
    int64_t q_bs, q_rs, y_bs, y_rs;
    FastDiv cpr;          // chunks per row (N / 8)
    FastDiv per_batch;    // chunks per batch slab (M * N / 8)
    FastDiv rows;         // M
    uint32_t total;
    int dense;
};

__global__ void __launch_bounds__(kThreads) nvfp4_dequant_kernel(const DequantArgs a) {
    const uint32_t stride = gridDim.x * blockDim.x;
    for (uint32_t base = blockIdx.x * blockDim.x + threadIdx.x; base < a.total;
         base += stride * kUnroll) {
        uint32_t codes[kUnroll], sbyte[kUnroll], bidx[kUnroll];
        int64_t yo[kUnroll];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const uint32_t c = base + u * stride;
            const uint32_t b = fdiv(c, a.per_batch);
            int64_t qo;
            if (a.dense) {
                qo = (int64_t)c * 4;
                yo[u] = (int64_t)c * 16;
            } else {
                const uint32_t r = fdiv(c, a.cpr);          // global row
                const uint32_t k = c - r * a.cpr.d;
                const uint32_t mrow = r - b * a.rows.d;
                qo = (int64_t)b * a.q_bs + (int64_t)mrow * a.q_rs + (int64_t)k * 4;
                yo[u] = (int64_t)b * a.y_bs + (int64_t)mrow * a.y_rs + (int64_t)k * 16;
            }
            bidx[u] = b;
            codes[u] = 0u;
            sbyte[u] = 0u;
            if (c < a.total) {
                codes[u] = ld_stream_u32(a.q + qo);
                sbyte[u] = __ldg(a.sb + (c >> 1));
            }
        }
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const uint32_t c = base + u * stride;
            if (c < a.total) {
                const float gs = __ldg(a.gs + bidx[u]);
                st_v4(a.y + yo[u], dequant_half(codes[u], e4m3_decode(sbyte[u]), gs));
            }
        }
    }
}

bool dense_rows(const View& v, int64_t row_bytes) {
    return v.rstride == row_bytes;
}

}  // namespace

cudaError_t launch_nvfp4_amax(const View* x, int n, uint32_t* amax_bits, cudaStream_t s) {
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
        S.dense_x = dense_rows(x[i], x[i].cols * 2);
        max_chunks = std::max<int64_t>(max_chunks, S.chunks);
    }
    const int64_t total_ctas = (max_chunks + int64_t(kThreads) * kUnroll - 1) / (int64_t(kThreads) * kUnroll);
    // spread about 4 resident CTAs per SM over all groups
    const int64_t budget = (int64_t)sm_count(current_device()) * 4;
    int gx = (int)std::max<int64_t>(1, std::min<int64_t>(total_ctas, (budget + B - 1) / B));
    dim3 grid(gx, (unsigned)B);
    nvfp4_amax_kernel<<<grid, kThreads, 0, s>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_nvfp4_encode(const View* x, int n, const View* out, uint8_t* const* sb,
                                bool fake, const uint32_t* amax_bits, const float* amax_in,
                                float* gs_out, float* amax_out, cudaStream_t s) {
    const int64_t B = x[0].batch;
    EncodeArgs a{};
    a.n = n;
    a.amax_bits = amax_bits;
    a.amax_in = amax_in;
    a.gs_out = gs_out;
    a.amax_out = amax_out;
    int64_t max_chunks = 0;
    for (int i = 0; i < n; ++i) {
        Sib& S = a.s[i];
        S.x = x[i].ptr;
        S.x_bs = x[i].bstride;
        S.x_rs = x[i].rstride;
        S.out = out[i].ptr;
        S.o_bs = out[i].bstride;
        S.o_rs = out[i].rstride;
        S.sb = fake ? nullptr : sb[i];
        S.chunks = (uint32_t)(x[i].rows * (x[i].cols / 8));
        S.cpr = make_fastdiv((uint32_t)std::max<int64_t>(1, x[i].cols / 8));
        S.dense_x = dense_rows(x[i], x[i].cols * 2);
        S.dense_o = dense_rows(out[i], fake ? out[i].cols * 2 : out[i].cols / 2);
        max_chunks = std::max<int64_t>(max_chunks, S.chunks);
    }
    const int64_t span = int64_t(kThreads) * kUnroll;
    const int64_t total_ctas = (max_chunks + span - 1) / span;
    const int64_t budget = (int64_t)sm_count(current_device()) * 8;
    int gx = (int)std::max<int64_t>(1, std::min<int64_t>(total_ctas, (budget + B - 1) / B));
    dim3 grid(gx, (unsigned)B);
    if (fake)
        nvfp4_encode_kernel<true><<<grid, kThreads, 0, s>>>(a);
    else
        nvfp4_encode_kernel<false><<<grid, kThreads, 0, s>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_nvfp4_dequant(const View& q, const uint8_t* sb, const float* gs, const View& y,
                                 cudaStream_t s) {
    DequantArgs a;
    a.q = q.ptr;
    a.y = y.ptr;
    a.sb = sb;
    a.gs = gs;
    a.q_bs = q.bstride;
    a.q_rs = q.rstride;
    a.y_bs = y.bstride;
    a.y_rs = y.rstride;
    const int64_t cpr = q.cols / 8;
    a.cpr = make_fastdiv((uint32_t)cpr);
    a.per_batch = make_fastdiv((uint32_t)(q.rows * cpr));
    a.rows = make_fastdiv((uint32_t)q.rows);
    a.total = (uint32_t)(q.batch * q.rows * cpr);
    a.dense = q.rstride == q.cols / 2 && y.rstride == y.cols * 2 &&
              (q.batch == 1 || (q.bstride == q.rows * q.rstride && y.bstride == y.rows * y.rstride));
    const int64_t span = int64_t(kThreads) * kUnroll;
    const int grid = persistent_grid((a.total + span - 1) / span, 8);
    nvfp4_dequant_kernel<<<grid, kThreads, 0, s>>>(a);
    return cudaGetLastError();
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
    constexpr int kMaxDevices = 64;
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
