// fp8_block.cu -- FP8 block-wise quantise / dequantise: 128x128 tiles, one
// FP32 scale per tile (s = fl(amax / 448), the dequant multiplier), E4M3
// codes.  Source: "Low Precision RL", "Choose a precision" table and
// "Modes" 2 (DeepSeek-style 128x128 block-wise FP8 with FP32 scales);
// "低精度训练与 Rollout", "FP8 训练 + FP8 Rollout" (FP32 block scales; FP8
// weights dequantised to BF16 on weight update).
//
// Every kernel takes a list of up to kMaxLaunchTensors independent tensors
// (one decoder layer's weights, say) and walks the concatenation of their
// work units with a persistent grid, so a whole list costs one launch: tile
// pairs for the quantiser, rows of 16-code chunks for the dequantiser when
// every tensor has N % 16 == 0 and 16-byte aligned code rows (tiles
// otherwise), tiles for the FP8 -> FP8 re-quantiser.
//
// Quantise: one 512-thread CTA per SM over pairs of horizontally adjacent
// tiles.  Each pair is brought into shared memory by one 3-D TMA box load
// (cp.async.bulk.tensor, no multicast, 128 rows x 256 columns) from its
// tensor's map; the out-of-range part of an edge box is zero-filled, and
// zeros never raise the amax, so the load side needs no masking.  A ring of
// kPairStages box buffers keeps the next pairs in flight while the current
// one is reduced: every thread copies its 64 elements to registers, one
// barrier publishes the warp maxima and frees the buffer, which is refilled
// at once, and each half of the CTA computes its tile's codes from
// registers with one correctly rounded reciprocal per tile plus an FMA
// residual correction per element (proved to give the IEEE-division codes
// by the exhaustive self-test).
#include <algorithm>
#include <cuda.h>

#include "pwq_internal.h"

namespace pwq {
namespace {

constexpr int kTile = 128;
constexpr int kThreads = 256;
constexpr int kTileBytes = kTile * kTile * 2;  // BF16
constexpr int kChunksPerThread = kTile * kTile / 8 / kThreads;  // 8
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s

// Device-side error word of this library (bit kErrTmaTimeout: a TMA wait
// gave up).  Read and cleared by pwq_device_error().
__device__ uint32_t g_device_error = 0u;

// One tensor of a grouped launch (byte strides).
struct TileTensor {
    char* q;              // E4M3 codes: quant output, dequant input
    char* y;              // dequant: BF16 output
    int64_t q_bs, q_rs, y_bs, y_rs;
    float* scale;         // dense [B][TM][TN]
    int rows, cols;
    uint32_t tile_begin;  // first tile of this tensor in the launch
    FastDiv tiles_n;      // tiles per tile row (TN)
    FastDiv tiles_mn;     // tiles per batch matrix (TM * TN)
    int q16, y32;         // dequant: code rows 16-byte, BF16 rows 32-byte aligned
    uint32_t pair_begin;  // quantise: first tile pair of this tensor in the launch
    FastDiv pairs_n;      // quantise: tile pairs per tile row (ceil(TN / 2))
    FastDiv pairs_mn;     // quantise: tile pairs per batch matrix (TM * ceil(TN / 2))
};

struct TileLoc {
    int i;                // tensor
    uint32_t lt;          // tile within the tensor (= its scale index)
    int b, tm, tn;
};

template <class Args>
__device__ __forceinline__ TileLoc locate(const Args& a, uint32_t tile) {
    int i = 0;
    for (int k = 1; k < a.n; ++k)
        if (tile >= a.t[k].tile_begin) i = k;
    const TileTensor& T = a.t[i];
    TileLoc L;
    L.i = i;
    L.lt = tile - T.tile_begin;
    const uint32_t b = fdiv(L.lt, T.tiles_mn);
    const uint32_t rem = L.lt - b * T.tiles_mn.d;
    const uint32_t tm = fdiv(rem, T.tiles_n);
    L.b = (int)b;
    L.tm = (int)tm;
    L.tn = (int)(rem - tm * T.tiles_n.d);
    return L;
}

struct QuantArgs {
    CUtensorMap tmap[kMaxLaunchTensors];
    TileTensor t[kMaxLaunchTensors];
    int n;
    uint32_t total_tiles;
};

// E4M3 codes of a thread's 8 chunks (64 elements) for tile scale s with
// r = RN(1/s); kFast selects the reciprocal path for the whole tile.
template <bool kFast>
__device__ __forceinline__ void encode_chunks(const uint4 (&v)[kChunksPerThread], float s, float r,
                                              uint2 (&out)[kChunksPerThread]) {
#pragma unroll
    for (int j = 0; j < kChunksPerThread; ++j) {
        float q[8];
        quotients8<kFast>(v[j], s, r, q);
        out[j].x = e4m3x4(q[0], q[1], q[2], q[3]);
        out[j].y = e4m3x4(q[4], q[5], q[6], q[7]);
    }
}

// Quantise kernel: one CTA per SM takes pairs of horizontally adjacent tiles
// (one 3-D TMA box of 128 rows x 256 columns, 512 contiguous bytes per row;
// the tile walk reads memory in longer contiguous pieces than a box per
// tile, which the DRAM serves more efficiently).  Threads 0..255 own the
// left tile, 256..511 the right one, each half exactly as one tile's worth
// of work: 64 elements per thread.  A right tile beyond the tensor's last
// tile column (an odd tile count) is zero-filled by the load and skipped.
constexpr int kPairThreads = 2 * kThreads;
constexpr int kPairStages = 3;
constexpr int kPairCols = 2 * kTile;
constexpr int kPairBytes = kTile * kPairCols * 2;  // BF16

struct PairLoc {
    int i;                // tensor
    int b, tm, tp;        // batch, tile row, tile pair (tiles 2 tp, 2 tp + 1)
};

__device__ __forceinline__ PairLoc locate_pair(const QuantArgs& a, uint32_t pair) {
    int i = 0;
    for (int k = 1; k < a.n; ++k)
        if (pair >= a.t[k].pair_begin) i = k;
    const TileTensor& T = a.t[i];
    PairLoc L;
    L.i = i;
    const uint32_t lp = pair - T.pair_begin;
    const uint32_t b = fdiv(lp, T.pairs_mn);
    const uint32_t rem = lp - b * T.pairs_mn.d;
    const uint32_t tm = fdiv(rem, T.pairs_n);
    L.b = (int)b;
    L.tm = (int)tm;
    L.tp = (int)(rem - tm * T.pairs_n.d);
    return L;
}

__global__ void __launch_bounds__(kPairThreads, 1)
fp8_block_quant_kernel(const __grid_constant__ QuantArgs a) {
    extern __shared__ unsigned char smem[];
    __shared__ __align__(8) uint64_t bars[kPairStages];
    __shared__ PairLoc meta[kPairStages];
    __shared__ uint32_t red[2][kPairThreads / 32];

    const uint32_t tid = threadIdx.x;
    // the ring starts at the first 1024-byte boundary of dynamic shared memory
    const uint32_t pad = (1024u - (smem_addr(smem) & 1023u)) & 1023u;
    unsigned char* ring = smem + pad;
    const uint32_t smem0 = smem_addr(ring);
    if (tid == 0) {
        for (int s = 0; s < kPairStages; ++s) mbar_init(smem_addr(&bars[s]), 1);
        fence_mbar_init();
    }
    __syncthreads();

    // thread 0 locates a tile pair, records it for the consumers (visible to
    // them once they observe the barrier phase) and starts its TMA load
    auto issue = [&](uint32_t p, uint32_t s) {
        const PairLoc L = locate_pair(a, p);
        meta[s] = L;
        const uint32_t bar = smem_addr(&bars[s]);
        mbar_arrive_expect_tx(bar, kPairBytes);
        tma_load_3d(smem0 + s * kPairBytes, &a.tmap[L.i], bar, L.tp * kPairCols, L.tm * kTile, L.b);
    };

    const uint32_t first = blockIdx.x, step = gridDim.x;
    if (tid == 0) {
        for (int s = 0; s < kPairStages; ++s) {
            const uint32_t p = first + (uint32_t)s * step;
            if (p < a.total_tiles) issue(p, (uint32_t)s);
        }
    }

    // half h of the CTA owns tile 2 tp + h; within it, thread lt owns 16
    // consecutive elements of rows (lt >> 3) + 32 i, i = 0..3, at columns
    // (lt & 7) * 16: chunk j (8 elements) is row (lt >> 3) + 32 (j >> 1),
    // columns (lt & 7) * 16 + 8 (j & 1), so a row's 16 codes leave in one
    // 16-byte store
    const uint32_t h = tid >> 8, lt = tid & 255u;
    const int c16 = (int)(lt & 7u) * 16;
    const int r16 = (int)(lt >> 3);

    uint32_t it = 0;
    for (uint32_t p = first; p < a.total_tiles; p += step, ++it) {
        const uint32_t s = it % kPairStages;
        const uint32_t parity = (it / kPairStages) & 1u;
        const bool ok = mbar_wait_bounded(smem_addr(&bars[s]), parity, kWaitLimitNs);
        const unsigned char* buf = ring + s * kPairBytes + h * (kTile * 2);
        const PairLoc L = meta[s];
        uint4 v[kChunksPerThread];
        uint32_t m = 0u;
#pragma unroll
        for (int j = 0; j < kChunksPerThread; ++j) {
            v[j] = make_uint4(0u, 0u, 0u, 0u);
            if (ok) v[j] = *reinterpret_cast<const uint4*>(buf + (r16 + 32 * (j >> 1)) * (kPairCols * 2) + (c16 + 8 * (j & 1)) * 2);
            m = max(m, amax_bits8(v[j]));
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, o));
        if ((tid & 31u) == 0u) red[it & 1u][tid >> 5] = m;
        // one barrier: publishes the warp maxima, ends every read of buffer
        // s and of meta[s], and makes a timed-out wait a CTA-uniform decision
        if (__syncthreads_or(!ok)) {
            if (tid == 0) {
                atomicOr(&g_device_error, kErrTmaTimeout);
                // let every issued copy land before shared memory is released
                for (uint32_t k = 0; k < (uint32_t)kPairStages; ++k) {
                    if (p + k * step < a.total_tiles)
                        (void)mbar_wait_bounded(smem_addr(&bars[(it + k) % kPairStages]),
                                                ((it + k) / kPairStages) & 1u, kWaitLimitNs);
                }
            }
            return;
        }
        if (tid == 0) {
            const uint32_t pn = p + (uint32_t)kPairStages * step;
            if (pn < a.total_tiles) issue(pn, s);
        }
        const TileTensor& T = a.t[L.i];
        const int tn = 2 * L.tp + (int)h;
        if (tn >= (int)T.tiles_n.d) continue;   // uniform over the half: no right tile
        uint32_t am = red[it & 1u][h * 8u];
#pragma unroll
        for (int w = 1; w < kThreads / 32; ++w) am = max(am, red[it & 1u][h * 8u + w]);

        const float sc = fp8_tile_scale(__uint_as_float(am << 16));
        const float rc = __frcp_rn(sc);
        uint2 out[kChunksPerThread];
        if (div_fast_ok(sc))   // uniform over the half
            encode_chunks<true>(v, sc, rc, out);
        else
            encode_chunks<false>(v, sc, rc, out);

        if (lt == 0) T.scale[(uint32_t)L.b * T.tiles_mn.d + (uint32_t)L.tm * T.tiles_n.d + (uint32_t)tn] = sc;
        const int rows_here = min(kTile, T.rows - L.tm * kTile);
        const int cols_here = min(kTile, T.cols - tn * kTile);
        char* qtile = T.q + (int64_t)L.b * T.q_bs + (int64_t)L.tm * kTile * T.q_rs + (int64_t)tn * kTile;
        if (rows_here == kTile && cols_here == kTile && T.q16) {
#pragma unroll
            for (int i = 0; i < kChunksPerThread / 2; ++i)
                st_v4(qtile + (int64_t)(r16 + 32 * i) * T.q_rs + c16,
                      make_uint4(out[2 * i].x, out[2 * i].y, out[2 * i + 1].x, out[2 * i + 1].y));
        } else {
#pragma unroll
            for (int j = 0; j < kChunksPerThread; ++j) {
                const int r = r16 + 32 * (j >> 1), ccol = c16 + 8 * (j & 1);
                if (r >= rows_here || ccol >= cols_here) continue;
                char* dst = qtile + (int64_t)r * T.q_rs + ccol;
                if (ccol + 8 <= cols_here) {
                    st_v2(dst, out[j]);
                } else {
                    for (int e = 0; e < cols_here - ccol; ++e)
                        dst[e] = (char)((e < 4 ? out[j].x >> (8 * e) : out[j].y >> (8 * (e - 4))) & 0xffu);
                }
            }
        }
    }
}

// Dequantise: a persistent grid walks the tiles of the list; the tile scale
// is one load per tile.  Thread t owns 8-code chunks at column (t & 15) * 8
// of rows (t >> 4) + 16 j, j = 0..7 (the quantiser's mapping): an 8-byte
// code load becomes one 16-byte BF16 store, and the 16 lanes of a row write
// 256 contiguous bytes.  Edge tiles take a masked element-wise path.
struct DequantArgs {
    TileTensor t[kMaxLaunchTensors];
    int n;
    uint32_t total_tiles;
};

constexpr int kDqRowsPerPass = kThreads / 16;        // 16
constexpr int kDqChunks = kTile / kDqRowsPerPass;     // 8

__global__ void __launch_bounds__(kThreads) fp8_block_dequant_kernel(const __grid_constant__ DequantArgs a) {
    const int ccol = (int)(threadIdx.x & 15u) * 8;
    const int row0 = (int)(threadIdx.x >> 4);
    for (uint32_t t = blockIdx.x; t < a.total_tiles; t += gridDim.x) {
        const TileLoc L = locate(a, t);
        const TileTensor& T = a.t[L.i];
        const float sc = __ldg(T.scale + L.lt);
        const char* qt = T.q + (int64_t)L.b * T.q_bs + (int64_t)L.tm * kTile * T.q_rs + (int64_t)L.tn * kTile;
        char* yt = T.y + (int64_t)L.b * T.y_bs + (int64_t)L.tm * kTile * T.y_rs + (int64_t)L.tn * kTile * 2;
        const int rows_here = min(kTile, T.rows - L.tm * kTile);
        const int cols_here = min(kTile, T.cols - L.tn * kTile);
        if (rows_here == kTile && cols_here == kTile && T.q16) {
            // 16 codes per thread per row pass: 8 threads per 128-code row
            const int c16 = (int)(threadIdx.x & 7u) * 16;
            const int r16 = (int)(threadIdx.x >> 3);
            uint4 v[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) v[j] = ld_stream_v4(qt + (int64_t)(r16 + 32 * j) * T.q_rs + c16);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const uint4 y0 = fp8_dequant8(make_uint2(v[j].x, v[j].y), sc);
                const uint4 y1 = fp8_dequant8(make_uint2(v[j].z, v[j].w), sc);
                char* dst = yt + (int64_t)(r16 + 32 * j) * T.y_rs + c16 * 2;
                if (T.y32) {
                    st_v8(dst, y0, y1);
                } else {
                    st_v4(dst, y0);
                    st_v4(dst + 16, y1);
                }
            }
        } else if (rows_here == kTile && cols_here == kTile) {
            uint2 v[kDqChunks];
#pragma unroll
            for (int j = 0; j < kDqChunks; ++j)
                v[j] = ld_stream_v2(qt + (int64_t)(row0 + kDqRowsPerPass * j) * T.q_rs + ccol);
#pragma unroll
            for (int j = 0; j < kDqChunks; ++j)
                st_v4(yt + (int64_t)(row0 + kDqRowsPerPass * j) * T.y_rs + ccol * 2, fp8_dequant8(v[j], sc));
        } else {
            for (int j = 0; j < kDqChunks; ++j) {
                const int r = row0 + kDqRowsPerPass * j;
                if (r >= rows_here) break;
                const unsigned char* src = reinterpret_cast<const unsigned char*>(qt + (int64_t)r * T.q_rs);
                unsigned short* dst = reinterpret_cast<unsigned short*>(yt + (int64_t)r * T.y_rs);
                for (int c = ccol; c < min(ccol + 8, cols_here); ++c) {
                    const float f = __fmul_rn(e4m3_decode(src[c]), sc);
                    dst[c] = (unsigned short)(pack_bf16x2(f, 0.0f) & 0xffffu);
                }
            }
        }
    }
}

// Dequantise by rows: the dequantiser needs no reduction over a tile, so
// when every tensor of a launch has N % 16 == 0 and 16-byte aligned code
// rows it streams the rows like the MXFP8 dequantiser instead of walking
// tiles: 16-code chunks in row-major order (a chunk never leaves its tile:
// 128 is a multiple of 16), a warp span of 32 consecutive chunks per step,
// kRowDqUnroll chunks per lane loaded before any is stored, one cached
// tile-scale load per chunk, 32 bytes of BF16 out per chunk (one 256-bit
// store when the BF16 rows are 32-byte aligned).
struct RowDqTensor {
    const char* q;
    char* y;
    int64_t q_bs, q_rs, y_bs, y_rs;   // bytes
    const float* scale;               // dense [B][TM][TN]
    uint32_t chunks;                  // B * M * N / 16
    uint32_t slot_begin;              // multiple of kRowDqSpan
    FastDiv cpr;                      // chunks per row (N / 16)
    FastDiv rows;                     // M
    uint32_t tm, tn;                  // tiles per column / per row
    int dense;
    int y32;
};

struct RowDqArgs {
    RowDqTensor t[kMaxLaunchTensors];
    int n;
    uint32_t total_slots;
};

constexpr int kRowDqUnroll = 8;
constexpr uint32_t kRowDqSpan = 32u * kRowDqUnroll;

__global__ void __launch_bounds__(kThreads) fp8_block_dequant_rows_kernel(const __grid_constant__ RowDqArgs a) {
    const uint32_t lane = threadIdx.x & 31u;
    const uint32_t gwarp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const uint32_t nwarps = (gridDim.x * blockDim.x) >> 5;
    for (uint32_t slot = gwarp * kRowDqSpan; slot < a.total_slots; slot += nwarps * kRowDqSpan) {
        int ti = 0;
        for (int k = 1; k < a.n; ++k)
            if (slot >= a.t[k].slot_begin) ti = k;
        const RowDqTensor& T = a.t[ti];
        const uint32_t base = slot - T.slot_begin;
        uint4 v[kRowDqUnroll];
        float sc[kRowDqUnroll];
        int64_t yo[kRowDqUnroll];
#pragma unroll
        for (int u = 0; u < kRowDqUnroll; ++u) {
            const uint32_t c = base + u * 32u + lane;
            const uint32_t r = fdiv(c, T.cpr);            // row over all batches
            const uint32_t k = c - r * T.cpr.d;           // chunk within the row
            const uint32_t b = fdiv(r, T.rows);
            const uint32_t m = r - b * T.rows.d;
            int64_t qo;
            if (T.dense) {
                qo = (int64_t)c * 16;
                yo[u] = (int64_t)c * 32;
            } else {
                qo = (int64_t)b * T.q_bs + (int64_t)m * T.q_rs + (int64_t)k * 16;
                yo[u] = (int64_t)b * T.y_bs + (int64_t)m * T.y_rs + (int64_t)k * 32;
            }
            v[u] = make_uint4(0u, 0u, 0u, 0u);
            sc[u] = 0.0f;
            if (c < T.chunks) {
                v[u] = ld_stream_v4(T.q + qo);
                sc[u] = __ldg(T.scale + ((int64_t)b * T.tm + (m >> 7)) * T.tn + (k >> 3));
            }
        }
#pragma unroll
        for (int u = 0; u < kRowDqUnroll; ++u) {
            const uint32_t c = base + u * 32u + lane;
            if (c >= T.chunks) continue;
            const uint4 y0 = fp8_dequant8(make_uint2(v[u].x, v[u].y), sc[u]);
            const uint4 y1 = fp8_dequant8(make_uint2(v[u].z, v[u].w), sc[u]);
            if (T.y32) {
                st_v8(T.y + yo[u], y0, y1);
            } else {
                st_v4(T.y + yo[u], y0);
                st_v4(T.y + yo[u] + 16, y1);
            }
        }
    }
}

// FP8 block-wise -> FP8 block-wise re-quantisation (the composition
// fp8_block_quant(fp8_block_dequant(q, s)), see requant.cu) with the code
// tiles staged by TMA like the quantiser's BF16 tiles: 16 KB per tile, a
// ring of kRqStages buffers, 2 CTAs per SM.  The ring depth trades the two
// per-tile paths against each other (ms per 36-layer sweep, identity tiles /
// table lookups): 2 CTAs x 6 stages 1.24 / 1.56, 3 x 4 1.41 / 1.42, 4 x 3
// 1.43 / 1.33; the copy of identity tiles (every tile a quantiser wrote)
// wants the deep ring, the lookups want warps.  Used when every input code
// tensor has 16-byte aligned rows (a TMA stride rule); the tile of old
// scales is read before the CTA's barrier and the new scale written after
// it, so in-place use is safe.
constexpr int kRqStages = 6;
constexpr int kRqTileBytes = kTile * kTile;   // E4M3

struct RequantTmaArgs {
    CUtensorMap tmap[kMaxLaunchTensors];   // input codes
    TileTensor t[kMaxLaunchTensors];       // q = output codes, scale = new scales
    const float* s_in[kMaxLaunchTensors];
    int n;
    uint32_t total_tiles;
};

__global__ void __launch_bounds__(kThreads, 2)
fp8_requant_tma_kernel(const __grid_constant__ RequantTmaArgs a) {
    extern __shared__ unsigned char smem[];
    __shared__ __align__(8) uint64_t bars[kRqStages];
    __shared__ TileLoc meta[kRqStages];
    __shared__ uint32_t red[2][kThreads / 32];
    __shared__ __align__(16) uint8_t lut[128];   // per tile: input magnitude -> output code

    const uint32_t tid = threadIdx.x;
    const uint32_t pad = (1024u - (smem_addr(smem) & 1023u)) & 1023u;
    unsigned char* ring = smem + pad;
    const uint32_t smem0 = smem_addr(ring);
    if (tid == 0) {
        for (int s = 0; s < kRqStages; ++s) mbar_init(smem_addr(&bars[s]), 1);
        fence_mbar_init();
    }
    __syncthreads();

    auto issue = [&](uint32_t t, uint32_t s) {
        const TileLoc L = locate(a, t);
        meta[s] = L;
        const uint32_t bar = smem_addr(&bars[s]);
        mbar_arrive_expect_tx(bar, kRqTileBytes);
        tma_load_3d(smem0 + s * kRqTileBytes, &a.tmap[L.i], bar, L.tn * kTile, L.tm * kTile, L.b);
    };

    const uint32_t first = blockIdx.x, step = gridDim.x;
    if (tid == 0) {
        for (int s = 0; s < kRqStages; ++s) {
            const uint32_t t = first + (uint32_t)s * step;
            if (t < a.total_tiles) issue(t, (uint32_t)s);
        }
    }
    // thread -> 16 consecutive codes of rows (tid >> 3) + 32 i, i = 0..3, at
    // column (tid & 7) * 16; chunk j (8 codes) is row (tid >> 3) + 32 (j >> 1),
    // columns (tid & 7) * 16 + 8 (j & 1)
    const int c16 = (int)(tid & 7u) * 16;
    const int r16 = (int)(tid >> 3);

    uint32_t it = 0;
    for (uint32_t t = first; t < a.total_tiles; t += step, ++it) {
        const uint32_t s = it % kRqStages;
        const uint32_t parity = (it / kRqStages) & 1u;
        const bool ok = mbar_wait_bounded(smem_addr(&bars[s]), parity, kWaitLimitNs);
        const unsigned char* buf = ring + s * kRqTileBytes;
        const TileLoc L = meta[s];
        const float sc = a.s_in[L.i][L.lt];
        uint2 v[kChunksPerThread];
        uint32_t m = 0u;
#pragma unroll
        for (int i = 0; i < kChunksPerThread / 2; ++i) {
            uint4 w = make_uint4(0u, 0u, 0u, 0u);
            if (ok) w = *reinterpret_cast<const uint4*>(buf + (r16 + 32 * i) * kTile + c16);
            v[2 * i] = make_uint2(w.x, w.y);
            v[2 * i + 1] = make_uint2(w.z, w.w);
            m = __vmaxu2(m, __vmaxu2(e4m3_maxmag_lanes(v[2 * i]), e4m3_maxmag_lanes(v[2 * i + 1])));
        }
        m = e4m3_maxmag_fin(m);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, o));
        if ((tid & 31u) == 0u) red[it & 1u][tid >> 5] = m;
        if (__syncthreads_or(!ok)) {
            if (tid == 0) {
                atomicOr(&g_device_error, kErrTmaTimeout);
                for (uint32_t k = 0; k < (uint32_t)kRqStages; ++k) {
                    if (t + k * step < a.total_tiles)
                        (void)mbar_wait_bounded(smem_addr(&bars[(it + k) % kRqStages]),
                                                ((it + k) / kRqStages) & 1u, kWaitLimitNs);
                }
            }
            return;
        }
        if (tid == 0) {
            const uint32_t tn = t + (uint32_t)kRqStages * step;
            if (tn < a.total_tiles) issue(tn, s);
        }
        uint32_t mc = red[it & 1u][0];
#pragma unroll
        for (int w = 1; w < kThreads / 32; ++w) mc = max(mc, red[it & 1u][w]);
        const float s2 = fp8_tile_scale(__uint_as_float(fp8_amax_bits16(mc, sc) << 16));
        // Within a tile every output code is a function of the input code
        // alone (y = bf16(fl(dec(q) * s)), q' = e4m3(fl(y / s2))), so the
        // codes are mapped through a per-tile table and the per-element
        // arithmetic becomes a byte lookup.  Every step is symmetric in sign
        // (a product, RNE to BF16, a quotient whose zero-divisor case keeps
        // the sign of zero, RNE to E4M3), so the map of code q ^ 0x80 is the
        // map of q with the sign bit flipped: the table holds the 128
        // magnitudes (thread m encodes magnitude m, with the same quotient
        // path, reciprocal or IEEE chosen by s2, as the per-element form),
        // one byte per shared-memory bank word position, so a warp's lookups
        // never conflict, and the input sign bit is xor-ed into the result.
        //
        // When the table is the identity on every non-NaN magnitude the
        // tile's codes are copied unchanged.  That is the usual case, not a
        // special one: if the tile's largest magnitude code is 448 (every
        // tile a quantiser writes) then s2 = fl(bf16(fl(448 s)) / 448) and
        // each quotient is dec(q) times a factor within about 2^-8 of 1, far
        // inside the half-step of E4M3 (2^-5 relative, 2^-10 absolute for
        // subnormal codes), so every code maps to itself.  The decision is
        // taken from the computed table, not from that argument.  The NaN
        // magnitude 0x7F is left out of the test: a tile holding a NaN code
        // has a NaN s2 and a table that is not the identity anywhere else.
        bool ident;
        {
            uint32_t code = 0u;
            if (tid < 128u) {
                const bool fast = div_fast_ok(s2);   // CTA-uniform
                const float r2 = fast ? __frcp_rn(s2) : 0.0f;
                const float y =
                    __uint_as_float((pack_bf16x2(__fmul_rn(e4m3_decode(tid), sc), 0.0f) & 0xffffu) << 16);
                const float q = fast ? div_fast(y, s2, r2) : div_slow(y, s2);
                code = e4m3x2(q, 0.0f) & 0xffu;
                // one table: every thread finished mapping the previous tile
                // before the barrier above
                lut[tid] = (uint8_t)code;
            }
            // the table is complete, and whether it is the identity is known
            ident = __syncthreads_and(tid >= 127u || code == tid) != 0;
        }
        uint2 out[kChunksPerThread];
        if (ident) {
#pragma unroll
            for (int j = 0; j < kChunksPerThread; ++j) out[j] = v[j];
        } else {
#pragma unroll
            for (int j = 0; j < kChunksPerThread; ++j) {
                const uint32_t w[2] = {v[j].x, v[j].y};
                uint32_t o[2];
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const uint32_t mag = w[h] & 0x7f7f7f7fu;
                    const uint32_t b0 = lut[__byte_perm(mag, 0u, 0x4440u)];
                    const uint32_t b1 = lut[__byte_perm(mag, 0u, 0x4441u)];
                    const uint32_t b2 = lut[__byte_perm(mag, 0u, 0x4442u)];
                    const uint32_t b3 = lut[__byte_perm(mag, 0u, 0x4443u)];
                    o[h] = __byte_perm(__byte_perm(b0, b1, 0x0040u), __byte_perm(b2, b3, 0x0040u), 0x5410u) ^
                           (w[h] & 0x80808080u);
                }
                out[j] = make_uint2(o[0], o[1]);
            }
        }

        const TileTensor& T = a.t[L.i];
        if (tid == 0) T.scale[L.lt] = s2;
        const int rows_here = min(kTile, T.rows - L.tm * kTile);
        const int cols_here = min(kTile, T.cols - L.tn * kTile);
        char* qtile = T.q + (int64_t)L.b * T.q_bs + (int64_t)L.tm * kTile * T.q_rs + (int64_t)L.tn * kTile;
        if (rows_here == kTile && cols_here == kTile && T.q16) {
#pragma unroll
            for (int i = 0; i < kChunksPerThread / 2; ++i)
                st_v4(qtile + (int64_t)(r16 + 32 * i) * T.q_rs + c16,
                      make_uint4(out[2 * i].x, out[2 * i].y, out[2 * i + 1].x, out[2 * i + 1].y));
        } else {
#pragma unroll
            for (int j = 0; j < kChunksPerThread; ++j) {
                const int r = r16 + 32 * (j >> 1), ccol = c16 + 8 * (j & 1);
                if (r >= rows_here || ccol >= cols_here) continue;
                char* dst = qtile + (int64_t)r * T.q_rs + ccol;
                if (ccol + 8 <= cols_here) {
                    st_v2(dst, out[j]);
                } else {
                    for (int e = 0; e < cols_here - ccol; ++e)
                        dst[e] = (char)((e < 4 ? out[j].x >> (8 * e) : out[j].y >> (8 * (e - 4))) & 0xffu);
                }
            }
        }
    }
}

// cuTensorMapEncodeTiled through the runtime's driver entry point (no
// link-time dependency on libcuda).
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*,
                                  CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                  CUtensorMapFloatOOBfill);

EncodeTiledFn encode_tiled_fn() {
    static EncodeTiledFn fn = [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) !=
                cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            p = nullptr;
        return reinterpret_cast<EncodeTiledFn>(p);
    }();
    return fn;
}

// Fills the per-tensor descriptor; returns the tensor's tile count.
uint32_t fill_tile_tensor(TileTensor& T, const Job& j, bool quant, uint32_t tile_begin) {
    const View& q = quant ? j.out : j.in;
    T.q = q.ptr;
    T.q_bs = q.bstride;
    T.q_rs = q.rstride;
    T.y = quant ? nullptr : j.out.ptr;
    T.y_bs = quant ? 0 : j.out.bstride;
    T.y_rs = quant ? 0 : j.out.rstride;
    T.scale = static_cast<float*>(j.scale);
    T.rows = (int)q.rows;
    T.cols = (int)q.cols;
    const uint32_t tm = (uint32_t)((q.rows + kTile - 1) / kTile);
    const uint32_t tn = (uint32_t)((q.cols + kTile - 1) / kTile);
    T.tile_begin = tile_begin;
    T.tiles_n = make_fastdiv(tn);
    T.tiles_mn = make_fastdiv(tm * tn);
    const uint32_t tp = (tn + 1) / 2;
    T.pair_begin = 0;
    T.pairs_n = make_fastdiv(tp);
    T.pairs_mn = make_fastdiv(tm * tp);
    T.q16 = (uintptr_t)q.ptr % 16 == 0 && q.rstride % 16 == 0 && (q.batch == 1 || q.bstride % 16 == 0);
    T.y32 = !quant && (uintptr_t)j.out.ptr % 32 == 0 && j.out.rstride % 32 == 0 &&
            (j.out.batch == 1 || j.out.bstride % 32 == 0);
    return (uint32_t)q.batch * tm * tn;
}

}  // namespace

cudaError_t read_and_clear_device_error(uint32_t* code) {
    uint32_t zero = 0u;
    cudaError_t e = cudaMemcpyFromSymbol(code, g_device_error, sizeof(uint32_t));
    if (e != cudaSuccess) return e;
    return cudaMemcpyToSymbol(g_device_error, &zero, sizeof(uint32_t));
}

cudaError_t launch_fp8_block_quant(const Job* jobs, int n, cudaStream_t s) {
    EncodeTiledFn encode = encode_tiled_fn();
    if (!encode) return cudaErrorNotSupported;
    const size_t smem = (size_t)kPairStages * kPairBytes + 1024;
    static int configured[kMaxDevices] = {0};
    const int dev = current_device();
    {
        const void* fn = (const void*)fp8_block_quant_kernel;
        const cudaError_t e = set_smem_limit_once(configured, &fn, 1, (int)smem);
        if (e != cudaSuccess) return e;
    }
    for (int j0 = 0; j0 < n; j0 += kMaxLaunchTensors) {
        QuantArgs a;
        a.n = std::min(n - j0, kMaxLaunchTensors);
        uint32_t pairs = 0;
        for (int k = 0; k < a.n; ++k) {
            const Job& j = jobs[j0 + k];
            const View& x = j.in;
            const cuuint64_t dims[3] = {(cuuint64_t)x.cols, (cuuint64_t)x.rows, (cuuint64_t)x.batch};
            const cuuint64_t strides[2] = {(cuuint64_t)x.rstride,
                                           (cuuint64_t)(x.batch > 1 ? x.bstride : x.rows * x.rstride)};
            const cuuint32_t box[3] = {kPairCols, kTile, 1};
            const cuuint32_t estr[3] = {1, 1, 1};
            CUresult cr = encode(&a.tmap[k], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, x.ptr, dims, strides, box, estr,
                                 CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                                 CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
            if (cr != CUDA_SUCCESS) return cudaErrorInvalidValue;
            TileTensor& T = a.t[k];
            fill_tile_tensor(T, j, true, 0);
            T.pair_begin = pairs;
            pairs += (uint32_t)x.batch * T.pairs_mn.d;
        }
        a.total_tiles = pairs;   // work units of this kernel: tile pairs
        if (pairs == 0) continue;
        const int grid = (int)std::min<int64_t>(pairs, (int64_t)sm_count(dev));
        fp8_block_quant_kernel<<<grid, kPairThreads, smem, s>>>(a);
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

// Row-streaming dequantise of a list whose tensors all have N % 16 == 0 and
// 16-byte aligned code rows.
cudaError_t launch_fp8_block_dequant_rows(const Job* jobs, int n, cudaStream_t s) {
    const uint64_t kMaxSlots = uint64_t(1) << 31;   // chunk indices stay 32-bit
    for (int j0 = 0; j0 < n;) {
        RowDqArgs a;
        a.n = 0;
        uint32_t slots = 0;
        for (; j0 + a.n < n && a.n < kMaxLaunchTensors; ++a.n) {
            const Job& j = jobs[j0 + a.n];
            const View& q = j.in;
            const View& y = j.out;
            const uint64_t chunks = (uint64_t)(q.batch * q.rows * (q.cols / 16));
            const uint64_t padded = (chunks + kRowDqSpan - 1) / kRowDqSpan * kRowDqSpan;
            if (a.n > 0 && slots + padded > kMaxSlots) break;
            RowDqTensor& T = a.t[a.n];
            T.q = q.ptr;
            T.y = y.ptr;
            T.q_bs = q.bstride;
            T.q_rs = q.rstride;
            T.y_bs = y.bstride;
            T.y_rs = y.rstride;
            T.scale = static_cast<const float*>(j.scale);
            T.chunks = (uint32_t)chunks;
            T.slot_begin = slots;
            T.cpr = make_fastdiv((uint32_t)std::max<int64_t>(1, q.cols / 16));
            T.rows = make_fastdiv((uint32_t)std::max<int64_t>(1, q.rows));
            T.tm = (uint32_t)((q.rows + kTile - 1) / kTile);
            T.tn = (uint32_t)((q.cols + kTile - 1) / kTile);
            T.dense = q.rstride == q.cols && y.rstride == y.cols * 2 &&
                      (q.batch == 1 || (q.bstride == q.rows * q.cols && y.bstride == y.rows * y.cols * 2));
            T.y32 = (uintptr_t)y.ptr % 32 == 0 && y.rstride % 32 == 0 && (y.batch == 1 || y.bstride % 32 == 0);
            slots += (uint32_t)padded;
        }
        j0 += a.n;
        a.total_slots = slots;
        if (slots == 0) continue;
        const int grid = persistent_grid((slots + kThreads * kRowDqUnroll - 1) / (kThreads * kRowDqUnroll), 8);
        fp8_block_dequant_rows_kernel<<<grid, kThreads, 0, s>>>(a);
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

cudaError_t launch_fp8_block_dequant(const Job* jobs, int n, cudaStream_t s) {
    bool rows = true;
    for (int i = 0; i < n; ++i) {
        const View& q = jobs[i].in;
        rows = rows && q.cols % 16 == 0 && (uintptr_t)q.ptr % 16 == 0 && q.rstride % 16 == 0 &&
               (q.batch == 1 || q.bstride % 16 == 0);
    }
    if (rows) return launch_fp8_block_dequant_rows(jobs, n, s);
    for (int j0 = 0; j0 < n; j0 += kMaxLaunchTensors) {
        DequantArgs a;
        a.n = std::min(n - j0, kMaxLaunchTensors);
        uint32_t tiles = 0;
        for (int k = 0; k < a.n; ++k) tiles += fill_tile_tensor(a.t[k], jobs[j0 + k], false, tiles);
        a.total_tiles = tiles;
        if (tiles == 0) continue;
        const int grid = persistent_grid(tiles, 8);
        fp8_block_dequant_kernel<<<grid, kThreads, 0, s>>>(a);
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

// FP8 -> FP8 re-quantisation through TMA-staged tiles; false (nothing
// launched) when a tensor's code rows are not 16-byte aligned.
bool fp8_requant_tma_ok(const RequantJob* jobs, int n) {
    for (int i = 0; i < n; ++i) {
        const View& q = jobs[i].in;
        if ((uintptr_t)q.ptr % 16 != 0 || q.rstride % 16 != 0 || (q.batch > 1 && q.bstride % 16 != 0)) return false;
    }
    return encode_tiled_fn() != nullptr;
}

cudaError_t launch_fp8_requant_tma(const RequantJob* jobs, int n, cudaStream_t s) {
    EncodeTiledFn encode = encode_tiled_fn();
    if (!encode) return cudaErrorNotSupported;
    const size_t smem = (size_t)kRqStages * kRqTileBytes + 1024;
    static int configured[kMaxDevices] = {0};
    const int dev = current_device();
    {
        const void* fn = (const void*)fp8_requant_tma_kernel;
        const cudaError_t e = set_smem_limit_once(configured, &fn, 1, (int)smem);
        if (e != cudaSuccess) return e;
    }
    for (int j0 = 0; j0 < n;) {
        RequantTmaArgs a;
        a.n = 0;
        uint32_t tiles = 0;
        for (; j0 + a.n < n && a.n < kMaxLaunchTensors; ++a.n) {
            const RequantJob& J = jobs[j0 + a.n];
            const View& q = J.in;
            const uint32_t tm = (uint32_t)((q.rows + kTile - 1) / kTile);
            const uint32_t tn = (uint32_t)((q.cols + kTile - 1) / kTile);
            const uint64_t count = (uint64_t)q.batch * tm * tn;
            if (a.n > 0 && tiles + count > (uint64_t(1) << 31)) break;
            const cuuint64_t dims[3] = {(cuuint64_t)q.cols, (cuuint64_t)q.rows, (cuuint64_t)q.batch};
            const cuuint64_t strides[2] = {(cuuint64_t)q.rstride,
                                           (cuuint64_t)(q.batch > 1 ? q.bstride : q.rows * q.rstride)};
            const cuuint32_t box[3] = {kTile, kTile, 1};
            const cuuint32_t estr[3] = {1, 1, 1};
            CUresult cr = encode(&a.tmap[a.n], CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, q.ptr, dims, strides, box, estr,
                                 CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                                 CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
            if (cr != CUDA_SUCCESS) return cudaErrorInvalidValue;
            TileTensor& T = a.t[a.n];
            T.q = J.out.ptr;
            T.y = nullptr;
            T.q_bs = J.out.bstride;
            T.q_rs = J.out.rstride;
            T.y_bs = T.y_rs = 0;
            T.q16 = (uintptr_t)J.out.ptr % 16 == 0 && J.out.rstride % 16 == 0 &&
                    (J.out.batch == 1 || J.out.bstride % 16 == 0);
            T.scale = static_cast<float*>(J.scale_out);
            T.rows = (int)q.rows;
            T.cols = (int)q.cols;
            T.tile_begin = tiles;
            T.tiles_n = make_fastdiv(tn);
            T.tiles_mn = make_fastdiv(tm * tn);
            a.s_in[a.n] = static_cast<const float*>(J.scale_in);
            tiles += (uint32_t)count;
        }
        j0 += a.n;
        a.total_tiles = tiles;
        if (tiles == 0) continue;
        const int grid = (int)std::min<int64_t>(tiles, (int64_t)sm_count(dev) * 2);
        fp8_requant_tma_kernel<<<grid, kThreads, smem, s>>>(a);
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

}  // namespace pwq
