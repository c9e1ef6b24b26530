// pwq_internal.h -- host-side launch interface between the C ABI layer
// (pwq_api.cu: validation) and the kernel files.  Byte strides throughout.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "pwq_device.cuh"

namespace pwq {

// A validated [batch][rows][cols] operand with strides in bytes.
struct View {
    char* ptr;
    int64_t batch, rows, cols;
    int64_t bstride, rstride;  // bytes
};

// Per-device properties cached on first use.
int sm_count(int device);
int current_device();

// Raises the dynamic shared-memory limit of the n kernels `fns` to `bytes`
// on the current device, once per device for each call site (`done` is that
// site's per-device flag array of kMaxDevices entries).  Thread-safe: the
// flags are read and written under one lock.
constexpr int kMaxDevices = 64;
cudaError_t set_smem_limit_once(int* done, const void* const* fns, int n, int bytes);

// Grid size for a persistent elementwise kernel: enough CTAs to cover
// `work_ctas`, at most `per_sm` resident CTAs per SM.
int persistent_grid(int64_t work_ctas, int per_sm);

// Tensors per kernel launch of a grouped call (their descriptors, TMA maps
// included, travel as kernel parameters); longer lists are split.
constexpr int kMaxLaunchTensors = 16;

// One independent tensor of a grouped elementwise call.
struct Job {
    View in, out;
    void* scale;       // FP8: float [B][TM][TN]; MXFP8: uint8 [B][M][N/32]; NVFP4 dequant: uint8 sb [B][M][N/16]
    const float* gs;   // NVFP4 dequant: [B]
    int scale_mma = 0; // MXFP8 quantise: scale bytes in the tensor-core tile layout instead of dense
};

// The tensor-core (block-scaled MMA) layout of an [B][M][S] array of scale
// bytes: per batch slab, tiles of 128 rows x 4 scale columns, 512
// contiguous bytes each, ordered along S within a 128-row band and band
// after band; the scale of tile row r and column c at byte
// (r % 32) * 16 + (r / 32) * 4 + c; rows padded to 128, columns to 4.
inline int64_t mma_scale_col_tiles(int64_t S) { return (S + 3) / 4; }
inline int64_t mma_scale_slab_bytes(int64_t M, int64_t S) { return (M + 127) / 128 * mma_scale_col_tiles(S) * 512; }
inline bool mma_scale_padded(int64_t M, int64_t S) { return M % 128 != 0 || S % 4 != 0; }
// Byte offset of (row r, scale column c) inside one slab (device and host).
__host__ __device__ __forceinline__ uint32_t mma_scale_offset(uint32_t r, uint32_t c, uint32_t col_tiles) {
    return ((r >> 7) * col_tiles + (c >> 2)) * 512u + (r & 31u) * 16u + ((r >> 5) & 3u) * 4u + (c & 3u);
}
cudaError_t launch_scales_to_mma(const uint8_t* dense, int64_t B, int64_t M, int64_t S, uint8_t* mma,
                                 cudaStream_t s);
cudaError_t launch_scales_from_mma(const uint8_t* mma, int64_t B, int64_t M, int64_t S, uint8_t* dense,
                                   cudaStream_t s);

cudaError_t launch_fp8_block_quant(const Job* jobs, int n, cudaStream_t s);
cudaError_t launch_fp8_block_dequant(const Job* jobs, int n, cudaStream_t s);
cudaError_t launch_mxfp8_quant(const Job* jobs, int n, cudaStream_t s);
cudaError_t launch_mxfp8_dequant(const Job* jobs, int n, cudaStream_t s);
cudaError_t launch_nvfp4_dequant(const Job* jobs, int n, cudaStream_t s);

// NVFP4 sibling group: members share the per-batch-index group amax.
struct NvGroup {
    const View* x;          // n members
    const View* out;        // packed codes (quant) or BF16 (fake-quant)
    uint8_t* const* sb;     // quant: n block-scale arrays [B][M][N/16]; fake: null
    int n;
    const float* amax_in;   // [B] or null
    float* gs_out;          // [B] or null
    float* amax_out;        // [B] or null
    const float* const* ts = nullptr;   // FP8 block-wise source: n tile-scale arrays (x are E4M3 code views)
    int sb_mma = 0;                     // quantise: block scales in the tensor-core tile layout
};

// NVFP4 single-pass quantise / fake-quantise of groups whose amax is reduced
// on the device (amax_in null for every group): one dataflow launch per
// piece.  Workspace: nvfp4_flow_workspace_bytes(total batch over groups).
// wait_ns bounds an encode item's wait for its instance's amax (2 s);
// wait_on_idle_counts (the self-test of that bound only) makes the encode
// items wait on counts that no amax item adds to, so every wait runs out;
// its workspace is nvfp4_flow_timeout_selftest_bytes(instances).
constexpr uint64_t kFlowWaitLimitNs = 2000000000ull;
size_t nvfp4_flow_workspace_bytes(int64_t instances);
size_t nvfp4_flow_timeout_selftest_bytes(int64_t instances);
cudaError_t launch_nvfp4_flow(const NvGroup* groups, int n_groups, bool fake, void* workspace,
                              cudaStream_t s, uint64_t wait_ns = kFlowWaitLimitNs,
                              bool wait_on_idle_counts = false);

// NVFP4 group amax of one group set (nvfp4_group_amax, and the amax launch
// of the no-allocation entry point): amax_bits receives B words holding
// max |x| of each group as binary32 bits (cleared first).  With ts non-null
// the members are E4M3 code views (FP8 block-wise, ts[i] the member's tile
// scales [B][TM][TN]) and the values are their dequantised BF16 values.
cudaError_t launch_nvfp4_amax(const View* x, int n, uint32_t* amax_bits, cudaStream_t s,
                              const float* const* ts = nullptr);
// NVFP4 "4over6" quantise / fake-quantise of sibling groups (launches of up
// to kMaxLaunchTensors members): the group amax (unless the group has
// amax_in) and the encode that keeps, per block, the candidate -- amax
// mapped to 6 or to 4 -- with the smaller squared error; gs = fl(A / (6
// e4m3_max)).  Workspace: nvfp4_4over6_workspace_bytes(total batch over
// groups), one amax word per instance.
size_t nvfp4_4over6_workspace_bytes(int64_t instances);

// NVFP4 quantise / fake-quantise of groups whose every instance has at most
// 131072 elements (BF16 source, dense block scales): one thread-block
// cluster per instance, one launch, no workspace.  nvfp4_cluster_ok tells
// whether a call qualifies.
bool nvfp4_cluster_ok(const NvGroup* groups, int n_groups);

// NVFP4 quantise / fake-quantise of sibling groups whose amax is known before
// the launch: G.amax_in per group, else amax_bits (one word per instance,
// numbered across the call).  One streaming launch per kMaxLaunchTensors
// members; with G.ts set the source is FP8 block-wise (quantise only).
cudaError_t launch_nvfp4_units_encode(const NvGroup* groups, int n_groups, bool fake, const uint32_t* amax_bits,
                                      cudaStream_t s);
cudaError_t launch_nvfp4_cluster(const NvGroup* groups, int n_groups, bool fake, cudaStream_t s);
cudaError_t launch_nvfp4_4over6(const NvGroup* groups, int n_groups, bool fake, int e4m3_max, void* workspace,
                               cudaStream_t s);

// FP8 block-wise codes + tile scales re-quantised (dequantise, quantise) into
// FP8 block-wise (new FP32 tile scales) or MXFP8 (UE8M0 bytes), a list of
// tensors per call; out may be in exactly, scale_out may be scale_in (FP8).
struct RequantJob {
    View in, out;           // E4M3 codes
    const void* scale_in;   // FP32 [B][TM][TN]
    void* scale_out;        // FP8: FP32 [B][TM][TN]; MXFP8: uint8 [B][M][N/32]
};
cudaError_t launch_fp8_requant_fp8(const RequantJob* jobs, int n, cudaStream_t st);
// The TMA-staged form of the FP8 -> FP8 re-quantisation (fp8_block.cu),
// usable when every input code tensor has 16-byte aligned rows.
bool fp8_requant_tma_ok(const RequantJob* jobs, int n);
cudaError_t launch_fp8_requant_tma(const RequantJob* jobs, int n, cudaStream_t st);
cudaError_t launch_fp8_requant_mxfp8(const RequantJob* jobs, int n, cudaStream_t st);

// Device address (on the current device) of the file-scope group-amax
// scratch used by nvfp4_fake_quant_noalloc; kStaticScratchGroups words.
constexpr int64_t kStaticScratchGroups = 4096;
cudaError_t static_amax_scratch(uint32_t** ptr);

// Read and clear the device error words (synchronous): TMA waits (FP8
// block-wise quantise) and the NVFP4 single-pass amax waits.
cudaError_t read_and_clear_device_error(uint32_t* code);
cudaError_t read_and_clear_flow_error(uint32_t* code);

// W4A4 activation observer step over x (BF16): state (lo, hi) updated per
// `kind` (0 memoryless, 1 static, 2 moving average with constant c),
// amax_out / gs_out (nullable) = A and fl(A / 2688).  words: 2 scratch words.
cudaError_t launch_activation_observe(const View& x, int kind, float c, float* state, float* amax_out,
                                      float* gs_out, uint32_t* words, cudaStream_t s);

cudaError_t launch_selftest_division(int which, unsigned long long* counts, cudaStream_t s);
cudaError_t launch_selftest_codecs(uint32_t first, uint32_t count, uint8_t* e4m3, uint8_t* e2m1,
                                   uint16_t* bf16, cudaStream_t s);

}  // namespace pwq
