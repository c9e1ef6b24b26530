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

// Grid size for a persistent elementwise kernel: enough CTAs to cover
// `work_ctas`, at most `per_sm` resident CTAs per SM.
int persistent_grid(int64_t work_ctas, int per_sm);

cudaError_t launch_fp8_block_quant(const View& x, const View& q, float* scale, cudaStream_t s);
cudaError_t launch_fp8_block_dequant(const View& q, const float* scale, const View& y, cudaStream_t s);
cudaError_t launch_mxfp8_quant(const View& x, const View& q, uint8_t* scale, cudaStream_t s);
cudaError_t launch_mxfp8_dequant(const View& q, const uint8_t* scale, const View& y, cudaStream_t s);

// NVFP4.  amax_bits: B words holding max |x| of each group as binary32 bits.
cudaError_t launch_nvfp4_amax(const View* x, int n, uint32_t* amax_bits, cudaStream_t s);
cudaError_t launch_nvfp4_encode(const View* x, int n, const View* out, uint8_t* const* sb,
                                bool fake, const uint32_t* amax_bits, const float* amax_in,
                                float* gs_out, float* amax_out, cudaStream_t s);
cudaError_t launch_nvfp4_dequant(const View& q, const uint8_t* sb, const float* gs, const View& y,
                                 cudaStream_t s);

// Device address (on the current device) of the file-scope group-amax
// scratch used by nvfp4_fake_quant_noalloc; kStaticScratchGroups words.
constexpr int64_t kStaticScratchGroups = 4096;
cudaError_t static_amax_scratch(uint32_t** ptr);

// Reads and clears the device error word (synchronous).
cudaError_t read_and_clear_device_error(uint32_t* code);

cudaError_t launch_selftest_division(int which, unsigned long long* counts, cudaStream_t s);
cudaError_t launch_selftest_codecs(uint32_t first, uint32_t count, uint8_t* e4m3, uint8_t* e2m1,
                                   uint16_t* bf16, cudaStream_t s);

}  // namespace pwq
