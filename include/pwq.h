/*
 * pwq.h -- C ABI of libpwq: block-scaled quantisation of BF16 tensors on
 * NVIDIA B200 (sm_100a), in the three formats of "Low Precision RL"
 * ("Choose a precision" table):
 *
 *   FP8 block-wise  128x128 tiles, one FP32 scale per tile, E4M3 codes
 *   MXFP8           1x32 blocks along a row, UE8M0 (power-of-two) scale byte,
 *                   E4M3 codes
 *   NVFP4           1x16 blocks along a row, E4M3 block scale, one FP32 global
 *                   scale per group, E2M1 codes packed two per byte
 *
 * plus NVFP4 fake-quantisation (quantise then dequantise, BF16 out) as used
 * by quantisation-aware training (verl NVFP4 QAT article, section 2.3), with
 * q/k/v or gate/up siblings sharing one global amax (same article, 2.4).
 *
 * ---------------------------------------------------------------------
 * Conventions shared by every call
 * ---------------------------------------------------------------------
 * Tensors.  A pwq_tensor describes a row-major [batch][rows][cols] array
 * whose last dimension is contiguous.  Strides are counted in storage units
 * of that array: 2-byte units for BF16, bytes for E4M3 codes, bytes for
 * packed E2M1 codes (one byte holds two elements).  `cols` is always the
 * logical number of elements per row.  batch >= 1 (batch > 1 is a stack of
 * independent matrices, e.g. the experts of a MoE layer).
 *
 * Memory.  Every data pointer is a device pointer.  The caller owns every
 * buffer, including outputs and workspace; the library allocates nothing,
 * keeps no state between calls and never synchronises.
 *
 * Alignment.  BF16 tensors: base pointer 16-byte aligned, row and batch
 * strides multiples of 16 bytes.  E4M3 code and packed E2M1 tensors: base
 * pointer and strides multiples of 8 bytes.  Otherwise PWQ_ERR_ALIGN (there
 * is no unaligned slow path).  Scale arrays are dense (layouts below) and
 * need only their natural alignment.
 *
 * Streams.  Every call enqueues its kernels on `stream` (NULL = the legacy
 * default stream) and returns; the status covers host-side validation and
 * the launch itself (cudaGetLastError right after each launch).  Device code
 * never traps; a bounded wait that gives up records a code readable with
 * pwq_device_error().  The outputs of a call that records such a code are
 * unspecified (an encode step that gave up waiting for its group amax goes
 * on with a partial one): a caller that needs to know reads
 * pwq_device_error() after the stream has finished the call.
 *
 * Empty tensors (batch, rows or cols equal to 0) return PWQ_OK and launch
 * nothing.  Outputs may not overlap inputs or each other (PWQ_ERR_OVERLAP),
 * except that nvfp4_fake_quant accepts y == x exactly (in place).
 *
 * Numerics.  Built without fast math (-ftz=false -prec-div=true
 * -prec-sqrt=true -fmad=false); every rounding below is IEEE
 * round-to-nearest-even, as the NVFP4 QDQ review thread on vime pull
 * request #503 requires (fast math refused).  fl() is one binary32 rounding,
 * bf16() rounds binary32 to BF16, e4m3() rounds to E4M3 (FN variant, max 448)
 * saturating, e2m1() rounds to {0,0.5,1,1.5,2,3,4,6} saturating; ties go to
 * the even code; the sign of zero is kept.  NaN and Inf inputs are outside
 * the contract.
 */
#ifndef PWQ_H
#define PWQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* A CUDA stream handle (same object as cudaStream_t). */
typedef struct CUstream_st* pwq_stream_t;

typedef enum pwq_status {
    PWQ_OK = 0,
    PWQ_ERR_NULL = 1,      /* a required pointer is NULL */
    PWQ_ERR_ALIGN = 2,     /* base pointer or stride not aligned as stated below */
    PWQ_ERR_SHAPE = 3,     /* negative extent, mismatched shapes, cols % 32 (MXFP8) or % 16 (NVFP4) != 0 */
    PWQ_ERR_STRIDE = 4,    /* row stride < row length, or batch stride < rows * row stride */
    PWQ_ERR_OVERLAP = 5,   /* an output overlaps an input or another output */
    PWQ_ERR_WORKSPACE = 6, /* workspace NULL or smaller than nvfp4_workspace_size() */
    PWQ_ERR_CUDA = 7,      /* a CUDA runtime call or a kernel launch failed */
    PWQ_ERR_ARG = 8        /* other bad argument: sibling count, batch mismatch, too many tensors */
} pwq_status;

typedef struct pwq_tensor {
    void*   ptr;           /* device address of element [0][0][0] */
    int64_t batch;         /* B */
    int64_t rows;          /* M */
    int64_t cols;          /* N, logical elements per row */
    int64_t batch_stride;  /* storage units between [b][0][0] and [b+1][0][0] */
    int64_t row_stride;    /* storage units between [b][m][0] and [b][m+1][0] */
} pwq_tensor;

/* Largest number of sibling tensors in one NVFP4 group. */
#define PWQ_MAX_SIBLINGS 8

/* ===================================================================== */
/* FP8 block-wise (DeepSeek-style), 128x128 tiles                        */
/* ===================================================================== */

/* fp8_block_quant
 * Source: "Low Precision RL", "Choose a precision" table (FP8 block-wise:
 * 128x128, FP32 scales) and "Modes" 2 ("Unified block-wise FP8");
 * "低精度训练与 Rollout", "FP8 训练 + FP8 Rollout" (FP32 block scales via
 * NVTE_FP8_BLOCK_SCALING_FP32_SCALES=1).
 * For each 128x128 tile (edge tiles cover only the elements that exist):
 *   amax = max |x| over the tile, s = fl(amax / 448),
 *   q = e4m3(fl(x / s)) for every element (s == 0: q = +-0 with x's sign).
 * x      BF16 [B][M][N], any N >= 1.
 * q      E4M3 codes, same [B][M][N] shape, caller-allocated.
 * scale  FP32, dense [B][ceil(M/128)][ceil(N/128)]; s is the dequantisation
 *        multiplier (x ~= dec(q) * s).
 * Errors: PWQ_ERR_NULL, _ALIGN, _SHAPE (q shape != x shape), _STRIDE,
 * _OVERLAP, _CUDA. */
pwq_status fp8_block_quant(const pwq_tensor* x, const pwq_tensor* q, float* scale,
                           pwq_stream_t stream);

/* fp8_block_dequant
 * Source: "低精度训练与 Rollout", "FP8 训练 + FP8 Rollout" (FP8 weights are
 * dequantised to BF16 before each weight update and on checkpoint save).
 *   y = bf16(fl(dec(q) * s)) with s the element's tile scale.
 * q      E4M3 codes [B][M][N]; scale FP32 dense [B][ceil(M/128)][ceil(N/128)].
 * y      BF16 [B][M][N], caller-allocated.
 * Errors as fp8_block_quant. */
pwq_status fp8_block_dequant(const pwq_tensor* q, const float* scale, const pwq_tensor* y,
                             pwq_stream_t stream);

/* ===================================================================== */
/* MXFP8, 1x32 blocks, UE8M0 scale                                        */
/* ===================================================================== */

/* mxfp8_quant
 * Source: "Low Precision RL", "Choose a precision" table (MXFP8: 1x32, UE8M0
 * scales) and "Modes" 3 ("Unified MXFP8": power-of-two UE8M0 scales packed
 * as uint8, weights float8_e4m3fn; converter quantises tensors whose last
 * dimension is divisible by 32).
 * For each block of 32 consecutive elements of a row:
 *   e = min{k integer : amax <= 448 * 2^k} clamped to [-127, 127]
 *       (amax = 0 gives -127), scale byte = e + 127,
 *   q = e4m3(x * 2^-e) (the scaling is exact; no element saturates).
 * x      BF16 [B][M][N] with N % 32 == 0 (else PWQ_ERR_SHAPE).
 * q      E4M3 codes [B][M][N].
 * scale  uint8, dense [B][M][N/32].
 * Errors: PWQ_ERR_NULL, _ALIGN, _SHAPE, _STRIDE, _OVERLAP, _CUDA. */
pwq_status mxfp8_quant(const pwq_tensor* x, const pwq_tensor* q, uint8_t* scale,
                       pwq_stream_t stream);

/* mxfp8_dequant
 *   y = bf16(fl(dec(q) * 2^e)), e = scale byte - 127.
 * q E4M3 [B][M][N] (N % 32 == 0); scale uint8 dense [B][M][N/32];
 * y BF16 [B][M][N].  Errors as mxfp8_quant. */
pwq_status mxfp8_dequant(const pwq_tensor* q, const uint8_t* scale, const pwq_tensor* y,
                         pwq_stream_t stream);

/* ===================================================================== */
/* NVFP4, 1x16 blocks, two-level scale                                    */
/* ===================================================================== */
/*
 * Source: verl NVFP4 QAT article, section 2.3 (global scale = amax / (6 *
 * 448) in FP32, per-16 block scale in E4M3 precision, nearest E2M1 value,
 * multiply back to dequantise), 2.4 (q/k/v and gate/up fusion siblings share
 * the group's maximum amax), 2.5 / 3.3 (export: packed uint8 codes,
 * E4M3 weight_scale per 16 elements, FP32 weight_scale_2 = amax /
 * (6.0 * 448.0)); "Low Precision RL", "Choose a precision" table and
 * "Modes" 4 (NVFP4: E2M1, 1x16, two-level FP8 + FP32 scales).
 *
 * Groups.  A call takes n_siblings (1..PWQ_MAX_SIBLINGS) tensors x[0..n-1]
 * with the same batch B; group b is {x[i][b] : all i}.  A plain tensor is
 * n_siblings = 1; batched experts give one group per expert.
 *   A_b  = max |x| over every element of group b (or amax_in[b] if given),
 *   gs_b = fl(A_b / 2688)                       (2688 = 6 * 448),
 * and for each block of 16 consecutive elements of a row, with block
 * amax a:
 *   sb = e4m3(fl(a / fl(6 * gs_b)))             (gs_b == 0: sb = 0),
 *   d  = fl(dec(sb) * gs_b),
 *   c  = e2m1(fl(x / d))                        (d == 0: c = +-0),
 * and the dequantised value is y = bf16(fl((dec(c) * dec(sb)) * gs_b)).
 * Packed codes: element 2j of a row in the low nibble of byte j, 2j+1 in
 * the high nibble; bit 3 of a nibble is the sign.
 *
 * Single pass.  When amax_in is NULL, quantise and fake-quantise run as one
 * launch: a queue of amax items and encode items, ordered so that the amax
 * of the next group (or batch index) is reduced while the current one is
 * encoded from data still in L2.  The per-group amax words, completion
 * counters and queue head live in caller-provided workspace of at least
 * nvfp4_workspace_size() / nvfp4_workspace_size_grouped() bytes (4-byte
 * aligned; 256-byte aligned is best).  Its contents on entry do not matter.
 * When amax_in is given, workspace may be NULL.  Calls whose every group
 * instance has at most 131072 elements (and whose block scales are dense)
 * run one thread-block cluster per instance instead, also one launch, with
 * the group amax exchanged in distributed shared memory; the workspace is
 * still validated but not used.
 */

/* Bytes of workspace an NVFP4 quantise / fake-quantise call over these
 * siblings needs: 4 * (2 * min(B, 512) + 1), rounded up to 256.  x points
 * to n_siblings descriptors; returns 0 on bad input. */
size_t nvfp4_workspace_size(int n_siblings, const pwq_tensor* x);

/* nvfp4_group_amax: A_b for every group, as FP32, into amax_out[B] (device).
 * This is the one value a data-parallel caller must all-reduce (MAX) when a
 * group is sharded across devices, before nvfp4_quant with amax_in.
 * Errors: PWQ_ERR_NULL, _ALIGN, _SHAPE (cols % 16), _STRIDE, _ARG, _CUDA. */
pwq_status nvfp4_group_amax(const pwq_tensor* x, int n_siblings, float* amax_out,
                            pwq_stream_t stream);

/* nvfp4_quant
 * x            n_siblings BF16 descriptors [B][M_i][N_i], N_i % 16 == 0.
 * q_packed     n_siblings descriptors of packed codes, [B][M_i][N_i] logical
 *              shape (N_i / 2 bytes per row).
 * sb           host array of n_siblings device pointers, each a dense
 *              uint8 [B][M_i][N_i/16] array of E4M3 block scales.
 * global_scale FP32 [B] device output: gs_b (the dequant multiplier).
 * amax_in      optional FP32 [B] device input: precomputed / all-reduced /
 *              cached group amax; NULL = reduce it here (needs workspace).
 * Errors: PWQ_ERR_NULL, _ALIGN, _SHAPE, _STRIDE, _OVERLAP, _WORKSPACE,
 * _ARG, _CUDA. */
pwq_status nvfp4_quant(const pwq_tensor* x, int n_siblings, const pwq_tensor* q_packed,
                       uint8_t* const* sb, float* global_scale, const float* amax_in,
                       void* workspace, size_t workspace_bytes, pwq_stream_t stream);

/* nvfp4_dequant: one tensor.
 * q_packed  packed codes [B][M][N] logical shape; sb dense uint8 [B][M][N/16];
 * global_scale FP32 [B]; y BF16 [B][M][N].
 * Errors: PWQ_ERR_NULL, _ALIGN, _SHAPE, _STRIDE, _OVERLAP, _CUDA. */
pwq_status nvfp4_dequant(const pwq_tensor* q_packed, const uint8_t* sb,
                         const float* global_scale, const pwq_tensor* y, pwq_stream_t stream);

/* nvfp4_fake_quant: y = dequant(quant(x)) for every sibling, BF16 in and
 * out, without writing codes or scales; bitwise equal to nvfp4_dequant of
 * nvfp4_quant.  y[i] may be exactly x[i] (in place).  The backward of
 * fake-quantisation is the straight-through estimator (grad_x = grad_y, no
 * gradient for the scales; verl NVFP4 QAT article, section 2.3), which
 * needs no kernel.
 * amax_out optional FP32 [B] device output: the group amax that was used.
 * Errors: PWQ_ERR_NULL, _ALIGN, _SHAPE, _STRIDE, _OVERLAP, _WORKSPACE,
 * _ARG, _CUDA. */
pwq_status nvfp4_fake_quant(const pwq_tensor* x, const pwq_tensor* y, int n_siblings,
                            const float* amax_in, float* amax_out, void* workspace,
                            size_t workspace_bytes, pwq_stream_t stream);

/* ===================================================================== */
/* NVFP4 "4over6"                                                         */
/* ===================================================================== */
/*
 * Source: vime pull request #503, review thread on the NVFP4 QDQ config
 * (NVTE_NVFP4_4OVER6 switches the variant on; NVTE_NVFP4_4OVER6_E4M3_USE_256
 * makes the E4M3 maximum of the global scale 256 instead of 448, and
 * defaults to on with the variant).  The pages name the variant and the
 * constant only; the per-block rule below is this library's reading, taken
 * from the variant's name (a block's amax maps to 4 or to 6):
 *   gs_b = fl(A_b / (6 E)),                     E = e4m3_max (256 or 448),
 * and for each block, for t = 6 and t = 4:
 *   sb_t = e4m3(fl(a / fl(t * gs_b))),  codes and values y_t as in NVFP4,
 *   err_t = fl(fl(x_0 - y_t,0)^2) + ... + fl(fl(x_15 - y_t,15)^2), added
 *           left to right in binary32;
 * the block keeps t = 4 when err_4 < err_6, else t = 6.  With E = 256 the
 * block scale of t = 4 stays below 384, inside E4M3.  The result is plain
 * NVFP4 (nvfp4_dequant reads it); siblings, layouts, amax_in and amax_out
 * are those of nvfp4_quant / nvfp4_fake_quant.
 *
 * The grouped forms take several sibling groups with the layout rules of
 * nvfp4_quant_grouped / nvfp4_fake_quant_grouped (the amax is always
 * reduced on the device).
 *
 * Two launches per PWQ_LAUNCH_TENSORS members: the group amaxes (skipped
 * when amax_in is given) into workspace of at least
 * nvfp4_4over6_workspace_size() / _grouped() bytes (4-byte aligned; 4 bytes
 * per batch index of every group, rounded up to 256; its contents on entry
 * do not matter), then one encode launch that evaluates both candidates of
 * every block.
 * Errors: PWQ_ERR_NULL, _ALIGN, _SHAPE, _STRIDE, _OVERLAP, _WORKSPACE,
 * _ARG (e4m3_max not 256 or 448, n_siblings / group sizes), _CUDA. */
size_t nvfp4_4over6_workspace_size(int n_siblings, const pwq_tensor* x);
pwq_status nvfp4_4over6_quant(const pwq_tensor* x, int n_siblings, const pwq_tensor* q_packed,
                              uint8_t* const* sb, float* global_scale, const float* amax_in, int e4m3_max,
                              void* workspace, size_t workspace_bytes, pwq_stream_t stream);
pwq_status nvfp4_4over6_fake_quant(const pwq_tensor* x, const pwq_tensor* y, int n_siblings,
                                   const float* amax_in, float* amax_out, int e4m3_max, void* workspace,
                                   size_t workspace_bytes, pwq_stream_t stream);
size_t nvfp4_4over6_workspace_size_grouped(int n_groups, const int* group_sizes, const pwq_tensor* x);
pwq_status nvfp4_4over6_quant_grouped(int n_groups, const int* group_sizes, const pwq_tensor* x,
                                      const pwq_tensor* q_packed, uint8_t* const* sb,
                                      float* const* global_scale, int e4m3_max, void* workspace,
                                      size_t workspace_bytes, pwq_stream_t stream);
pwq_status nvfp4_4over6_fake_quant_grouped(int n_groups, const int* group_sizes, const pwq_tensor* x,
                                           const pwq_tensor* y, float* const* amax_out, int e4m3_max,
                                           void* workspace, size_t workspace_bytes, pwq_stream_t stream);

/* ===================================================================== */
/* Grouped calls: a list of independent tensors in one launch             */
/* ===================================================================== */
/*
 * Source: verl NVFP4 QAT article, section 2.5 (the exporter buffers one
 * decoder layer's parameters and quantises the layer at once) and section
 * 3.3 (per-parameter export inside the weight-update stream); "Low Precision
 * RL", "Unified training recipe" (weights re-quantised on every weight
 * update).  Each grouped call computes exactly what the single-tensor call
 * computes for every tensor of the list, with one kernel launch per
 * PWQ_LAUNCH_TENSORS tensors, so small tensors (k/v projections) no longer
 * pay a launch and a ramp each.  n is the list length (0 .. PWQ_MAX_GROUPED;
 * 0 is a no-op); x, q, y are host arrays of n descriptors; scale, sb and
 * global_scale are host arrays of n device pointers with the per-tensor
 * layouts of the single-tensor calls.  No output may overlap any input or
 * another output of the list.  Errors: as the single-tensor calls, plus
 * PWQ_ERR_ARG for n out of range.
 */
#define PWQ_MAX_GROUPED 256
#define PWQ_LAUNCH_TENSORS 16

pwq_status fp8_block_quant_grouped(int n, const pwq_tensor* x, const pwq_tensor* q,
                                   float* const* scale, pwq_stream_t stream);
pwq_status fp8_block_dequant_grouped(int n, const pwq_tensor* q, const float* const* scale,
                                     const pwq_tensor* y, pwq_stream_t stream);
pwq_status mxfp8_quant_grouped(int n, const pwq_tensor* x, const pwq_tensor* q,
                               uint8_t* const* scale, pwq_stream_t stream);
pwq_status mxfp8_dequant_grouped(int n, const pwq_tensor* q, const uint8_t* const* scale,
                                 const pwq_tensor* y, pwq_stream_t stream);
pwq_status nvfp4_dequant_grouped(int n, const pwq_tensor* q_packed, const uint8_t* const* sb,
                                 const float* const* global_scale, const pwq_tensor* y,
                                 pwq_stream_t stream);

/* NVFP4 over several sibling groups (e.g. {q,k,v}, {o}, {gate,up}, {down}
 * of one layer): group g has group_sizes[g] consecutive members of x (and
 * of q_packed / sb / y), 1 <= group_sizes[g] <= PWQ_MAX_SIBLINGS, at most
 * PWQ_MAX_GROUPED members in all; members of a group share one batch B_g and
 * one amax per batch index.  global_scale[g] (quantise) and amax_out[g]
 * (fake-quantise; the array or any entry may be NULL) are per-group FP32
 * [B_g] device arrays.  The amax is always reduced on the device: workspace
 * of at least nvfp4_workspace_size_grouped() bytes is required. */
size_t nvfp4_workspace_size_grouped(int n_groups, const int* group_sizes, const pwq_tensor* x);
pwq_status nvfp4_quant_grouped(int n_groups, const int* group_sizes, const pwq_tensor* x,
                               const pwq_tensor* q_packed, uint8_t* const* sb,
                               float* const* global_scale, void* workspace,
                               size_t workspace_bytes, pwq_stream_t stream);
pwq_status nvfp4_fake_quant_grouped(int n_groups, const int* group_sizes, const pwq_tensor* x,
                                    const pwq_tensor* y, float* const* amax_out, void* workspace,
                                    size_t workspace_bytes, pwq_stream_t stream);

/* nvfp4_fake_quant_noalloc
 * The pages have no counterpart to this entry point; it exists for callers
 * that cannot allocate device memory.  Such callers include code running
 * inside a framework or plugin host that owns all device memory and offers
 * no allocator, real-time loops that forbid allocation after start-up, and
 * steps where a cudaMalloc would be unacceptable because it can implicitly
 * synchronise the device.  It computes exactly what nvfp4_fake_quant
 * computes, with the same arguments minus the workspace: the per-group amax
 * scratch lives in a file-scope device array of the library instead.
 * Limits and behaviour:
 *   - at most 4096 groups (batch) per call when amax_in is NULL; larger
 *     batches return PWQ_ERR_SHAPE (with amax_in the scratch is unused);
 *   - the array takes 16 KB on every device that loads the library, held
 *     until the process exits;
 *   - the first call on a device looks up the array's device address (with
 *     that device current) and caches it; make that first call before any
 *     stream capture;
 *   - every call shares the one array and it keeps the last call's contents
 *     (each call clears the words it needs before using them), so calls
 *     that may overlap on the GPU -- on different streams without ordering
 *     between them, or from several host threads -- race: order them;
 *   - a call whose every group has at most 131072 elements runs one
 *     thread-block cluster per group (the path nvfp4_fake_quant takes for
 *     such calls) and does not touch the array, so such calls do not race;
 *   - it calls no cudaMalloc, cudaFree or other allocating routine.
 * Errors as nvfp4_fake_quant, except that there is no PWQ_ERR_WORKSPACE. */
pwq_status nvfp4_fake_quant_noalloc(const pwq_tensor* x, const pwq_tensor* y, int n_siblings,
                                    const float* amax_in, float* amax_out, pwq_stream_t stream);

/* ===================================================================== */
/* Block scales in the tensor-core (block-scaled MMA) layout              */
/* ===================================================================== */
/*
 * The rollout GEMM consumes the quantised weights ("Low Precision RL",
 * "Modes" 3; the NVFP4 exporter repacks the scales for the inference
 * kernels, verl NVFP4 QAT article 2.5); the pages do not give the layout
 * such a GEMM reads.  The one used here is the layout in which the sm_100
 * block-scaled tensor-core MMA takes its scale factors (NVIDIA PTX ISA,
 * tcgen05.mma with block scaling and tcgen05.cp's 32x128b.warpx4 shape;
 * cuBLAS documentation, 1D block-scaling-factor layout).  For an [B][M][S]
 * array of scale bytes (S = N / 32 for MXFP8, N / 16 for NVFP4), every
 * batch slab is ceil(M/128) x ceil(S/4) tiles of 512 contiguous bytes;
 * tiles follow each other along S within a 128-row band, then band after
 * band; the scale of tile row r (0..127) and column c (0..3) is at byte
 * (r % 32) * 16 + (r / 32) * 4 + c of its tile.  Rows past M and columns
 * past S are zero bytes (the calls below write them).
 */

/* Bytes of one such array: B * ceil(M/128) * ceil(S/4) * 512 (0 on negative input). */
size_t pwq_mma_scale_bytes(int64_t batch, int64_t rows, int64_t scale_cols);

/* Dense [B][M][S] scale bytes -> the tile layout (padding written as zero),
 * and back (padding ignored).  mma: 16-byte aligned device array of
 * pwq_mma_scale_bytes() bytes; dense: device array of B*M*S bytes.  The two
 * may not overlap.  Errors: PWQ_ERR_NULL, _ALIGN, _SHAPE, _OVERLAP, _CUDA. */
pwq_status pwq_scales_to_mma(const uint8_t* dense, int64_t batch, int64_t rows, int64_t scale_cols, uint8_t* mma,
                             pwq_stream_t stream);
pwq_status pwq_scales_from_mma(const uint8_t* mma, int64_t batch, int64_t rows, int64_t scale_cols, uint8_t* dense,
                               pwq_stream_t stream);

/* mxfp8_quant_grouped / nvfp4_quant_grouped writing every tensor's block
 * scales straight into the tile layout (scale_mma[i] / sb_mma[i]: device
 * arrays of pwq_mma_scale_bytes(B, M, N/32) / (B, M, N/16) bytes, any
 * alignment); codes, global scales and every other rule as the dense
 * calls.  When M % 128 or S % 4 is not zero the call first clears the
 * array (one memset on the stream) so that the padding is zero. */
pwq_status mxfp8_quant_grouped_mma(int n, const pwq_tensor* x, const pwq_tensor* q, uint8_t* const* scale_mma,
                                   pwq_stream_t stream);
pwq_status nvfp4_quant_grouped_mma(int n_groups, const int* group_sizes, const pwq_tensor* x,
                                   const pwq_tensor* q_packed, uint8_t* const* sb_mma, float* const* global_scale,
                                   void* workspace, size_t workspace_bytes, pwq_stream_t stream);

/* ===================================================================== */
/* FP8 block-wise weights into a rollout format                           */
/* ===================================================================== */

/* "低精度训练与 Rollout", "FP8 训练 + FP8 Rollout" / "实现说明" item 3: on a
 * weight update the FP8 training weights are dequantised to BF16 and the
 * BF16 weights quantised into the rollout format.  These calls compute
 * exactly that composition in one pass, without the BF16 tensor in memory:
 * the input is FP8 block-wise (E4M3 codes q [B][M][N], FP32 tile scales
 * s [B][ceil(M/128)][ceil(N/128)], as fp8_block_quant writes them), the
 * values are y = bf16(fl(dec(q) * s)) as fp8_block_dequant computes them,
 * and the outputs are bit for bit those of the named quantiser applied to
 * y.  Code tensors: 8-byte aligned base and row stride (bytes = elements).
 * Same error codes as the quantisers; no call allocates. */

/* fp8_block_requant: FP8 block-wise -> FP8 block-wise with fresh tile
 * scales, fp8_block_quant(fp8_block_dequant(q, s)).  q_out may be q exactly
 * and scale_out may be scale_in (in place); other overlaps are
 * PWQ_ERR_OVERLAP.  Any N. */
pwq_status fp8_block_requant(const pwq_tensor* q_in, const float* scale_in, const pwq_tensor* q_out,
                             float* scale_out, pwq_stream_t stream);

/* fp8_block_requant_mxfp8: FP8 block-wise -> MXFP8,
 * mxfp8_quant(fp8_block_dequant(q, s)): codes into q_out (same shape; may
 * be q_in exactly), UE8M0 bytes into scale_ue8m0 [B][M][N/32].  N % 32 == 0
 * (a 1x32 block then never leaves its 128-wide tile). */
pwq_status fp8_block_requant_mxfp8(const pwq_tensor* q_in, const float* scale_in, const pwq_tensor* q_out,
                                   uint8_t* scale_ue8m0, pwq_stream_t stream);

/* Grouped forms: n tensors (at most 256; one launch per 16), e.g. the seven
 * weights of a decoder layer; q_in / q_out / scale arrays indexed alike,
 * each tensor under the rules of the single call.  The MXFP8 form reads 16
 * codes per 16-byte load when every code tensor of the call has 16-byte
 * aligned base and strides, and falls back to one launch per tensor with
 * 8-byte loads otherwise. */
pwq_status fp8_block_requant_grouped(int n, const pwq_tensor* q_in, const float* const* scale_in,
                                     const pwq_tensor* q_out, float* const* scale_out, pwq_stream_t stream);
pwq_status fp8_block_requant_mxfp8_grouped(int n, const pwq_tensor* q_in, const float* const* scale_in,
                                           const pwq_tensor* q_out, uint8_t* const* scale_ue8m0,
                                           pwq_stream_t stream);

/* Bytes of workspace fp8_block_requant_nvfp4 / _grouped need: as
 * nvfp4_workspace_size / nvfp4_workspace_size_grouped for the same shapes;
 * 0 on bad input. */
size_t fp8_block_requant_nvfp4_workspace_size(int n_siblings, const pwq_tensor* q_in);
size_t fp8_block_requant_nvfp4_workspace_size_grouped(int n_groups, const int* group_sizes,
                                                      const pwq_tensor* q_in);

/* fp8_block_requant_nvfp4: a sibling group of FP8 block-wise members ->
 * NVFP4, nvfp4_quant(fp8_block_dequant(q_i, s_i) for every member i): the
 * group amax is taken over the dequantised members (per batch index), then
 * every member is encoded with it.  q_in: n_siblings code tensors (N % 16
 * == 0, same batch), scale_in: their tile scales; outputs as nvfp4_quant
 * (q_packed, sb [B][M][N/16] per member, global_scale [B]).  amax_in
 * (device, [B], nullable) replaces the reduction, e.g. after an all-reduce
 * of a sharded group; otherwise workspace of
 * fp8_block_requant_nvfp4_workspace_size() bytes is required. */
pwq_status fp8_block_requant_nvfp4(const pwq_tensor* q_in, const float* const* scale_in, int n_siblings,
                                   const pwq_tensor* q_packed, uint8_t* const* sb, float* global_scale,
                                   const float* amax_in, void* workspace, size_t workspace_bytes,
                                   pwq_stream_t stream);

/* fp8_block_requant_nvfp4_grouped: several sibling groups in one call (e.g.
 * a decoder layer's {q,k,v}, {o}, {gate,up}, {down}), laid out as in
 * nvfp4_quant_grouped: group g has group_sizes[g] members, consecutive in
 * q_in / scale_in / q_packed / sb, and writes global_scale[g] ([B_g]).
 * Without amax_in the group amax is reduced on the device in the same
 * single-pass launch that encodes (the codes are read once for the amax and
 * once more, mostly from L2, for the encode pass). */
pwq_status fp8_block_requant_nvfp4_grouped(int n_groups, const int* group_sizes, const pwq_tensor* q_in,
                                           const float* const* scale_in, const pwq_tensor* q_packed,
                                           uint8_t* const* sb, float* const* global_scale, void* workspace,
                                           size_t workspace_bytes, pwq_stream_t stream);

/* ===================================================================== */
/* W4A4 activation observers                                              */
/* ===================================================================== */

/* verl NVFP4 QAT article, 2.2 and 3.1: in W4A4 mode each activation has its
 * own NVFP4 global scale (input_global_scale), kept by an activation observer
 * named static_minmax (the default), memoryless_minmax or minmax.  The pages
 * give only the names; this library reads them as follows.  The observer
 * state is two binary32 values (lo, hi), the minimum and maximum of the
 * values observed so far, numerically ordered with -0 < +0; an empty state
 * is (+inf, -inf) (any lo > hi), which the caller writes once.  One step on
 * a tensor x with extremes (mn, mx):
 *   PWQ_OBSERVER_MEMORYLESS_MINMAX  (lo, hi) = (mn, mx);
 *   PWQ_OBSERVER_STATIC_MINMAX      (lo, hi) = (min(lo, mn), max(hi, mx));
 *   PWQ_OBSERVER_MINMAX             moving average with constant c in [0, 1]:
 *       an empty state takes (mn, mx), otherwise
 *       lo = fl(fl(fl(1 - c) * lo) + fl(c * mn)) and hi alike;
 * then A = max(|lo|, |hi|) and input_global_scale = fl(A / 2688), as the
 * weight global scale.  Quantising the activation is then nvfp4_fake_quant
 * (or nvfp4_quant) with amax_in = A: the step observes, then quantises. */
#define PWQ_OBSERVER_MEMORYLESS_MINMAX 0
#define PWQ_OBSERVER_STATIC_MINMAX 1
#define PWQ_OBSERVER_MINMAX 2

/* Bytes of workspace nvfp4_activation_observe needs (256). */
size_t nvfp4_observe_workspace_size(void);

/* nvfp4_activation_observe: one observer step over every element of x
 * (BF16 [B][M][N], N % 16 == 0; the whole tensor is one observation).
 * state: device float[2], read and written.  amax_out, input_global_scale:
 * device float[1] each, nullable.  averaging_constant is used by
 * PWQ_OBSERVER_MINMAX only (PWQ_ERR_ARG outside [0, 1]).  An empty x leaves
 * everything unchanged.  Errors: PWQ_ERR_NULL, _ALIGN, _SHAPE, _STRIDE,
 * _OVERLAP, _WORKSPACE, _ARG, _CUDA. */
pwq_status nvfp4_activation_observe(const pwq_tensor* x, int observer, float averaging_constant, float* state,
                                    float* amax_out, float* input_global_scale, void* workspace,
                                    size_t workspace_bytes, pwq_stream_t stream);

/* ===================================================================== */
/* Diagnostics                                                            */
/* ===================================================================== */

/* Human-readable name of a status code (static string). */
const char* pwq_status_string(pwq_status status);

/* One line on the most recent failure in the calling thread: the argument
 * that failed validation, or the CUDA error name and message. */
const char* pwq_last_error_detail(void);

/* Build description: target architecture and the exact-math compiler flags
 * (static string). */
const char* pwq_build_info(void);

/* Reads and clears the device-side error word of the current device
 * (synchronous; 0 = no error; bit 0 = a TMA load wait gave up, bit 1 = an
 * NVFP4 single-pass encode item gave up waiting for its group amax).  When
 * a bit is set, the outputs of the calls since the previous read are
 * unspecified.  Returns PWQ_ERR_NULL or PWQ_ERR_CUDA on failure. */
pwq_status pwq_device_error(uint32_t* code);

/* Exhaustive self-check of the device arithmetic against CUDA's IEEE
 * division (__fdiv_rn), for every divisor the formats can produce and every
 * finite BF16 numerator that can be paired with it:
 *   which = 0  FP8 block code divisor s = fl(a / 448), a every positive
 *              finite BF16; numerators |x| <= a.  Compares E4M3 codes.
 *   which = 1  NVFP4 code divisor d = fl(dec(sb) * fl(a / 2688)) for every
 *              positive finite BF16 a and every non-zero E4M3 sb;
 *              numerators |x| <= 16 d.  Compares E2M1 codes.
 *   which = 2  NVFP4 block-scale divisor fl(6 * fl(a / 2688)); numerators
 *              |x| <= a.  Compares E4M3 codes.
 *   which = 3  FP8 tile scale s = fl(a / 448) as the kernels form it, for
 *              every BF16 amax a >= 0: [0] = values checked, [1] = [2] =
 *              binary32 mismatches against __fdiv_rn (s is stored, so it
 *              must be exact), [3] = values taking the IEEE path.
 *   which = 4  BF16 magnitude max (bf16x2 abs-max form) against the
 *              integer max of the magnitude bits, for every ordered pair of
 *              finite BF16 values: [0] = pairs, [1] = mismatches.
 *   which = 5  NVFP4 dequantisation through an exact binary16 product
 *              against the binary32 form bf16(fl(fl(dec(c) dec(sb)) gs)),
 *              for every E2M1 code pair, block scale code 0..126 and global
 *              scale fl(a / 2688) (a = 0 or a positive finite BF16):
 *              [0] = code pairs, [1] = mismatching BF16 pairs.
 *   which = 6  as 1 with the 4over6 global scale fl(a / 1536) (E = 256).
 *   which = 7  as 2 with fl(6 * fl(a / 1536)).
 *   which = 8  the 4over6 block-scale divisor of the candidate 4,
 *              fl(4 * fl(a / 1536)); numerators |x| <= a.
 *   which = 9  as 8 with fl(4 * fl(a / 2688)) (E = 448).
 * counts (device, 4 x uint64, zeroed by the call): [0] pairs checked,
 * [1] code mismatches, [2] binary32 quotient mismatches where |x| >= 2^-100
 * and the IEEE quotient is normal, [3] pairs whose divisor takes the
 * IEEE-division path instead of the reciprocal path.  Asynchronous. */
pwq_status pwq_selftest_division(int which, unsigned long long* counts, pwq_stream_t stream);

/* Self-test of the bounded wait of the NVFP4 single-pass kernel (the wait
 * of an encode item for its group's amax, which normal calls bound at 2 s).
 * It runs nvfp4_fake_quant of one BF16 tensor x ([B][M][N], B <= 512,
 * N % 16 == 0, non-empty) into y through the single-pass kernel with that
 * limit set to wait_ns (1 us .. 2 s) and with every encode item waiting on
 * a completion count that no amax item adds to, so every such wait runs
 * out.  Expected: the kernel returns after about wait_ns per waiting CTA,
 * pwq_device_error() then reports bit 1, and y is unspecified; nothing
 * faults or hangs, and the next call runs normally.  workspace: device,
 * at least pwq_selftest_flow_timeout_workspace_size(x) bytes (0 on bad x).
 * Errors: PWQ_ERR_NULL, _ALIGN, _SHAPE, _STRIDE, _OVERLAP, _WORKSPACE,
 * _ARG (wait_ns out of range), _CUDA. */
size_t pwq_selftest_flow_timeout_workspace_size(const pwq_tensor* x);
pwq_status pwq_selftest_flow_timeout(const pwq_tensor* x, const pwq_tensor* y, uint64_t wait_ns, void* workspace,
                                     size_t workspace_bytes, pwq_stream_t stream);

/* Runs the device codecs over `count` consecutive binary32 bit patterns
 * starting at `first`
 * and writes: e4m3 codes (count bytes), e2m1 codes (count bytes, one code
 * per byte), bf16 bit patterns (count x uint16).  Any of the outputs may be
 * NULL.  Used to compare the device conversions with the oracle. */
pwq_status pwq_selftest_codecs(uint32_t first, uint32_t count, uint8_t* e4m3, uint8_t* e2m1,
                               uint16_t* bf16, pwq_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* PWQ_H */
