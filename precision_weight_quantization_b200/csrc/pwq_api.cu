// pwq_api.cu -- the extern "C" entry points declared in include/pwq.h:
// argument validation (null, alignment, shape, stride, overlap, workspace),
// conversion to byte-stride views and dispatch to the kernel launchers.
// Nothing here allocates device memory or synchronises.
#include <algorithm>
#include <atomic>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <vector>

#include "pwq.h"
#include "pwq_internal.h"

#ifndef PWQ_BUILD_FLAGS
#define PWQ_BUILD_FLAGS "unknown"
#endif

namespace pwq {

int current_device() {
    int d = 0;
    if (cudaGetDevice(&d) != cudaSuccess) return 0;
    return d;
}

int sm_count(int device) {
    static std::atomic<int> cache[kMaxDevices] = {};
    const bool cacheable = device >= 0 && device < kMaxDevices;
    if (cacheable) {
        const int c = cache[device].load(std::memory_order_relaxed);
        if (c > 0) return c;
    }
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, device) != cudaSuccess || n <= 0) n = 148;
    if (cacheable) cache[device].store(n, std::memory_order_relaxed);
    return n;
}

cudaError_t set_smem_limit_once(int* done, const void* const* fns, int n, int bytes) {
    static std::mutex mu;
    const int dev = current_device();
    std::lock_guard<std::mutex> lock(mu);
    if (dev >= 0 && dev < kMaxDevices && done[dev]) return cudaSuccess;
    for (int f = 0; f < n; ++f) {
        const cudaError_t e = cudaFuncSetAttribute(fns[f], cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
        if (e != cudaSuccess) return e;
    }
    if (dev >= 0 && dev < kMaxDevices) done[dev] = 1;
    return cudaSuccess;
}

int persistent_grid(int64_t work_ctas, int per_sm) {
    const int64_t cap = (int64_t)sm_count(current_device()) * per_sm;
    return (int)std::max<int64_t>(1, std::min<int64_t>(work_ctas, cap));
}

}  // namespace pwq

namespace {

using pwq::Job;
using pwq::View;

thread_local char g_detail[256] = "";

pwq_status fail(pwq_status st, const char* what) {
    std::snprintf(g_detail, sizeof(g_detail), "%s", what);
    return st;
}

pwq_status cuda_fail(cudaError_t e) {
    std::snprintf(g_detail, sizeof(g_detail), "%s: %s", cudaGetErrorName(e), cudaGetErrorString(e));
    return PWQ_ERR_CUDA;
}

pwq_status from_cuda(cudaError_t e) { return e == cudaSuccess ? PWQ_OK : cuda_fail(e); }

enum class Kind { kBF16, kByte, kPacked4 };

struct Extent {
    uintptr_t lo = 0, hi = 0;  // [lo, hi) in bytes; empty when lo == hi
};

bool overlaps(const Extent& a, const Extent& b) { return a.lo < a.hi && b.lo < b.hi && a.lo < b.hi && b.lo < a.hi; }

Extent extent_of(const void* p, size_t bytes) {
    Extent e;
    e.lo = (uintptr_t)p;
    e.hi = e.lo + bytes;
    return e;
}

bool empty(const pwq_tensor* t) { return t->batch == 0 || t->rows == 0 || t->cols == 0; }

constexpr int64_t kMaxDim = (int64_t(1) << 31) - 1;
// chunk (8-element) and tile counts of one tensor stay below 2^31
constexpr int64_t kMaxChunks = (int64_t(1) << 31) - 1024;

// Validates one tensor descriptor; fills a byte-stride view and its extent.
pwq_status check_tensor(const pwq_tensor* t, Kind k, View* v, Extent* ext, const char* name) {
    if (!t) return fail(PWQ_ERR_NULL, name);
    if (t->batch < 0 || t->rows < 0 || t->cols < 0 || t->batch > kMaxDim || t->rows > kMaxDim ||
        t->cols > kMaxDim)
        return fail(PWQ_ERR_SHAPE, name);
    const int64_t unit = (k == Kind::kBF16) ? 2 : 1;
    const int64_t row_units = (k == Kind::kPacked4) ? (t->cols + 1) / 2 : t->cols;
    v->ptr = static_cast<char*>(t->ptr);
    v->batch = t->batch;
    v->rows = t->rows;
    v->cols = t->cols;
    v->bstride = t->batch_stride * unit;
    v->rstride = t->row_stride * unit;
    if (empty(t)) {
        *ext = Extent{};
        return PWQ_OK;
    }
    if (!t->ptr) return fail(PWQ_ERR_NULL, name);
    if ((t->batch * t->rows) > kMaxDim || t->batch * t->rows * ((t->cols + 7) / 8) > kMaxChunks)
        return fail(PWQ_ERR_SHAPE, "tensor too large (more than 2^31 8-element chunks)");
    // BF16 rows are moved in 16-byte vectors (and by TMA); code rows in
    // 8-byte (E4M3) or 4-byte (packed E2M1) pieces
    const int64_t align = (k == Kind::kBF16) ? 16 : 8;
    if ((uintptr_t)t->ptr % align != 0 || (t->row_stride * unit) % align != 0 ||
        (t->batch > 1 && (t->batch_stride * unit) % align != 0))
        return fail(PWQ_ERR_ALIGN, name);
    if (t->row_stride < row_units || (t->batch > 1 && t->batch_stride < t->rows * t->row_stride))
        return fail(PWQ_ERR_STRIDE, name);
    const int64_t last = (t->batch - 1) * v->bstride + (t->rows - 1) * v->rstride + row_units * unit;
    *ext = extent_of(t->ptr, (size_t)last);
    return PWQ_OK;
}

bool same_shape(const pwq_tensor* a, const pwq_tensor* b) {
    return a->batch == b->batch && a->rows == b->rows && a->cols == b->cols;
}

bool exact_alias(const pwq_tensor* a, const pwq_tensor* b) {
    return a->ptr == b->ptr && same_shape(a, b) && a->row_stride == b->row_stride &&
           (a->batch <= 1 || a->batch_stride == b->batch_stride);
}

// Fails if any output extent intersects an input extent or another output.
pwq_status check_overlaps(const Extent* in, int n_in, const Extent* out, int n_out) {
    for (int i = 0; i < n_out; ++i) {
        for (int j = 0; j < n_in; ++j)
            if (overlaps(out[i], in[j])) return fail(PWQ_ERR_OVERLAP, "output overlaps an input");
        for (int j = i + 1; j < n_out; ++j)
            if (overlaps(out[i], out[j])) return fail(PWQ_ERR_OVERLAP, "two outputs overlap");
    }
    return PWQ_OK;
}

int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

// ------------------------------------------------------------------ elementwise ops over tensor lists

enum class Op { kFp8Quant, kFp8Dequant, kMxQuant, kMxDequant, kNvDequant };

// in / out kinds and the scale array size (bytes) of one tensor
struct OpSpec {
    Kind in, out;
    const char* name;
};

OpSpec spec(Op op) {
    switch (op) {
        case Op::kFp8Quant: return {Kind::kBF16, Kind::kByte, "fp8_block_quant"};
        case Op::kFp8Dequant: return {Kind::kByte, Kind::kBF16, "fp8_block_dequant"};
        case Op::kMxQuant: return {Kind::kBF16, Kind::kByte, "mxfp8_quant"};
        case Op::kMxDequant: return {Kind::kByte, Kind::kBF16, "mxfp8_dequant"};
        case Op::kNvDequant: return {Kind::kPacked4, Kind::kBF16, "nvfp4_dequant"};
    }
    return {Kind::kBF16, Kind::kBF16, "?"};
}

size_t scale_bytes(Op op, const pwq_tensor* t) {
    switch (op) {
        case Op::kFp8Quant:
        case Op::kFp8Dequant: return (size_t)(t->batch * ceil_div(t->rows, 128) * ceil_div(t->cols, 128)) * 4;
        case Op::kMxQuant:
        case Op::kMxDequant: return (size_t)(t->batch * t->rows * (t->cols / 32));
        case Op::kNvDequant: return (size_t)(t->batch * t->rows * (t->cols / 16));
    }
    return 0;
}

// Validates n (in, out, scale[, gs]) tensors and launches them as one
// grouped call.  scale[i] is an input for dequantise ops and an output for
// quantise ops; gs (NVFP4 dequant only) an input.
pwq_status run_list(Op op, int n, const pwq_tensor* in, const pwq_tensor* out, void* const* scale,
                    const float* const* gs, pwq_stream_t stream, bool scale_mma = false) {
    if (n < 0 || n > PWQ_MAX_GROUPED) return fail(PWQ_ERR_ARG, "tensor count out of range");
    if (n == 0) return PWQ_OK;
    if (!in || !out || !scale) return fail(PWQ_ERR_NULL, "tensor or scale array");
    if (op == Op::kNvDequant && !gs) return fail(PWQ_ERR_NULL, "global_scale array");
    const OpSpec sp = spec(op);
    const bool quant = (op == Op::kFp8Quant || op == Op::kMxQuant);
    std::vector<Job> jobs;
    std::vector<Extent> ins, outs;
    jobs.reserve(n);
    for (int i = 0; i < n; ++i) {
        const pwq_tensor* a = &in[i];
        const pwq_tensor* b = &out[i];
        if (!same_shape(a, b)) return fail(PWQ_ERR_SHAPE, "output shape != input shape");
        Job j;
        Extent ea, eb;
        pwq_status st;
        if ((st = check_tensor(a, sp.in, &j.in, &ea, "input")) != PWQ_OK) return st;
        if ((st = check_tensor(b, sp.out, &j.out, &eb, "output")) != PWQ_OK) return st;
        if ((op == Op::kMxQuant || op == Op::kMxDequant) && a->cols % 32 != 0)
            return fail(PWQ_ERR_SHAPE, "cols % 32 != 0");
        if (op == Op::kNvDequant && a->cols % 16 != 0) return fail(PWQ_ERR_SHAPE, "cols % 16 != 0");
        if (empty(a)) continue;
        if (!scale[i]) return fail(PWQ_ERR_NULL, "scale");
        const bool fp8 = (op == Op::kFp8Quant || op == Op::kFp8Dequant);
        if (fp8 && (uintptr_t)scale[i] % 4 != 0) return fail(PWQ_ERR_ALIGN, "scale");
        j.scale = scale[i];
        j.gs = nullptr;
        j.scale_mma = scale_mma ? 1 : 0;
        const Extent es = extent_of(scale[i], scale_mma ? (size_t)(a->batch * pwq::mma_scale_slab_bytes(
                                                              a->rows, a->cols / 32))
                                                        : scale_bytes(op, a));
        ins.push_back(ea);
        outs.push_back(eb);
        (quant ? outs : ins).push_back(es);
        if (op == Op::kNvDequant) {
            if (!gs[i]) return fail(PWQ_ERR_NULL, "global_scale");
            if ((uintptr_t)gs[i] % 4 != 0) return fail(PWQ_ERR_ALIGN, "global_scale");
            j.gs = gs[i];
            ins.push_back(extent_of(gs[i], (size_t)a->batch * 4));
        }
        jobs.push_back(j);
    }
    pwq_status st = check_overlaps(ins.data(), (int)ins.size(), outs.data(), (int)outs.size());
    if (st != PWQ_OK) return st;
    if (jobs.empty()) return PWQ_OK;
    cudaStream_t s = (cudaStream_t)stream;
    const int m = (int)jobs.size();
    if (scale_mma)
        for (const Job& j : jobs)
            if (pwq::mma_scale_padded(j.in.rows, j.in.cols / 32)) {
                cudaError_t e = cudaMemsetAsync(
                    j.scale, 0, (size_t)(j.in.batch * pwq::mma_scale_slab_bytes(j.in.rows, j.in.cols / 32)), s);
                if (e != cudaSuccess) return cuda_fail(e);
            }
    switch (op) {
        case Op::kFp8Quant: return from_cuda(pwq::launch_fp8_block_quant(jobs.data(), m, s));
        case Op::kFp8Dequant: return from_cuda(pwq::launch_fp8_block_dequant(jobs.data(), m, s));
        case Op::kMxQuant: return from_cuda(pwq::launch_mxfp8_quant(jobs.data(), m, s));
        case Op::kMxDequant: return from_cuda(pwq::launch_mxfp8_dequant(jobs.data(), m, s));
        case Op::kNvDequant: return from_cuda(pwq::launch_nvfp4_dequant(jobs.data(), m, s));
    }
    return fail(PWQ_ERR_ARG, "op");
}

}  // namespace

extern "C" {

const char* pwq_status_string(pwq_status s) {
    switch (s) {
        case PWQ_OK: return "PWQ_OK";
        case PWQ_ERR_NULL: return "PWQ_ERR_NULL";
        case PWQ_ERR_ALIGN: return "PWQ_ERR_ALIGN";
        case PWQ_ERR_SHAPE: return "PWQ_ERR_SHAPE";
        case PWQ_ERR_STRIDE: return "PWQ_ERR_STRIDE";
        case PWQ_ERR_OVERLAP: return "PWQ_ERR_OVERLAP";
        case PWQ_ERR_WORKSPACE: return "PWQ_ERR_WORKSPACE";
        case PWQ_ERR_CUDA: return "PWQ_ERR_CUDA";
        case PWQ_ERR_ARG: return "PWQ_ERR_ARG";
    }
    return "PWQ_ERR_UNKNOWN";
}

const char* pwq_last_error_detail(void) { return g_detail; }

const char* pwq_build_info(void) { return "libpwq sm_100a; " PWQ_BUILD_FLAGS; }

pwq_status pwq_device_error(uint32_t* code) {
    if (!code) return fail(PWQ_ERR_NULL, "code");
    uint32_t a = 0, b = 0;
    cudaError_t e = pwq::read_and_clear_device_error(&a);
    if (e != cudaSuccess) return cuda_fail(e);
    e = pwq::read_and_clear_flow_error(&b);
    if (e != cudaSuccess) return cuda_fail(e);
    *code = a | b;
    return PWQ_OK;
}

// ------------------------------------------------------------------ FP8 block-wise, MXFP8, NVFP4 dequant

pwq_status fp8_block_quant(const pwq_tensor* x, const pwq_tensor* q, float* scale, pwq_stream_t stream) {
    if (!x || !q) return fail(PWQ_ERR_NULL, "tensor descriptor");
    void* sc[1] = {scale};
    return run_list(Op::kFp8Quant, 1, x, q, sc, nullptr, stream);
}

pwq_status fp8_block_dequant(const pwq_tensor* q, const float* scale, const pwq_tensor* y,
                             pwq_stream_t stream) {
    if (!q || !y) return fail(PWQ_ERR_NULL, "tensor descriptor");
    void* sc[1] = {const_cast<float*>(scale)};
    return run_list(Op::kFp8Dequant, 1, q, y, sc, nullptr, stream);
}

pwq_status mxfp8_quant(const pwq_tensor* x, const pwq_tensor* q, uint8_t* scale, pwq_stream_t stream) {
    if (!x || !q) return fail(PWQ_ERR_NULL, "tensor descriptor");
    void* sc[1] = {scale};
    return run_list(Op::kMxQuant, 1, x, q, sc, nullptr, stream);
}

pwq_status mxfp8_dequant(const pwq_tensor* q, const uint8_t* scale, const pwq_tensor* y, pwq_stream_t stream) {
    if (!q || !y) return fail(PWQ_ERR_NULL, "tensor descriptor");
    void* sc[1] = {const_cast<uint8_t*>(scale)};
    return run_list(Op::kMxDequant, 1, q, y, sc, nullptr, stream);
}

pwq_status nvfp4_dequant(const pwq_tensor* q_packed, const uint8_t* sb, const float* global_scale,
                         const pwq_tensor* y, pwq_stream_t stream) {
    if (!q_packed || !y) return fail(PWQ_ERR_NULL, "tensor descriptor");
    void* sc[1] = {const_cast<uint8_t*>(sb)};
    const float* g[1] = {global_scale};
    return run_list(Op::kNvDequant, 1, q_packed, y, sc, g, stream);
}

pwq_status fp8_block_quant_grouped(int n, const pwq_tensor* x, const pwq_tensor* q, float* const* scale,
                                   pwq_stream_t stream) {
    return run_list(Op::kFp8Quant, n, x, q, reinterpret_cast<void* const*>(scale), nullptr, stream);
}

pwq_status fp8_block_dequant_grouped(int n, const pwq_tensor* q, const float* const* scale, const pwq_tensor* y,
                                     pwq_stream_t stream) {
    return run_list(Op::kFp8Dequant, n, q, y, reinterpret_cast<void* const*>(const_cast<float**>(scale)),
                    nullptr, stream);
}

pwq_status mxfp8_quant_grouped(int n, const pwq_tensor* x, const pwq_tensor* q, uint8_t* const* scale,
                               pwq_stream_t stream) {
    return run_list(Op::kMxQuant, n, x, q, reinterpret_cast<void* const*>(scale), nullptr, stream);
}

pwq_status mxfp8_quant_grouped_mma(int n, const pwq_tensor* x, const pwq_tensor* q, uint8_t* const* scale_mma,
                                   pwq_stream_t stream) {
    return run_list(Op::kMxQuant, n, x, q, reinterpret_cast<void* const*>(scale_mma), nullptr, stream, true);
}

size_t pwq_mma_scale_bytes(int64_t batch, int64_t rows, int64_t scale_cols) {
    if (batch < 0 || rows < 0 || scale_cols < 0) return 0;
    return (size_t)(batch * pwq::mma_scale_slab_bytes(rows, scale_cols));
}

namespace {
pwq_status scale_layout_args(const void* dense, int64_t batch, int64_t rows, int64_t scale_cols, const void* mma) {
    if (batch < 0 || rows < 0 || scale_cols < 0 || batch > kMaxDim || rows > kMaxDim || scale_cols > kMaxDim)
        return fail(PWQ_ERR_SHAPE, "negative or too large extent");
    if (batch * rows * scale_cols > ((int64_t)1 << 40)) return fail(PWQ_ERR_SHAPE, "scale array too large");
    if (batch == 0 || rows == 0 || scale_cols == 0) return PWQ_OK;
    if (!dense || !mma) return fail(PWQ_ERR_NULL, "scale array");
    if ((uintptr_t)mma % 16 != 0) return fail(PWQ_ERR_ALIGN, "tile-layout array (16-byte aligned)");
    const Extent ed = extent_of(dense, (size_t)(batch * rows * scale_cols));
    const Extent em = extent_of(mma, (size_t)(batch * pwq::mma_scale_slab_bytes(rows, scale_cols)));
    if (overlaps(ed, em)) return fail(PWQ_ERR_OVERLAP, "dense and tile-layout arrays overlap");
    return PWQ_OK;
}
}  // namespace

pwq_status pwq_scales_to_mma(const uint8_t* dense, int64_t batch, int64_t rows, int64_t scale_cols, uint8_t* mma,
                             pwq_stream_t stream) {
    pwq_status st = scale_layout_args(dense, batch, rows, scale_cols, mma);
    if (st != PWQ_OK || batch == 0 || rows == 0 || scale_cols == 0) return st;
    return from_cuda(pwq::launch_scales_to_mma(dense, batch, rows, scale_cols, mma, (cudaStream_t)stream));
}

pwq_status pwq_scales_from_mma(const uint8_t* mma, int64_t batch, int64_t rows, int64_t scale_cols, uint8_t* dense,
                               pwq_stream_t stream) {
    pwq_status st = scale_layout_args(dense, batch, rows, scale_cols, mma);
    if (st != PWQ_OK || batch == 0 || rows == 0 || scale_cols == 0) return st;
    return from_cuda(pwq::launch_scales_from_mma(mma, batch, rows, scale_cols, dense, (cudaStream_t)stream));
}

pwq_status mxfp8_dequant_grouped(int n, const pwq_tensor* q, const uint8_t* const* scale, const pwq_tensor* y,
                                 pwq_stream_t stream) {
    return run_list(Op::kMxDequant, n, q, y, reinterpret_cast<void* const*>(const_cast<uint8_t**>(scale)),
                    nullptr, stream);
}

pwq_status nvfp4_dequant_grouped(int n, const pwq_tensor* q_packed, const uint8_t* const* sb,
                                 const float* const* global_scale, const pwq_tensor* y, pwq_stream_t stream) {
    return run_list(Op::kNvDequant, n, q_packed, y, reinterpret_cast<void* const*>(const_cast<uint8_t**>(sb)),
                    global_scale, stream);
}

// ------------------------------------------------------------------ NVFP4 quantise / fake-quantise

namespace {

// Validates a sibling set; fills views and extents.  Returns PWQ_OK with
// *all_empty set when there is nothing to do.
pwq_status check_siblings(const pwq_tensor* x, int n, View* vx, Extent* ex, bool* all_empty) {
    if (n < 1 || n > PWQ_MAX_SIBLINGS) return fail(PWQ_ERR_ARG, "n_siblings out of range");
    if (!x) return fail(PWQ_ERR_NULL, "x");
    *all_empty = true;
    for (int i = 0; i < n; ++i) {
        pwq_status st = check_tensor(&x[i], Kind::kBF16, &vx[i], &ex[i], "x[i]");
        if (st != PWQ_OK) return st;
        if (x[i].batch != x[0].batch) return fail(PWQ_ERR_ARG, "siblings differ in batch");
        if (x[i].cols % 16 != 0) return fail(PWQ_ERR_SHAPE, "cols % 16 != 0");
        if (!empty(&x[i])) *all_empty = false;
    }
    if (x[0].batch > 65535) return fail(PWQ_ERR_SHAPE, "batch > 65535");
    return PWQ_OK;
}

// One validated NVFP4 sibling group of a (possibly grouped) call.
struct GroupCheck {
    View x[PWQ_MAX_SIBLINGS], out[PWQ_MAX_SIBLINGS];
    uint8_t* sb[PWQ_MAX_SIBLINGS];
    int n;
    bool all_empty;
};

// Validates group g (x, out of n members; sb for quantise) and appends the
// extents of its inputs and outputs.  y[i] == x[i] exactly is allowed for
// fake-quantise.
pwq_status check_nv_group(const pwq_tensor* x, const pwq_tensor* out, uint8_t* const* sb, int n, bool fake,
                          GroupCheck* G, std::vector<Extent>& ins, std::vector<Extent>& outs,
                          std::vector<std::pair<Extent, Extent>>& aliases, bool sb_mma = false) {
    Extent ex[PWQ_MAX_SIBLINGS];
    pwq_status st = check_siblings(x, n, G->x, ex, &G->all_empty);
    if (st != PWQ_OK) return st;
    if (!out) return fail(PWQ_ERR_NULL, fake ? "y" : "q_packed");
    if (!fake && !sb) return fail(PWQ_ERR_NULL, "sb");
    G->n = n;
    const int64_t B = x[0].batch;
    for (int i = 0; i < n; ++i) {
        if (!same_shape(&x[i], &out[i])) return fail(PWQ_ERR_SHAPE, "output shape != input shape");
        Extent eo;
        if ((st = check_tensor(&out[i], fake ? Kind::kBF16 : Kind::kPacked4, &G->out[i], &eo, "output")) !=
            PWQ_OK)
            return st;
        G->sb[i] = nullptr;
        if (empty(&x[i])) continue;
        if (fake && exact_alias(&x[i], &out[i])) {
            aliases.push_back({ex[i], eo});   // in place: checked against everything else
        } else {
            ins.push_back(ex[i]);
            outs.push_back(eo);
        }
        if (!fake) {
            if (!sb[i]) return fail(PWQ_ERR_NULL, "sb[i]");
            G->sb[i] = sb[i];
            outs.push_back(extent_of(sb[i], sb_mma ? (size_t)(B * pwq::mma_scale_slab_bytes(x[i].rows, x[i].cols / 16))
                                                   : (size_t)(B * x[i].rows * (x[i].cols / 16))));
        }
    }
    return PWQ_OK;
}

// Overlap rules with in-place members: an aliased pair counts as an output
// that may coincide with exactly its own input.
pwq_status check_nv_overlaps(const std::vector<Extent>& ins, const std::vector<Extent>& outs,
                             const std::vector<std::pair<Extent, Extent>>& aliases) {
    pwq_status st = check_overlaps(ins.data(), (int)ins.size(), outs.data(), (int)outs.size());
    if (st != PWQ_OK) return st;
    for (size_t i = 0; i < aliases.size(); ++i) {
        for (const Extent& e : ins)
            if (overlaps(aliases[i].second, e)) return fail(PWQ_ERR_OVERLAP, "y[i] overlaps an input");
        for (const Extent& e : outs)
            if (overlaps(aliases[i].second, e)) return fail(PWQ_ERR_OVERLAP, "two outputs overlap");
        for (size_t j = i + 1; j < aliases.size(); ++j)
            if (overlaps(aliases[i].second, aliases[j].second)) return fail(PWQ_ERR_OVERLAP, "two outputs overlap");
    }
    return PWQ_OK;
}

pwq_status check_workspace(void* ws, size_t bytes, int64_t instances) {
    if (!ws || (uintptr_t)ws % 4 != 0 || bytes < pwq::nvfp4_flow_workspace_bytes(instances))
        return fail(PWQ_ERR_WORKSPACE, "workspace missing, misaligned or too small");
    return PWQ_OK;
}

}  // namespace

size_t nvfp4_workspace_size(int n_siblings, const pwq_tensor* x) {
    if (!x || n_siblings < 1 || n_siblings > PWQ_MAX_SIBLINGS || x[0].batch < 0) return 0;
    return pwq::nvfp4_flow_workspace_bytes(std::max<int64_t>(1, x[0].batch));
}

size_t nvfp4_workspace_size_grouped(int n_groups, const int* group_sizes, const pwq_tensor* x) {
    if (!x || !group_sizes || n_groups < 1) return 0;
    int64_t inst = 0;
    int m = 0;
    for (int g = 0; g < n_groups; ++g) {
        if (group_sizes[g] < 1 || group_sizes[g] > PWQ_MAX_SIBLINGS) return 0;
        inst += std::max<int64_t>(0, x[m].batch);
        m += group_sizes[g];
    }
    return pwq::nvfp4_flow_workspace_bytes(std::max<int64_t>(1, inst));
}

pwq_status nvfp4_group_amax(const pwq_tensor* x, int n_siblings, float* amax_out, pwq_stream_t stream) {
    View vx[PWQ_MAX_SIBLINGS];
    Extent ex[PWQ_MAX_SIBLINGS];
    bool all_empty;
    pwq_status st = check_siblings(x, n_siblings, vx, ex, &all_empty);
    if (st != PWQ_OK) return st;
    if (x[0].batch == 0) return PWQ_OK;
    if (!amax_out) return fail(PWQ_ERR_NULL, "amax_out");
    if ((uintptr_t)amax_out % 4 != 0) return fail(PWQ_ERR_ALIGN, "amax_out");
    const Extent outs[1] = {extent_of(amax_out, (size_t)x[0].batch * 4)};
    if ((st = check_overlaps(ex, n_siblings, outs, 1)) != PWQ_OK) return st;
    return from_cuda(pwq::launch_nvfp4_amax(vx, n_siblings, reinterpret_cast<uint32_t*>(amax_out),
                                            (cudaStream_t)stream));
}

namespace {

// Validates the groups of an NVFP4 call (nvfp4_quant / nvfp4_fake_quant,
// their grouped and 4over6 forms) and collects the non-empty ones for the
// launcher, with the extents of every input and output and the call's
// instance count.
pwq_status collect_nv_groups(int n_groups, const int* sizes, const pwq_tensor* x, const pwq_tensor* out,
                             uint8_t* const* sb, float* const* gs_out, const float* amax_in,
                             float* const* amax_out, bool fake, bool sb_mma, std::vector<GroupCheck>& groups,
                             std::vector<pwq::NvGroup>& launch, std::vector<Extent>& ins, std::vector<Extent>& outs,
                             std::vector<std::pair<Extent, Extent>>& aliases, int64_t* instances) {
    if (n_groups < 1 || n_groups > PWQ_MAX_GROUPED) return fail(PWQ_ERR_ARG, "group count out of range");
    if (!sizes || !x || !out) return fail(PWQ_ERR_NULL, "group sizes / tensors");
    groups.resize(n_groups);
    int m = 0;
    *instances = 0;
    for (int g = 0; g < n_groups; ++g) {
        const int n = sizes[g];
        if (n < 1 || n > PWQ_MAX_SIBLINGS || m + n > PWQ_MAX_GROUPED) return fail(PWQ_ERR_ARG, "group size");
        GroupCheck& G = groups[g];
        pwq_status st =
            check_nv_group(x + m, out + m, fake ? nullptr : sb + m, n, fake, &G, ins, outs, aliases, sb_mma);
        if (st != PWQ_OK) return st;
        const int64_t B = x[m].batch;
        if (!G.all_empty && B > 0) {
            pwq::NvGroup ng;
            ng.sb_mma = sb_mma ? 1 : 0;
            ng.x = G.x;
            ng.out = G.out;
            ng.sb = fake ? nullptr : G.sb;
            ng.n = n;
            ng.amax_in = amax_in;
            ng.gs_out = nullptr;
            ng.amax_out = nullptr;
            if (!fake) {
                if (!gs_out || !gs_out[g]) return fail(PWQ_ERR_NULL, "global_scale");
                if ((uintptr_t)gs_out[g] % 4 != 0) return fail(PWQ_ERR_ALIGN, "global_scale");
                ng.gs_out = gs_out[g];
                outs.push_back(extent_of(gs_out[g], (size_t)B * 4));
            }
            if (amax_out && amax_out[g]) {
                if ((uintptr_t)amax_out[g] % 4 != 0) return fail(PWQ_ERR_ALIGN, "amax_out");
                ng.amax_out = amax_out[g];
                outs.push_back(extent_of(amax_out[g], (size_t)B * 4));
            }
            launch.push_back(ng);
            *instances += B;
        }
        m += n;
    }
    if (amax_in) {
        if (n_groups != 1) return fail(PWQ_ERR_ARG, "amax_in needs a single group");
        if ((uintptr_t)amax_in % 4 != 0) return fail(PWQ_ERR_ALIGN, "amax_in");
        ins.push_back(extent_of(amax_in, (size_t)x[0].batch * 4));
    }
    return PWQ_OK;
}

// Shared body of nvfp4_quant / nvfp4_fake_quant and their grouped forms.
pwq_status nv_run(int n_groups, const int* sizes, const pwq_tensor* x, const pwq_tensor* out,
                  uint8_t* const* sb, float* const* gs_out, const float* amax_in, float* const* amax_out,
                  void* ws, size_t ws_bytes, bool fake, pwq_stream_t stream, bool sb_mma = false) {
    std::vector<GroupCheck> groups;
    std::vector<Extent> ins, outs;
    std::vector<std::pair<Extent, Extent>> aliases;
    std::vector<pwq::NvGroup> launch;
    int64_t instances = 0;
    pwq_status cst = collect_nv_groups(n_groups, sizes, x, out, sb, gs_out, amax_in, amax_out, fake, sb_mma, groups,
                                       launch, ins, outs, aliases, &instances);
    if (cst != PWQ_OK) return cst;
    if (launch.empty()) return PWQ_OK;
    if (!amax_in) {
        pwq_status st = check_workspace(ws, ws_bytes, instances);
        if (st != PWQ_OK) return st;
        outs.push_back(extent_of(ws, pwq::nvfp4_flow_workspace_bytes(instances)));
    }
    pwq_status st = check_nv_overlaps(ins, outs, aliases);
    if (st != PWQ_OK) return st;
    cudaStream_t s = (cudaStream_t)stream;
    if (sb_mma) {
        // the tile layout's padding (rows to 128, columns to 4) is zero bytes
        for (const pwq::NvGroup& G : launch)
            for (int i = 0; i < G.n; ++i) {
                const pwq::View& v = G.x[i];
                if (v.rows > 0 && pwq::mma_scale_padded(v.rows, v.cols / 16)) {
                    cudaError_t e = cudaMemsetAsync(G.sb[i], 0, (size_t)(v.batch * pwq::mma_scale_slab_bytes(
                                                                    v.rows, v.cols / 16)), s);
                    if (e != cudaSuccess) return cuda_fail(e);
                }
            }
    }
    // every instance small: one cluster each, one launch, the workspace unused
    if (pwq::nvfp4_cluster_ok(launch.data(), (int)launch.size()))
        return from_cuda(pwq::launch_nvfp4_cluster(launch.data(), (int)launch.size(), fake, s));
    if (amax_in) return from_cuda(pwq::launch_nvfp4_units_encode(launch.data(), 1, fake, nullptr, s));
    return from_cuda(pwq::launch_nvfp4_flow(launch.data(), (int)launch.size(), fake, ws, s));
}

}  // namespace

pwq_status nvfp4_quant(const pwq_tensor* x, int n_siblings, const pwq_tensor* q_packed, uint8_t* const* sb,
                       float* global_scale, const float* amax_in, void* workspace, size_t workspace_bytes,
                       pwq_stream_t stream) {
    const int sizes[1] = {n_siblings};
    float* gs[1] = {global_scale};
    return nv_run(1, sizes, x, q_packed, sb, gs, amax_in, nullptr, workspace, workspace_bytes, false, stream);
}

pwq_status nvfp4_fake_quant(const pwq_tensor* x, const pwq_tensor* y, int n_siblings, const float* amax_in,
                            float* amax_out, void* workspace, size_t workspace_bytes, pwq_stream_t stream) {
    const int sizes[1] = {n_siblings};
    float* ao[1] = {amax_out};
    return nv_run(1, sizes, x, y, nullptr, nullptr, amax_in, ao, workspace, workspace_bytes, true, stream);
}

pwq_status nvfp4_quant_grouped(int n_groups, const int* group_sizes, const pwq_tensor* x,
                               const pwq_tensor* q_packed, uint8_t* const* sb, float* const* global_scale,
                               void* workspace, size_t workspace_bytes, pwq_stream_t stream) {
    return nv_run(n_groups, group_sizes, x, q_packed, sb, global_scale, nullptr, nullptr, workspace,
                  workspace_bytes, false, stream);
}

pwq_status nvfp4_quant_grouped_mma(int n_groups, const int* group_sizes, const pwq_tensor* x,
                                   const pwq_tensor* q_packed, uint8_t* const* sb_mma, float* const* global_scale,
                                   void* workspace, size_t workspace_bytes, pwq_stream_t stream) {
    return nv_run(n_groups, group_sizes, x, q_packed, sb_mma, global_scale, nullptr, nullptr, workspace,
                  workspace_bytes, false, stream, true);
}

pwq_status nvfp4_fake_quant_grouped(int n_groups, const int* group_sizes, const pwq_tensor* x,
                                    const pwq_tensor* y, float* const* amax_out, void* workspace,
                                    size_t workspace_bytes, pwq_stream_t stream) {
    return nv_run(n_groups, group_sizes, x, y, nullptr, nullptr, nullptr, amax_out, workspace, workspace_bytes,
                  true, stream);
}

// ------------------------------------------------------------------ NVFP4 4over6

namespace {

// Shared body of the nvfp4_4over6_* calls: the checks of the NVFP4 calls
// (per group), then the group amaxes (unless amax_in is given) and the
// 4over6 encode.
pwq_status four_six_run(int n_groups, const int* sizes, const pwq_tensor* x, const pwq_tensor* out,
                        uint8_t* const* sb, float* const* gs_out, const float* amax_in, float* const* amax_out,
                        int e4m3_max, void* ws, size_t ws_bytes, bool fake, pwq_stream_t stream) {
    if (e4m3_max != 256 && e4m3_max != 448) return fail(PWQ_ERR_ARG, "e4m3_max must be 256 or 448");
    std::vector<GroupCheck> groups;
    std::vector<Extent> ins, outs;
    std::vector<std::pair<Extent, Extent>> aliases;
    std::vector<pwq::NvGroup> launch;
    int64_t instances = 0;
    pwq_status cst = collect_nv_groups(n_groups, sizes, x, out, sb, gs_out, amax_in, amax_out, fake, false, groups,
                                       launch, ins, outs, aliases, &instances);
    if (cst != PWQ_OK) return cst;
    if (launch.empty()) return PWQ_OK;
    if (!amax_in) {
        if (!ws || (uintptr_t)ws % 4 != 0 || ws_bytes < pwq::nvfp4_4over6_workspace_bytes(instances))
            return fail(PWQ_ERR_WORKSPACE, "workspace missing, misaligned or too small");
        outs.push_back(extent_of(ws, pwq::nvfp4_4over6_workspace_bytes(instances)));
    }
    pwq_status st = check_nv_overlaps(ins, outs, aliases);
    if (st != PWQ_OK) return st;
    return from_cuda(pwq::launch_nvfp4_4over6(launch.data(), (int)launch.size(), fake, e4m3_max, ws,
                                              (cudaStream_t)stream));
}

}  // namespace

size_t nvfp4_4over6_workspace_size(int n_siblings, const pwq_tensor* x) {
    if (!x || n_siblings < 1 || n_siblings > PWQ_MAX_SIBLINGS || x[0].batch < 0) return 0;
    return pwq::nvfp4_4over6_workspace_bytes(x[0].batch);
}

size_t nvfp4_4over6_workspace_size_grouped(int n_groups, const int* group_sizes, const pwq_tensor* x) {
    if (!x || !group_sizes || n_groups < 1 || n_groups > PWQ_MAX_GROUPED) return 0;
    int64_t inst = 0;
    int m = 0;
    for (int g = 0; g < n_groups; ++g) {
        if (group_sizes[g] < 1 || group_sizes[g] > PWQ_MAX_SIBLINGS || m + group_sizes[g] > PWQ_MAX_GROUPED) return 0;
        inst += std::max<int64_t>(0, x[m].batch);
        m += group_sizes[g];
    }
    return pwq::nvfp4_4over6_workspace_bytes(inst);
}

pwq_status nvfp4_4over6_quant(const pwq_tensor* x, int n_siblings, const pwq_tensor* q_packed, uint8_t* const* sb,
                              float* global_scale, const float* amax_in, int e4m3_max, void* workspace,
                              size_t workspace_bytes, pwq_stream_t stream) {
    const int sizes[1] = {n_siblings};
    float* gs[1] = {global_scale};
    return four_six_run(1, sizes, x, q_packed, sb, gs, amax_in, nullptr, e4m3_max, workspace, workspace_bytes,
                        false, stream);
}

pwq_status nvfp4_4over6_fake_quant(const pwq_tensor* x, const pwq_tensor* y, int n_siblings, const float* amax_in,
                                   float* amax_out, int e4m3_max, void* workspace, size_t workspace_bytes,
                                   pwq_stream_t stream) {
    const int sizes[1] = {n_siblings};
    float* ao[1] = {amax_out};
    return four_six_run(1, sizes, x, y, nullptr, nullptr, amax_in, ao, e4m3_max, workspace, workspace_bytes, true,
                        stream);
}

pwq_status nvfp4_4over6_quant_grouped(int n_groups, const int* group_sizes, const pwq_tensor* x,
                                      const pwq_tensor* q_packed, uint8_t* const* sb, float* const* global_scale,
                                      int e4m3_max, void* workspace, size_t workspace_bytes, pwq_stream_t stream) {
    return four_six_run(n_groups, group_sizes, x, q_packed, sb, global_scale, nullptr, nullptr, e4m3_max,
                        workspace, workspace_bytes, false, stream);
}

pwq_status nvfp4_4over6_fake_quant_grouped(int n_groups, const int* group_sizes, const pwq_tensor* x,
                                           const pwq_tensor* y, float* const* amax_out, int e4m3_max,
                                           void* workspace, size_t workspace_bytes, pwq_stream_t stream) {
    return four_six_run(n_groups, group_sizes, x, y, nullptr, nullptr, nullptr, amax_out, e4m3_max, workspace,
                        workspace_bytes, true, stream);
}

// ------------------------------------------------------------------ no-allocation variant

// nvfp4_fake_quant with the group-amax scratch in a file-scope device array
// (csrc/nvfp4.cu) instead of caller workspace; see include/pwq.h.
pwq_status nvfp4_fake_quant_noalloc(const pwq_tensor* x, const pwq_tensor* y, int n_siblings,
                                    const float* amax_in, float* amax_out, pwq_stream_t stream) {
    View vx[PWQ_MAX_SIBLINGS], vy[PWQ_MAX_SIBLINGS];
    Extent ex[PWQ_MAX_SIBLINGS + 1], ey[PWQ_MAX_SIBLINGS];
    bool all_empty;
    pwq_status st = check_siblings(x, n_siblings, vx, ex, &all_empty);
    if (st != PWQ_OK) return st;
    if (!y) return fail(PWQ_ERR_NULL, "y");
    for (int i = 0; i < n_siblings; ++i) {
        if (!same_shape(&x[i], &y[i])) return fail(PWQ_ERR_SHAPE, "y[i] shape != x[i] shape");
        if ((st = check_tensor(&y[i], Kind::kBF16, &vy[i], &ey[i], "y[i]")) != PWQ_OK) return st;
    }
    if (all_empty || x[0].batch == 0) return PWQ_OK;
    const int64_t B = x[0].batch;
    if (!amax_in && B > pwq::kStaticScratchGroups)
        return fail(PWQ_ERR_SHAPE, "batch exceeds the 4096-group static scratch of nvfp4_fake_quant_noalloc");
    for (int i = 0; i < n_siblings; ++i) {
        for (int j = 0; j < n_siblings; ++j) {
            if (i == j && exact_alias(&x[i], &y[i])) continue;
            if (overlaps(ey[i], ex[j])) return fail(PWQ_ERR_OVERLAP, "y[i] overlaps an input");
        }
        for (int j = i + 1; j < n_siblings; ++j)
            if (overlaps(ey[i], ey[j])) return fail(PWQ_ERR_OVERLAP, "two outputs overlap");
    }
    int n_in = n_siblings;
    if (amax_in) {
        if ((uintptr_t)amax_in % 4 != 0) return fail(PWQ_ERR_ALIGN, "amax_in");
        ex[n_in++] = extent_of(amax_in, (size_t)B * 4);
    }
    if (amax_out) {
        if ((uintptr_t)amax_out % 4 != 0) return fail(PWQ_ERR_ALIGN, "amax_out");
        const Extent eo = extent_of(amax_out, (size_t)B * 4);
        for (int j = 0; j < n_in; ++j)
            if (overlaps(eo, ex[j])) return fail(PWQ_ERR_OVERLAP, "amax_out overlaps an input");
        for (int i = 0; i < n_siblings; ++i)
            if (overlaps(eo, ey[i])) return fail(PWQ_ERR_OVERLAP, "amax_out overlaps y");
    }
    if (amax_in)
        for (int i = 0; i < n_siblings; ++i)
            if (overlaps(ey[i], ex[n_siblings])) return fail(PWQ_ERR_OVERLAP, "y overlaps amax_in");
    cudaStream_t s = (cudaStream_t)stream;
    // every instance small: one cluster each, the static scratch untouched
    pwq::NvGroup ng;
    ng.x = vx;
    ng.out = vy;
    ng.sb = nullptr;
    ng.n = n_siblings;
    ng.amax_in = amax_in;
    ng.gs_out = nullptr;
    ng.amax_out = amax_out;
    if (pwq::nvfp4_cluster_ok(&ng, 1)) return from_cuda(pwq::launch_nvfp4_cluster(&ng, 1, true, s));
    uint32_t* amax_bits = nullptr;
    if (!amax_in) {
        cudaError_t e = pwq::static_amax_scratch(&amax_bits);
        if (e != cudaSuccess) return cuda_fail(e);
        e = pwq::launch_nvfp4_amax(vx, n_siblings, amax_bits, s);  // clears the words first
        if (e != cudaSuccess) return cuda_fail(e);
    }
    return from_cuda(pwq::launch_nvfp4_units_encode(&ng, 1, true, amax_bits, s));
}

// ------------------------------------------------------------------ FP8 block-wise -> rollout formats

namespace {

// Overlap rule of the re-quantisation calls: no output may touch an input or
// another output, except the pairs listed in `allowed` (exact in-place use).
pwq_status check_requant_overlaps(const std::vector<Extent>& ins, const std::vector<Extent>& outs,
                                  const std::vector<std::pair<int, int>>& allowed) {
    for (size_t i = 0; i < outs.size(); ++i) {
        for (size_t j = 0; j < ins.size(); ++j) {
            bool ok = false;
            for (const auto& p : allowed) ok |= (p.first == (int)i && p.second == (int)j);
            if (!ok && overlaps(outs[i], ins[j])) return fail(PWQ_ERR_OVERLAP, "output overlaps an input");
        }
        for (size_t j = i + 1; j < outs.size(); ++j)
            if (overlaps(outs[i], outs[j])) return fail(PWQ_ERR_OVERLAP, "two outputs overlap");
    }
    return PWQ_OK;
}

size_t tile_scale_bytes(const pwq_tensor* t) {
    return (size_t)(t->batch * ceil_div(t->rows, 128) * ceil_div(t->cols, 128)) * 4;
}

// The FP8 block-wise input (codes + tile scales) and a same-shaped code
// output of the FP8 / MXFP8 re-quantisation.
pwq_status check_requant_io(const pwq_tensor* q_in, const float* scale_in, const pwq_tensor* q_out, View* vq,
                            View* vo, Extent* eq, Extent* eo, Extent* esi) {
    pwq_status st;
    if ((st = check_tensor(q_in, Kind::kByte, vq, eq, "q_in")) != PWQ_OK) return st;
    if (!q_out) return fail(PWQ_ERR_NULL, "q_out");
    if (!same_shape(q_in, q_out)) return fail(PWQ_ERR_SHAPE, "q_out shape != q_in shape");
    if ((st = check_tensor(q_out, Kind::kByte, vo, eo, "q_out")) != PWQ_OK) return st;
    if (empty(q_in)) return PWQ_OK;
    if (!scale_in) return fail(PWQ_ERR_NULL, "scale_in");
    if ((uintptr_t)scale_in % 4 != 0) return fail(PWQ_ERR_ALIGN, "scale_in");
    *esi = extent_of(scale_in, tile_scale_bytes(q_in));
    return PWQ_OK;
}

}  // namespace

namespace {

// Shared body of the FP8 -> FP8 / MXFP8 re-quantisation calls over a list of
// n tensors.  In place: q_out[i] == q_in[i] exactly, and for FP8 scale_out[i]
// == scale_in[i].
pwq_status requant_list(bool mx, int n, const pwq_tensor* q_in, const float* const* scale_in,
                        const pwq_tensor* q_out, void* const* scale_out, pwq_stream_t stream) {
    if (n < 0 || n > PWQ_MAX_GROUPED) return fail(PWQ_ERR_ARG, "tensor count out of range");
    if (n == 0) return PWQ_OK;
    if (!q_in || !q_out || !scale_in || !scale_out) return fail(PWQ_ERR_NULL, "tensor or scale array");
    std::vector<pwq::RequantJob> jobs;
    std::vector<Extent> ins, outs;
    std::vector<std::pair<int, int>> allowed;
    for (int i = 0; i < n; ++i) {
        pwq::RequantJob J;
        Extent eq, eo, esi;
        pwq_status st = check_requant_io(&q_in[i], scale_in[i], &q_out[i], &J.in, &J.out, &eq, &eo, &esi);
        if (st != PWQ_OK) return st;
        if (mx && q_in[i].cols % 32 != 0) return fail(PWQ_ERR_SHAPE, "cols % 32 != 0");
        if (empty(&q_in[i])) continue;
        if (!scale_out[i]) return fail(PWQ_ERR_NULL, "scale_out");
        if (!mx && (uintptr_t)scale_out[i] % 4 != 0) return fail(PWQ_ERR_ALIGN, "scale_out");
        const Extent eso = extent_of(scale_out[i], mx ? (size_t)(q_in[i].batch * q_in[i].rows * (q_in[i].cols / 32))
                                                      : tile_scale_bytes(&q_in[i]));
        const int in0 = (int)ins.size(), out0 = (int)outs.size();
        ins.push_back(eq);
        ins.push_back(esi);
        outs.push_back(eo);
        outs.push_back(eso);
        if (exact_alias(&q_in[i], &q_out[i])) allowed.push_back({out0, in0});
        if (!mx && scale_out[i] == (const void*)scale_in[i]) allowed.push_back({out0 + 1, in0 + 1});
        J.scale_in = scale_in[i];
        J.scale_out = scale_out[i];
        jobs.push_back(J);
    }
    pwq_status st = check_requant_overlaps(ins, outs, allowed);
    if (st != PWQ_OK) return st;
    if (jobs.empty()) return PWQ_OK;
    cudaStream_t s = (cudaStream_t)stream;
    return from_cuda(mx ? pwq::launch_fp8_requant_mxfp8(jobs.data(), (int)jobs.size(), s)
                        : pwq::launch_fp8_requant_fp8(jobs.data(), (int)jobs.size(), s));
}

}  // namespace

pwq_status fp8_block_requant(const pwq_tensor* q_in, const float* scale_in, const pwq_tensor* q_out,
                             float* scale_out, pwq_stream_t stream) {
    const float* si[1] = {scale_in};
    void* so[1] = {scale_out};
    return requant_list(false, 1, q_in, si, q_out, so, stream);
}

pwq_status fp8_block_requant_mxfp8(const pwq_tensor* q_in, const float* scale_in, const pwq_tensor* q_out,
                                   uint8_t* scale_ue8m0, pwq_stream_t stream) {
    const float* si[1] = {scale_in};
    void* so[1] = {scale_ue8m0};
    return requant_list(true, 1, q_in, si, q_out, so, stream);
}

pwq_status fp8_block_requant_grouped(int n, const pwq_tensor* q_in, const float* const* scale_in,
                                     const pwq_tensor* q_out, float* const* scale_out, pwq_stream_t stream) {
    return requant_list(false, n, q_in, scale_in, q_out, reinterpret_cast<void* const*>(scale_out), stream);
}

pwq_status fp8_block_requant_mxfp8_grouped(int n, const pwq_tensor* q_in, const float* const* scale_in,
                                           const pwq_tensor* q_out, uint8_t* const* scale_ue8m0,
                                           pwq_stream_t stream) {
    return requant_list(true, n, q_in, scale_in, q_out, reinterpret_cast<void* const*>(scale_ue8m0), stream);
}

namespace {

// One FP8 block-wise sibling group of a re-quantisation into NVFP4: codes
// (N % 16 == 0, same batch), their tile scales, packed outputs and block
// scales; appends extents.
pwq_status check_requant_nv_group(const pwq_tensor* q_in, const float* const* scale_in, int n,
                                  const pwq_tensor* q_packed, uint8_t* const* sb, View* vq, View* vo,
                                  std::vector<Extent>& ins, std::vector<Extent>& outs, bool* all_empty) {
    if (n < 1 || n > PWQ_MAX_SIBLINGS) return fail(PWQ_ERR_ARG, "n_siblings out of range");
    const int64_t B = q_in[0].batch;
    *all_empty = true;
    pwq_status st;
    for (int i = 0; i < n; ++i) {
        Extent eq, eo;
        if ((st = check_tensor(&q_in[i], Kind::kByte, &vq[i], &eq, "q_in[i]")) != PWQ_OK) return st;
        if (q_in[i].batch != B) return fail(PWQ_ERR_ARG, "siblings differ in batch");
        if (q_in[i].cols % 16 != 0) return fail(PWQ_ERR_SHAPE, "cols % 16 != 0");
        if (!same_shape(&q_in[i], &q_packed[i])) return fail(PWQ_ERR_SHAPE, "q_packed shape != q_in shape");
        if ((st = check_tensor(&q_packed[i], Kind::kPacked4, &vo[i], &eo, "q_packed[i]")) != PWQ_OK) return st;
        if (empty(&q_in[i])) continue;
        *all_empty = false;
        if (!scale_in || !scale_in[i]) return fail(PWQ_ERR_NULL, "scale_in[i]");
        if ((uintptr_t)scale_in[i] % 4 != 0) return fail(PWQ_ERR_ALIGN, "scale_in[i]");
        if (!sb || !sb[i]) return fail(PWQ_ERR_NULL, "sb[i]");
        ins.push_back(eq);
        ins.push_back(extent_of(scale_in[i], tile_scale_bytes(&q_in[i])));
        outs.push_back(eo);
        outs.push_back(extent_of(sb[i], (size_t)(B * q_in[i].rows * (q_in[i].cols / 16))));
    }
    if (B > 65535) return fail(PWQ_ERR_SHAPE, "batch > 65535");
    return PWQ_OK;
}

// Shared body of fp8_block_requant_nvfp4 and its grouped form.
pwq_status requant_nv_run(int n_groups, const int* sizes, const pwq_tensor* q_in, const float* const* scale_in,
                          const pwq_tensor* q_packed, uint8_t* const* sb, float* const* global_scale,
                          const float* amax_in, void* ws, size_t ws_bytes, pwq_stream_t stream) {
    if (n_groups < 1 || n_groups > PWQ_MAX_GROUPED) return fail(PWQ_ERR_ARG, "group count out of range");
    if (!sizes || !q_in || !q_packed) return fail(PWQ_ERR_NULL, "group sizes / tensors");
    struct G {
        View q[PWQ_MAX_SIBLINGS], o[PWQ_MAX_SIBLINGS];
    };
    std::vector<G> views(n_groups);
    std::vector<Extent> ins, outs;
    std::vector<pwq::NvGroup> launch;
    int m = 0;
    int64_t instances = 0;
    for (int g = 0; g < n_groups; ++g) {
        const int n = sizes[g];
        if (n < 1 || n > PWQ_MAX_SIBLINGS || m + n > PWQ_MAX_GROUPED) return fail(PWQ_ERR_ARG, "group size");
        bool all_empty;
        pwq_status st = check_requant_nv_group(q_in + m, scale_in ? scale_in + m : nullptr, n, q_packed + m,
                                               sb ? sb + m : nullptr, views[g].q, views[g].o, ins, outs,
                                               &all_empty);
        if (st != PWQ_OK) return st;
        const int64_t B = q_in[m].batch;
        if (!all_empty && B > 0) {
            if (!global_scale || !global_scale[g]) return fail(PWQ_ERR_NULL, "global_scale");
            if ((uintptr_t)global_scale[g] % 4 != 0) return fail(PWQ_ERR_ALIGN, "global_scale");
            outs.push_back(extent_of(global_scale[g], (size_t)B * 4));
            pwq::NvGroup ng;
            ng.x = views[g].q;
            ng.out = views[g].o;
            ng.sb = sb + m;
            ng.n = n;
            ng.amax_in = amax_in;
            ng.gs_out = global_scale[g];
            ng.amax_out = nullptr;
            ng.ts = scale_in + m;
            launch.push_back(ng);
            instances += B;
        }
        m += n;
    }
    if (amax_in) {
        if (n_groups != 1) return fail(PWQ_ERR_ARG, "amax_in needs a single group");
        if ((uintptr_t)amax_in % 4 != 0) return fail(PWQ_ERR_ALIGN, "amax_in");
        ins.push_back(extent_of(amax_in, (size_t)q_in[0].batch * 4));
    }
    if (launch.empty()) return PWQ_OK;
    if (!amax_in) {
        pwq_status st = check_workspace(ws, ws_bytes, instances);
        if (st != PWQ_OK) return st;
        outs.push_back(extent_of(ws, pwq::nvfp4_flow_workspace_bytes(instances)));
    }
    pwq_status st = check_requant_overlaps(ins, outs, {});
    if (st != PWQ_OK) return st;
    cudaStream_t s = (cudaStream_t)stream;
    if (amax_in) return from_cuda(pwq::launch_nvfp4_units_encode(launch.data(), 1, false, nullptr, s));
    return from_cuda(pwq::launch_nvfp4_flow(launch.data(), (int)launch.size(), false, ws, s));
}

}  // namespace

size_t fp8_block_requant_nvfp4_workspace_size(int n_siblings, const pwq_tensor* q_in) {
    return nvfp4_workspace_size(n_siblings, q_in);
}

size_t fp8_block_requant_nvfp4_workspace_size_grouped(int n_groups, const int* group_sizes,
                                                      const pwq_tensor* q_in) {
    return nvfp4_workspace_size_grouped(n_groups, group_sizes, q_in);
}

pwq_status fp8_block_requant_nvfp4(const pwq_tensor* q_in, const float* const* scale_in, int n_siblings,
                                   const pwq_tensor* q_packed, uint8_t* const* sb, float* global_scale,
                                   const float* amax_in, void* workspace, size_t workspace_bytes,
                                   pwq_stream_t stream) {
    const int sizes[1] = {n_siblings};
    float* gs[1] = {global_scale};
    if (n_siblings < 1 || n_siblings > PWQ_MAX_SIBLINGS) return fail(PWQ_ERR_ARG, "n_siblings out of range");
    return requant_nv_run(1, sizes, q_in, scale_in, q_packed, sb, gs, amax_in, workspace, workspace_bytes, stream);
}

pwq_status fp8_block_requant_nvfp4_grouped(int n_groups, const int* group_sizes, const pwq_tensor* q_in,
                                           const float* const* scale_in, const pwq_tensor* q_packed,
                                           uint8_t* const* sb, float* const* global_scale, void* workspace,
                                           size_t workspace_bytes, pwq_stream_t stream) {
    return requant_nv_run(n_groups, group_sizes, q_in, scale_in, q_packed, sb, global_scale, nullptr, workspace,
                          workspace_bytes, stream);
}

// ------------------------------------------------------------------ W4A4 activation observers

size_t nvfp4_observe_workspace_size(void) { return 256; }

pwq_status nvfp4_activation_observe(const pwq_tensor* x, int observer, float averaging_constant, float* state,
                                    float* amax_out, float* input_global_scale, void* workspace,
                                    size_t workspace_bytes, pwq_stream_t stream) {
    View vx;
    Extent ex;
    pwq_status st = check_tensor(x, Kind::kBF16, &vx, &ex, "x");
    if (st != PWQ_OK) return st;
    if (x->cols % 16 != 0) return fail(PWQ_ERR_SHAPE, "cols % 16 != 0");
    if (observer < PWQ_OBSERVER_MEMORYLESS_MINMAX || observer > PWQ_OBSERVER_MINMAX)
        return fail(PWQ_ERR_ARG, "observer kind");
    if (observer == PWQ_OBSERVER_MINMAX && !(averaging_constant >= 0.0f && averaging_constant <= 1.0f))
        return fail(PWQ_ERR_ARG, "averaging_constant outside [0, 1]");
    if (!state) return fail(PWQ_ERR_NULL, "state");
    if ((uintptr_t)state % 4 != 0 || ((uintptr_t)amax_out % 4) != 0 || ((uintptr_t)input_global_scale % 4) != 0)
        return fail(PWQ_ERR_ALIGN, "state / amax_out / input_global_scale");
    if (empty(x)) return PWQ_OK;
    if (!workspace || (uintptr_t)workspace % 4 != 0 || workspace_bytes < nvfp4_observe_workspace_size())
        return fail(PWQ_ERR_WORKSPACE, "workspace missing, misaligned or too small");
    std::vector<Extent> outs = {extent_of(state, 8), extent_of(workspace, nvfp4_observe_workspace_size())};
    if (amax_out) outs.push_back(extent_of(amax_out, 4));
    if (input_global_scale) outs.push_back(extent_of(input_global_scale, 4));
    if ((st = check_overlaps(&ex, 1, outs.data(), (int)outs.size())) != PWQ_OK) return st;
    return from_cuda(pwq::launch_activation_observe(vx, observer, averaging_constant, state, amax_out,
                                                    input_global_scale, static_cast<uint32_t*>(workspace),
                                                    (cudaStream_t)stream));
}

// ------------------------------------------------------------------ self-tests

size_t pwq_selftest_flow_timeout_workspace_size(const pwq_tensor* x) {
    if (!x || x->batch < 0 || x->batch > 512) return 0;
    return pwq::nvfp4_flow_timeout_selftest_bytes(std::max<int64_t>(1, x->batch));
}

pwq_status pwq_selftest_flow_timeout(const pwq_tensor* x, const pwq_tensor* y, uint64_t wait_ns, void* workspace,
                                     size_t workspace_bytes, pwq_stream_t stream) {
    if (wait_ns < 1000ull || wait_ns > pwq::kFlowWaitLimitNs)
        return fail(PWQ_ERR_ARG, "wait_ns outside [1 us, 2 s]");
    View vx, vy;
    Extent ex, ey;
    pwq_status st = check_tensor(x, Kind::kBF16, &vx, &ex, "x");
    if (st != PWQ_OK) return st;
    if (!y) return fail(PWQ_ERR_NULL, "y");
    if (!same_shape(x, y)) return fail(PWQ_ERR_SHAPE, "y shape != x shape");
    if ((st = check_tensor(y, Kind::kBF16, &vy, &ey, "y")) != PWQ_OK) return st;
    if (empty(x)) return fail(PWQ_ERR_SHAPE, "the self-test needs a non-empty x");
    if (x->cols % 16 != 0) return fail(PWQ_ERR_SHAPE, "cols % 16 != 0");
    if (x->batch > 512) return fail(PWQ_ERR_SHAPE, "the self-test takes at most 512 batch slabs");
    const size_t need = pwq::nvfp4_flow_timeout_selftest_bytes(x->batch);
    if (!workspace || (uintptr_t)workspace % 4 != 0 || workspace_bytes < need)
        return fail(PWQ_ERR_WORKSPACE, "workspace missing, misaligned or too small");
    const Extent ew = extent_of(workspace, need);
    if (overlaps(ey, ex) || overlaps(ew, ex) || overlaps(ew, ey)) return fail(PWQ_ERR_OVERLAP, "operands overlap");
    pwq::NvGroup g{};
    g.x = &vx;
    g.out = &vy;
    g.sb = nullptr;
    g.n = 1;
    return from_cuda(pwq::launch_nvfp4_flow(&g, 1, true, workspace, (cudaStream_t)stream, wait_ns, true));
}

pwq_status pwq_selftest_division(int which, unsigned long long* counts, pwq_stream_t stream) {
    if (!counts) return fail(PWQ_ERR_NULL, "counts");
    if (which < 0 || which > 9) return fail(PWQ_ERR_ARG, "which");
    return from_cuda(pwq::launch_selftest_division(which, counts, (cudaStream_t)stream));
}

pwq_status pwq_selftest_codecs(uint32_t first, uint32_t count, uint8_t* e4m3, uint8_t* e2m1, uint16_t* bf16,
                               pwq_stream_t stream) {
    return from_cuda(pwq::launch_selftest_codecs(first, count, e4m3, e2m1, bf16, (cudaStream_t)stream));
}

}  // extern "C"
