// pwq_api.cu -- the extern "C" entry points declared in include/pwq.h:
// argument validation (null, alignment, shape, stride, overlap, workspace),
// conversion to byte-stride views and dispatch to the kernel launchers.
// Nothing here allocates device memory or synchronises.
#include <algorithm>
#include <cstdio>
#include <cstring>

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
    static int cache[64] = {0};
    if (device >= 0 && device < 64 && cache[device] > 0) return cache[device];
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, device) != cudaSuccess || n <= 0) n = 148;
    if (device >= 0 && device < 64) cache[device] = n;
    return n;
}

int persistent_grid(int64_t work_ctas, int per_sm) {
    const int64_t cap = (int64_t)sm_count(current_device()) * per_sm;
    return (int)std::max<int64_t>(1, std::min<int64_t>(work_ctas, cap));
}

}  // namespace pwq

namespace {

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

constexpr int64_t kMaxU32 = (int64_t(1) << 32) - 1;

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
    return from_cuda(pwq::read_and_clear_device_error(code));
}

// ------------------------------------------------------------------ FP8 block

pwq_status fp8_block_quant(const pwq_tensor* x, const pwq_tensor* q, float* scale, pwq_stream_t stream) {
    if (!x || !q) return fail(PWQ_ERR_NULL, "tensor descriptor");
    if (!same_shape(x, q)) return fail(PWQ_ERR_SHAPE, "q shape != x shape");
    View vx, vq;
    Extent ex, eq;
    pwq_status st;
    if ((st = check_tensor(x, Kind::kBF16, &vx, &ex, "x")) != PWQ_OK) return st;
    if ((st = check_tensor(q, Kind::kByte, &vq, &eq, "q")) != PWQ_OK) return st;
    if (empty(x)) return PWQ_OK;
    if (!scale) return fail(PWQ_ERR_NULL, "scale");
    if ((uintptr_t)scale % 4 != 0) return fail(PWQ_ERR_ALIGN, "scale");
    const int64_t tiles = x->batch * ceil_div(x->rows, 128) * ceil_div(x->cols, 128);
    if (tiles > kMaxU32) return fail(PWQ_ERR_SHAPE, "too many tiles");
    const Extent es = extent_of(scale, (size_t)tiles * 4);
    const Extent ins[1] = {ex};
    const Extent outs[2] = {eq, es};
    if ((st = check_overlaps(ins, 1, outs, 2)) != PWQ_OK) return st;
    return from_cuda(pwq::launch_fp8_block_quant(vx, vq, scale, (cudaStream_t)stream));
}

pwq_status fp8_block_dequant(const pwq_tensor* q, const float* scale, const pwq_tensor* y,
                             pwq_stream_t stream) {
    if (!q || !y) return fail(PWQ_ERR_NULL, "tensor descriptor");
    if (!same_shape(q, y)) return fail(PWQ_ERR_SHAPE, "y shape != q shape");
    View vq, vy;
    Extent eq, ey;
    pwq_status st;
    if ((st = check_tensor(q, Kind::kByte, &vq, &eq, "q")) != PWQ_OK) return st;
    if ((st = check_tensor(y, Kind::kBF16, &vy, &ey, "y")) != PWQ_OK) return st;
    if (empty(q)) return PWQ_OK;
    if (!scale) return fail(PWQ_ERR_NULL, "scale");
    if ((uintptr_t)scale % 4 != 0) return fail(PWQ_ERR_ALIGN, "scale");
    if (q->batch * q->rows * ceil_div(q->cols, 8) > kMaxU32) return fail(PWQ_ERR_SHAPE, "too large");
    const int64_t tiles = q->batch * ceil_div(q->rows, 128) * ceil_div(q->cols, 128);
    const Extent es = extent_of(scale, (size_t)tiles * 4);
    const Extent ins[2] = {eq, es};
    const Extent outs[1] = {ey};
    if ((st = check_overlaps(ins, 2, outs, 1)) != PWQ_OK) return st;
    return from_cuda(pwq::launch_fp8_block_dequant(vq, scale, vy, (cudaStream_t)stream));
}

// ------------------------------------------------------------------ MXFP8

pwq_status mxfp8_quant(const pwq_tensor* x, const pwq_tensor* q, uint8_t* scale, pwq_stream_t stream) {
    if (!x || !q) return fail(PWQ_ERR_NULL, "tensor descriptor");
    if (!same_shape(x, q)) return fail(PWQ_ERR_SHAPE, "q shape != x shape");
    View vx, vq;
    Extent ex, eq;
    pwq_status st;
    if ((st = check_tensor(x, Kind::kBF16, &vx, &ex, "x")) != PWQ_OK) return st;
    if ((st = check_tensor(q, Kind::kByte, &vq, &eq, "q")) != PWQ_OK) return st;
    if (x->cols % 32 != 0) return fail(PWQ_ERR_SHAPE, "cols % 32 != 0");
    if (empty(x)) return PWQ_OK;
    if (!scale) return fail(PWQ_ERR_NULL, "scale");
    if (x->rows * (x->cols / 8) > kMaxU32 / 2) return fail(PWQ_ERR_SHAPE, "matrix too large");
    const Extent es = extent_of(scale, (size_t)(x->batch * x->rows * (x->cols / 32)));
    const Extent ins[1] = {ex};
    const Extent outs[2] = {eq, es};
    if ((st = check_overlaps(ins, 1, outs, 2)) != PWQ_OK) return st;
    return from_cuda(pwq::launch_mxfp8_quant(vx, vq, scale, (cudaStream_t)stream));
}

pwq_status mxfp8_dequant(const pwq_tensor* q, const uint8_t* scale, const pwq_tensor* y, pwq_stream_t stream) {
    if (!q || !y) return fail(PWQ_ERR_NULL, "tensor descriptor");
    if (!same_shape(q, y)) return fail(PWQ_ERR_SHAPE, "y shape != q shape");
    View vq, vy;
    Extent eq, ey;
    pwq_status st;
    if ((st = check_tensor(q, Kind::kByte, &vq, &eq, "q")) != PWQ_OK) return st;
    if ((st = check_tensor(y, Kind::kBF16, &vy, &ey, "y")) != PWQ_OK) return st;
    if (q->cols % 32 != 0) return fail(PWQ_ERR_SHAPE, "cols % 32 != 0");
    if (empty(q)) return PWQ_OK;
    if (!scale) return fail(PWQ_ERR_NULL, "scale");
    if (q->rows * (q->cols / 8) > kMaxU32 / 2) return fail(PWQ_ERR_SHAPE, "matrix too large");
    const Extent es = extent_of(scale, (size_t)(q->batch * q->rows * (q->cols / 32)));
    const Extent ins[2] = {eq, es};
    const Extent outs[1] = {ey};
    if ((st = check_overlaps(ins, 2, outs, 1)) != PWQ_OK) return st;
    return from_cuda(pwq::launch_mxfp8_dequant(vq, scale, vy, (cudaStream_t)stream));
}

// ------------------------------------------------------------------ NVFP4

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
        if (x[i].rows * (x[i].cols / 8) > kMaxU32) return fail(PWQ_ERR_SHAPE, "matrix too large");
        if (!empty(&x[i])) *all_empty = false;
    }
    if (x[0].batch > 65535) return fail(PWQ_ERR_SHAPE, "batch > 65535");
    return PWQ_OK;
}

}  // namespace

size_t nvfp4_workspace_size(int n_siblings, const pwq_tensor* x) {
    if (!x || n_siblings < 1 || n_siblings > PWQ_MAX_SIBLINGS || x[0].batch < 0) return 0;
    const size_t b = (size_t)std::max<int64_t>(1, x[0].batch);
    return (b * 4 + 255) / 256 * 256;
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

pwq_status nvfp4_quant(const pwq_tensor* x, int n_siblings, const pwq_tensor* q_packed, uint8_t* const* sb,
                       float* global_scale, const float* amax_in, void* workspace, size_t workspace_bytes,
                       pwq_stream_t stream) {
    View vx[PWQ_MAX_SIBLINGS], vq[PWQ_MAX_SIBLINGS];
    Extent ex[PWQ_MAX_SIBLINGS + 1], eo[3 * PWQ_MAX_SIBLINGS + 2];
    bool all_empty;
    pwq_status st = check_siblings(x, n_siblings, vx, ex, &all_empty);
    if (st != PWQ_OK) return st;
    if (!q_packed || !sb) return fail(PWQ_ERR_NULL, "q_packed / sb");
    int n_out = 0;
    for (int i = 0; i < n_siblings; ++i) {
        if (!same_shape(&x[i], &q_packed[i])) return fail(PWQ_ERR_SHAPE, "q_packed[i] shape != x[i] shape");
        if ((st = check_tensor(&q_packed[i], Kind::kPacked4, &vq[i], &eo[n_out++], "q_packed[i]")) != PWQ_OK)
            return st;
    }
    if (all_empty || x[0].batch == 0) return PWQ_OK;
    const int64_t B = x[0].batch;
    for (int i = 0; i < n_siblings; ++i) {
        if (empty(&x[i])) continue;
        if (!sb[i]) return fail(PWQ_ERR_NULL, "sb[i]");
        eo[n_out++] = extent_of(sb[i], (size_t)(B * x[i].rows * (x[i].cols / 16)));
    }
    if (!global_scale) return fail(PWQ_ERR_NULL, "global_scale");
    if ((uintptr_t)global_scale % 4 != 0) return fail(PWQ_ERR_ALIGN, "global_scale");
    eo[n_out++] = extent_of(global_scale, (size_t)B * 4);
    int n_in = n_siblings;
    if (amax_in) {
        if ((uintptr_t)amax_in % 4 != 0) return fail(PWQ_ERR_ALIGN, "amax_in");
        ex[n_in++] = extent_of(amax_in, (size_t)B * 4);
    } else {
        if (!workspace || (uintptr_t)workspace % 4 != 0 || workspace_bytes < (size_t)B * 4)
            return fail(PWQ_ERR_WORKSPACE, "workspace missing, misaligned or too small");
        eo[n_out++] = extent_of(workspace, (size_t)B * 4);
    }
    if ((st = check_overlaps(ex, n_in, eo, n_out)) != PWQ_OK) return st;
    cudaStream_t s = (cudaStream_t)stream;
    uint32_t* amax_bits = static_cast<uint32_t*>(workspace);
    if (!amax_in) {
        cudaError_t e = pwq::launch_nvfp4_amax(vx, n_siblings, amax_bits, s);
        if (e != cudaSuccess) return cuda_fail(e);
    }
    return from_cuda(pwq::launch_nvfp4_encode(vx, n_siblings, vq, sb, false, amax_in ? nullptr : amax_bits,
                                              amax_in, global_scale, nullptr, s));
}

pwq_status nvfp4_dequant(const pwq_tensor* q_packed, const uint8_t* sb, const float* global_scale,
                         const pwq_tensor* y, pwq_stream_t stream) {
    if (!q_packed || !y) return fail(PWQ_ERR_NULL, "tensor descriptor");
    if (!same_shape(q_packed, y)) return fail(PWQ_ERR_SHAPE, "y shape != q_packed shape");
    View vq, vy;
    Extent eq, ey;
    pwq_status st;
    if ((st = check_tensor(q_packed, Kind::kPacked4, &vq, &eq, "q_packed")) != PWQ_OK) return st;
    if ((st = check_tensor(y, Kind::kBF16, &vy, &ey, "y")) != PWQ_OK) return st;
    if (q_packed->cols % 16 != 0) return fail(PWQ_ERR_SHAPE, "cols % 16 != 0");
    if (empty(q_packed)) return PWQ_OK;
    if (!sb || !global_scale) return fail(PWQ_ERR_NULL, "sb / global_scale");
    if ((uintptr_t)global_scale % 4 != 0) return fail(PWQ_ERR_ALIGN, "global_scale");
    if (q_packed->batch * q_packed->rows * (q_packed->cols / 8) > kMaxU32)
        return fail(PWQ_ERR_SHAPE, "too large");
    const int64_t B = q_packed->batch;
    const Extent ins[3] = {eq, extent_of(sb, (size_t)(B * q_packed->rows * (q_packed->cols / 16))),
                           extent_of(global_scale, (size_t)B * 4)};
    const Extent outs[1] = {ey};
    if ((st = check_overlaps(ins, 3, outs, 1)) != PWQ_OK) return st;
    return from_cuda(pwq::launch_nvfp4_dequant(vq, sb, global_scale, vy, (cudaStream_t)stream));
}

pwq_status nvfp4_fake_quant(const pwq_tensor* x, const pwq_tensor* y, int n_siblings, const float* amax_in,
                            float* amax_out, void* workspace, size_t workspace_bytes, pwq_stream_t stream) {
    View vx[PWQ_MAX_SIBLINGS], vy[PWQ_MAX_SIBLINGS];
    Extent ex[PWQ_MAX_SIBLINGS + 1], ey[PWQ_MAX_SIBLINGS + 2];
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
    // y[i] may alias x[i] exactly; any other intersection is an error
    for (int i = 0; i < n_siblings; ++i) {
        for (int j = 0; j < n_siblings; ++j) {
            if (i == j && exact_alias(&x[i], &y[i])) continue;
            if (overlaps(ey[i], ex[j])) return fail(PWQ_ERR_OVERLAP, "y[i] overlaps an input");
        }
        for (int j = i + 1; j < n_siblings; ++j)
            if (overlaps(ey[i], ey[j])) return fail(PWQ_ERR_OVERLAP, "two outputs overlap");
    }
    int n_in = n_siblings, n_out = 0;
    Extent extra_out[2];
    if (amax_in) {
        if ((uintptr_t)amax_in % 4 != 0) return fail(PWQ_ERR_ALIGN, "amax_in");
        ex[n_in++] = extent_of(amax_in, (size_t)B * 4);
    } else {
        if (!workspace || (uintptr_t)workspace % 4 != 0 || workspace_bytes < (size_t)B * 4)
            return fail(PWQ_ERR_WORKSPACE, "workspace missing, misaligned or too small");
        extra_out[n_out++] = extent_of(workspace, (size_t)B * 4);
    }
    if (amax_out) {
        if ((uintptr_t)amax_out % 4 != 0) return fail(PWQ_ERR_ALIGN, "amax_out");
        extra_out[n_out++] = extent_of(amax_out, (size_t)B * 4);
    }
    for (int k = 0; k < n_out; ++k) {
        for (int j = 0; j < n_in; ++j)
            if (overlaps(extra_out[k], ex[j])) return fail(PWQ_ERR_OVERLAP, "amax/workspace overlaps an input");
        for (int i = 0; i < n_siblings; ++i)
            if (overlaps(extra_out[k], ey[i])) return fail(PWQ_ERR_OVERLAP, "amax/workspace overlaps y");
        for (int j = k + 1; j < n_out; ++j)
            if (overlaps(extra_out[k], extra_out[j])) return fail(PWQ_ERR_OVERLAP, "amax_out overlaps workspace");
    }
    for (int i = 0; i < n_siblings; ++i)
        if (amax_in && overlaps(ey[i], ex[n_siblings])) return fail(PWQ_ERR_OVERLAP, "y overlaps amax_in");
    cudaStream_t s = (cudaStream_t)stream;
    uint32_t* amax_bits = static_cast<uint32_t*>(workspace);
    if (!amax_in) {
        cudaError_t e = pwq::launch_nvfp4_amax(vx, n_siblings, amax_bits, s);
        if (e != cudaSuccess) return cuda_fail(e);
    }
    return from_cuda(pwq::launch_nvfp4_encode(vx, n_siblings, vy, nullptr, true, amax_in ? nullptr : amax_bits,
                                              amax_in, nullptr, amax_out, s));
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
    uint32_t* amax_bits = nullptr;
    if (!amax_in) {
        cudaError_t e = pwq::static_amax_scratch(&amax_bits);
        if (e != cudaSuccess) return cuda_fail(e);
        e = pwq::launch_nvfp4_amax(vx, n_siblings, amax_bits, s);  // clears the words first
        if (e != cudaSuccess) return cuda_fail(e);
    }
    return from_cuda(pwq::launch_nvfp4_encode(vx, n_siblings, vy, nullptr, true, amax_bits, amax_in, nullptr,
                                              amax_out, s));
}

// ------------------------------------------------------------------ self-tests

pwq_status pwq_selftest_division(int which, unsigned long long* counts, pwq_stream_t stream) {
    if (!counts) return fail(PWQ_ERR_NULL, "counts");
    if (which < 0 || which > 2) return fail(PWQ_ERR_ARG, "which");
    return from_cuda(pwq::launch_selftest_division(which, counts, (cudaStream_t)stream));
}

pwq_status pwq_selftest_codecs(uint32_t first, uint32_t count, uint8_t* e4m3, uint8_t* e2m1, uint16_t* bf16,
                               pwq_stream_t stream) {
    return from_cuda(pwq::launch_selftest_codecs(first, count, e4m3, e2m1, bf16, (cudaStream_t)stream));
}

}  // extern "C"
