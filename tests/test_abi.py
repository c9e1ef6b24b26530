"""C ABI boundary tests that need no GPU: the shared library loads, exports
every function include/pwq.h declares, reports its exact-math build, and
rejects bad arguments with the documented status before any CUDA call."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "pwq.h")


def _lib():
    import __graft_entry__
    __graft_entry__._load_build_script().build()
    import precision_weight_quantization_b200._lib as L
    return L


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"^[A-Za-z_][\w \*]*?\b([a-z_][a-z0-9_]*)\s*\(", text, flags=re.M)
    return sorted(set(n for n in names if n not in ("defined",)))


def test_header_declares_the_named_entry_points():
    names = declared_functions()
    for n in ["fp8_block_quant", "fp8_block_dequant", "mxfp8_quant", "mxfp8_dequant",
              "nvfp4_quant", "nvfp4_dequant", "nvfp4_fake_quant", "nvfp4_group_amax",
              "nvfp4_workspace_size", "pwq_status_string", "pwq_build_info"]:
        assert n in names, n


def test_library_exports_every_declared_symbol():
    L = _lib()
    raw = ctypes.CDLL(L.LIB_PATH)
    missing = [n for n in declared_functions() if not hasattr(raw, n)]
    assert not missing, missing


def test_build_is_exact_math():
    L = _lib()
    info = L.lib.pwq_build_info().decode()
    assert "sm_100a" in info
    for flag in ("-ftz=false", "-prec-div=true", "-prec-sqrt=true", "-fmad=false"):
        assert flag in info
    assert "no --use_fast_math" in info


def test_status_strings():
    L = _lib()
    assert L.status_string(0) == "PWQ_OK"
    assert L.status_string(L.PWQ_ERR_OVERLAP) == "PWQ_ERR_OVERLAP"
    assert L.status_string(99) == "PWQ_ERR_UNKNOWN"


def T(L, ptr, b, m, n, bs, rs):
    return L.PwqTensor(ptr, b, m, n, bs, rs)


def test_validation_errors_without_gpu():
    L = _lib()
    lib = L.lib
    by = ctypes.byref
    base = 1 << 40                       # never dereferenced: validation fails first
    x = T(L, base, 1, 256, 512, 256 * 512, 512)
    q = T(L, base + (1 << 30), 1, 256, 512, 256 * 512, 512)
    s = base + (1 << 31)
    # null descriptors and pointers
    assert lib.fp8_block_quant(None, by(q), s, None) == L.PWQ_ERR_NULL
    assert lib.fp8_block_quant(by(x), by(q), None, None) == L.PWQ_ERR_NULL
    xn = T(L, None, 1, 256, 512, 256 * 512, 512)
    assert lib.fp8_block_quant(by(xn), by(q), s, None) == L.PWQ_ERR_NULL
    # alignment
    xa = T(L, base + 8, 1, 256, 512, 256 * 512, 512)                 # BF16 base must be 16-aligned
    assert lib.fp8_block_quant(by(xa), by(q), s, None) == L.PWQ_ERR_ALIGN
    xr = T(L, base, 1, 256, 512, 256 * 516, 516)          # 1032-byte rows: not 16-aligned
    assert lib.fp8_block_quant(by(xr), by(q), s, None) == L.PWQ_ERR_ALIGN
    assert lib.fp8_block_quant(by(x), by(q), s + 2, None) == L.PWQ_ERR_ALIGN
    # stride too small
    xs = T(L, base, 1, 256, 512, 256 * 256, 256)
    assert lib.fp8_block_quant(by(xs), by(q), s, None) == L.PWQ_ERR_STRIDE
    xb = T(L, base, 2, 256, 512, 100 * 512, 512)
    qb = T(L, base + (1 << 30), 2, 256, 512, 256 * 512, 512)
    assert lib.fp8_block_quant(by(xb), by(qb), s, None) == L.PWQ_ERR_STRIDE
    # shape mismatch, negative extents
    q2 = T(L, base + (1 << 30), 1, 128, 512, 128 * 512, 512)
    assert lib.fp8_block_quant(by(x), by(q2), s, None) == L.PWQ_ERR_SHAPE
    xneg = T(L, base, 1, -1, 512, 0, 512)
    assert lib.fp8_block_quant(by(xneg), by(xneg), s, None) == L.PWQ_ERR_SHAPE
    # overlap: codes written over the input, scales written over the codes
    qo = T(L, base + 4096, 1, 256, 512, 256 * 512, 512)
    assert lib.fp8_block_quant(by(x), by(qo), s, None) == L.PWQ_ERR_OVERLAP
    assert lib.fp8_block_quant(by(x), by(q), base + (1 << 30) + 64, None) == L.PWQ_ERR_OVERLAP
    # MXFP8 / NVFP4 divisibility
    x33 = T(L, base, 1, 4, 48, 4 * 48, 48)
    q33 = T(L, base + (1 << 30), 1, 4, 48, 4 * 48, 48)
    assert lib.mxfp8_quant(by(x33), by(q33), s, None) == L.PWQ_ERR_SHAPE
    x24 = T(L, base, 1, 4, 24, 4 * 24, 24)
    assert lib.nvfp4_group_amax(by(x24), 1, s, None) == L.PWQ_ERR_SHAPE
    # empty tensors are a no-op that succeeds (no CUDA call is made)
    xe = T(L, None, 1, 0, 512, 0, 512)
    assert lib.fp8_block_quant(by(xe), by(xe), None, None) == L.PWQ_OK
    assert lib.mxfp8_quant(by(xe), by(xe), None, None) == L.PWQ_OK


def test_nvfp4_validation_without_gpu():
    L = _lib()
    lib = L.lib
    base = 1 << 40
    xs = (L.PwqTensor * 2)(T(L, base, 1, 64, 256, 64 * 256, 256),
                           T(L, base + (1 << 24), 1, 32, 256, 32 * 256, 256))
    qs = (L.PwqTensor * 2)(T(L, base + (1 << 30), 1, 64, 256, 64 * 128, 128),
                           T(L, base + (1 << 30) + (1 << 24), 1, 32, 256, 32 * 128, 128))
    sb = (ctypes.c_void_p * 2)(base + (2 << 30), base + (2 << 30) + (1 << 24))
    gs = base + (3 << 30)
    ws = base + (4 << 30)
    assert lib.nvfp4_workspace_size(2, xs) == 256
    # sibling count
    assert lib.nvfp4_quant(xs, 0, qs, sb, gs, None, ws, 256, None) == L.PWQ_ERR_ARG
    assert lib.nvfp4_quant(xs, 9, qs, sb, gs, None, ws, 256, None) == L.PWQ_ERR_ARG
    # workspace required without amax_in
    assert lib.nvfp4_quant(xs, 2, qs, sb, gs, None, None, 0, None) == L.PWQ_ERR_WORKSPACE
    assert lib.nvfp4_quant(xs, 2, qs, sb, gs, None, ws, 2, None) == L.PWQ_ERR_WORKSPACE
    # batch mismatch between siblings
    xm = (L.PwqTensor * 2)(xs[0], T(L, base + (1 << 24), 2, 32, 256, 32 * 256, 256))
    assert lib.nvfp4_quant(xm, 2, qs, sb, gs, None, ws, 256, None) == L.PWQ_ERR_ARG
    # fake-quant: exact alias allowed (validation passes to the launch), partial overlap not
    ys = (L.PwqTensor * 2)(T(L, base + 32, 1, 64, 256, 64 * 256, 256), xs[1])
    assert lib.nvfp4_fake_quant(xs, ys, 2, None, None, ws, 256, None) == L.PWQ_ERR_OVERLAP
    xe = (L.PwqTensor * 2)(xs[0], T(L, base + (1 << 24), 1, 64, 256, 64 * 256, 256))
    ys2 = (L.PwqTensor * 2)(xe[1], xe[0])                # outputs swapped onto the other input
    assert lib.nvfp4_fake_quant(xe, ys2, 2, None, None, ws, 256, None) == L.PWQ_ERR_OVERLAP
    assert lib.nvfp4_fake_quant(xe, xe, 2, None, None, xs[0].ptr + 64, 256, None) == L.PWQ_ERR_OVERLAP
    # overlap of the block scales with an input
    sbo = (ctypes.c_void_p * 2)(base + 64, base + (2 << 30) + (1 << 24))
    assert lib.nvfp4_quant(xs, 2, qs, sbo, gs, None, ws, 256, None) == L.PWQ_ERR_OVERLAP


def test_python_binding_names_match_the_abi():
    import precision_weight_quantization_b200 as P
    for n in ["fp8_block_quant", "fp8_block_dequant", "mxfp8_quant", "mxfp8_dequant", "nvfp4_quant",
              "nvfp4_dequant", "nvfp4_fake_quant", "nvfp4_group_amax", "nvfp4_workspace_size"]:
        assert callable(getattr(P, n))
    with pytest.raises(ValueError):
        import torch
        P.fp8_block_quant(torch.zeros(4, 4, dtype=torch.bfloat16))    # CPU tensor refused


def test_requant_validation_without_gpu():
    L = _lib()
    lib = L.lib
    by = ctypes.byref
    base = 1 << 40
    q = T(L, base, 1, 256, 512, 256 * 512, 512)
    qo = T(L, base + (1 << 30), 1, 256, 512, 256 * 512, 512)
    s = base + (2 << 30)
    so = base + (3 << 30)
    # nulls, alignment, shape
    assert lib.fp8_block_requant(by(q), None, by(qo), so, None) == L.PWQ_ERR_NULL
    assert lib.fp8_block_requant(by(q), s, by(qo), None, None) == L.PWQ_ERR_NULL
    assert lib.fp8_block_requant(by(q), s + 2, by(qo), so, None) == L.PWQ_ERR_ALIGN
    qa = T(L, base + 4, 1, 256, 512, 256 * 512, 512)                  # codes: 8-byte aligned base
    assert lib.fp8_block_requant(by(qa), s, by(qo), so, None) == L.PWQ_ERR_ALIGN
    q2 = T(L, base + (1 << 30), 1, 128, 512, 128 * 512, 512)
    assert lib.fp8_block_requant(by(q), s, by(q2), so, None) == L.PWQ_ERR_SHAPE
    # overlap: partial overlap of the output codes, new scales over the input codes
    qp = T(L, base + 64, 1, 256, 512, 256 * 512, 512)
    assert lib.fp8_block_requant(by(q), s, by(qp), so, None) == L.PWQ_ERR_OVERLAP
    assert lib.fp8_block_requant(by(q), s, by(qo), base + 128, None) == L.PWQ_ERR_OVERLAP
    # MXFP8 target: N % 32, scale bytes must not overlap
    q48 = T(L, base, 1, 4, 48, 4 * 48, 48)
    assert lib.fp8_block_requant_mxfp8(by(q48), s, by(q48), so, None) == L.PWQ_ERR_SHAPE
    assert lib.fp8_block_requant_mxfp8(by(q), s, by(qo), base + 8, None) == L.PWQ_ERR_OVERLAP
    # NVFP4 target
    qs = (L.PwqTensor * 2)(q, T(L, base + (1 << 24), 1, 64, 512, 64 * 512, 512))
    pk = (L.PwqTensor * 2)(T(L, base + (4 << 30), 1, 256, 512, 256 * 256, 256),
                           T(L, base + (4 << 30) + (1 << 24), 1, 64, 512, 64 * 256, 256))
    ss = (ctypes.c_void_p * 2)(s, s + 4096)
    sb = (ctypes.c_void_p * 2)(base + (5 << 30), base + (5 << 30) + (1 << 24))
    gs = base + (6 << 30)
    ws = base + (7 << 30)
    assert lib.fp8_block_requant_nvfp4_workspace_size(2, qs) == lib.nvfp4_workspace_size(2, qs) == 256
    assert lib.fp8_block_requant_nvfp4(qs, ss, 0, pk, sb, gs, None, ws, 256, None) == L.PWQ_ERR_ARG
    assert lib.fp8_block_requant_nvfp4(qs, ss, 2, pk, sb, gs, None, None, 0, None) == L.PWQ_ERR_WORKSPACE
    ss_null = (ctypes.c_void_p * 2)(s, None)
    assert lib.fp8_block_requant_nvfp4(qs, ss_null, 2, pk, sb, gs, None, ws, 256, None) == L.PWQ_ERR_NULL
    sbo = (ctypes.c_void_p * 2)(base + 256, base + (5 << 30) + (1 << 24))   # block scales over the codes
    assert lib.fp8_block_requant_nvfp4(qs, ss, 2, pk, sbo, gs, None, ws, 256, None) == L.PWQ_ERR_OVERLAP
    q24 = (L.PwqTensor * 1)(T(L, base, 1, 4, 24, 4 * 24, 24))
    assert lib.fp8_block_requant_nvfp4(q24, ss, 1, q24, sb, gs, None, ws, 256, None) == L.PWQ_ERR_SHAPE
    # empty input: a no-op that succeeds
    qe = T(L, None, 1, 0, 512, 0, 512)
    assert lib.fp8_block_requant(by(qe), None, by(qe), None, None) == L.PWQ_OK


def test_observer_validation_without_gpu():
    L = _lib()
    lib = L.lib
    by = ctypes.byref
    base = 1 << 40
    x = T(L, base, 1, 64, 256, 64 * 256, 256)
    st = base + (1 << 30)
    ws = base + (2 << 30)
    assert lib.nvfp4_observe_workspace_size() == 256
    assert lib.nvfp4_activation_observe(by(x), 3, 0.0, st, None, None, ws, 256, None) == L.PWQ_ERR_ARG
    assert lib.nvfp4_activation_observe(by(x), 2, 1.5, st, None, None, ws, 256, None) == L.PWQ_ERR_ARG
    assert lib.nvfp4_activation_observe(by(x), 2, float("nan"), st, None, None, ws, 256, None) == L.PWQ_ERR_ARG
    assert lib.nvfp4_activation_observe(by(x), 1, 0.0, None, None, None, ws, 256, None) == L.PWQ_ERR_NULL
    assert lib.nvfp4_activation_observe(by(x), 1, 0.0, st + 2, None, None, ws, 256, None) == L.PWQ_ERR_ALIGN
    assert lib.nvfp4_activation_observe(by(x), 1, 0.0, st, None, None, None, 0, None) == L.PWQ_ERR_WORKSPACE
    assert lib.nvfp4_activation_observe(by(x), 1, 0.0, base + 64, None, None, ws, 256, None) == L.PWQ_ERR_OVERLAP
    x24 = T(L, base, 1, 4, 24, 4 * 32, 32)
    assert lib.nvfp4_activation_observe(by(x24), 1, 0.0, st, None, None, ws, 256, None) == L.PWQ_ERR_SHAPE


def test_noalloc_validation_without_gpu():
    """nvfp4_fake_quant_noalloc: the 4096-group limit of its static scratch,
    lifted when amax_in is given, and the overlap rules, all decided before
    any CUDA call."""
    L = _lib()
    lib = L.lib
    base = 1 << 40
    by = ctypes.byref
    big = T(L, base, 4097, 1, 16, 16, 16)
    ybig = T(L, base + (1 << 30), 4097, 1, 16, 16, 16)
    assert lib.nvfp4_fake_quant_noalloc(by(big), by(ybig), 1, None, None, None) == L.PWQ_ERR_SHAPE
    assert "4096" in lib.pwq_last_error_detail().decode()
    # y partly over x, amax_out over x, y over amax_in: overlaps
    x = T(L, base, 3, 64, 512, 64 * 512, 512)
    y_part = T(L, base + 1024, 3, 64, 512, 64 * 512, 512)
    y = T(L, base + (1 << 30), 3, 64, 512, 64 * 512, 512)
    assert lib.nvfp4_fake_quant_noalloc(by(x), by(y_part), 1, None, None, None) == L.PWQ_ERR_OVERLAP
    assert lib.nvfp4_fake_quant_noalloc(by(x), by(y), 1, None, base + 64, None) == L.PWQ_ERR_OVERLAP
    assert lib.nvfp4_fake_quant_noalloc(by(x), by(y), 1, base + (1 << 30) + 32, None, None) == L.PWQ_ERR_OVERLAP
    # misaligned amax_out; shape mismatch between x and y; N % 16
    assert lib.nvfp4_fake_quant_noalloc(by(x), by(y), 1, None, base + (2 << 30) + 2, None) == L.PWQ_ERR_ALIGN
    y2 = T(L, base + (1 << 30), 3, 32, 512, 32 * 512, 512)
    assert lib.nvfp4_fake_quant_noalloc(by(x), by(y2), 1, None, None, None) == L.PWQ_ERR_SHAPE
    x24 = T(L, base, 1, 4, 24, 4 * 24, 24)
    y24 = T(L, base + (1 << 30), 1, 4, 24, 4 * 24, 24)
    assert lib.nvfp4_fake_quant_noalloc(by(x24), by(y24), 1, None, None, None) == L.PWQ_ERR_SHAPE


def test_flow_timeout_selftest_validation_without_gpu():
    L = _lib()
    lib = L.lib
    base = 1 << 40
    by = ctypes.byref
    x = T(L, base, 3, 64, 512, 64 * 512, 512)
    y = T(L, base + (1 << 30), 3, 64, 512, 64 * 512, 512)
    ws = base + (2 << 30)
    n = lib.pwq_selftest_flow_timeout_workspace_size(by(x))
    assert n == 256
    assert lib.pwq_selftest_flow_timeout(by(x), by(y), 10, ws, n, None) == L.PWQ_ERR_ARG
    assert lib.pwq_selftest_flow_timeout(by(x), by(y), 3 * 10 ** 9, ws, n, None) == L.PWQ_ERR_ARG
    assert lib.pwq_selftest_flow_timeout(by(x), by(y), 10 ** 6, ws, n - 4, None) == L.PWQ_ERR_WORKSPACE
    assert lib.pwq_selftest_flow_timeout(by(x), by(y), 10 ** 6, None, n, None) == L.PWQ_ERR_WORKSPACE
    assert lib.pwq_selftest_flow_timeout(by(x), by(x), 10 ** 6, ws, n, None) == L.PWQ_ERR_OVERLAP
    assert lib.pwq_selftest_flow_timeout(by(x), by(y), 10 ** 6, base + 64, n, None) == L.PWQ_ERR_OVERLAP
    xb = T(L, base, 513, 1, 16, 16, 16)
    yb = T(L, base + (1 << 30), 513, 1, 16, 16, 16)
    assert lib.pwq_selftest_flow_timeout_workspace_size(by(xb)) == 0
    assert lib.pwq_selftest_flow_timeout(by(xb), by(yb), 10 ** 6, ws, 1 << 20, None) == L.PWQ_ERR_SHAPE
    xe = T(L, None, 1, 0, 512, 0, 512)
    assert lib.pwq_selftest_flow_timeout(by(xe), by(xe), 10 ** 6, ws, n, None) == L.PWQ_ERR_SHAPE


def test_scale_layout_validation_without_gpu():
    L = _lib()
    lib = L.lib
    base = 1 << 40
    assert lib.pwq_mma_scale_bytes(2, 200, 10) == 2 * 2 * 3 * 512
    assert lib.pwq_mma_scale_bytes(1, 128, 4) == 512
    assert lib.pwq_mma_scale_bytes(-1, 1, 1) == 0
    d, m = base, base + (1 << 30)
    assert lib.pwq_scales_to_mma(None, 1, 128, 4, m, None) == L.PWQ_ERR_NULL
    assert lib.pwq_scales_to_mma(d, 1, 128, 4, m + 8, None) == L.PWQ_ERR_ALIGN
    assert lib.pwq_scales_to_mma(d, 1, -1, 4, m, None) == L.PWQ_ERR_SHAPE
    assert lib.pwq_scales_to_mma(d, 1, 128, 4, d + 256, None) == L.PWQ_ERR_OVERLAP
    assert lib.pwq_scales_from_mma(m, 1, 128, 4, m + 100, None) == L.PWQ_ERR_OVERLAP
    assert lib.pwq_scales_to_mma(None, 0, 128, 4, None, None) == L.PWQ_OK           # empty: no-op
    # the fused quantisers check the tile-layout extent against the other operands
    by = ctypes.byref
    x = (L.PwqTensor * 1)(T(L, base, 1, 256, 512, 256 * 512, 512))
    q = (L.PwqTensor * 1)(T(L, base + (1 << 30), 1, 256, 512, 256 * 512, 512))
    sc_over_q = (ctypes.c_void_p * 1)(base + (1 << 30) + 64)
    assert lib.mxfp8_quant_grouped_mma(1, x, q, sc_over_q, None) == L.PWQ_ERR_OVERLAP
    pk = (L.PwqTensor * 1)(T(L, base + (1 << 30), 1, 256, 512, 256 * 256, 256))
    sb_over_x = (ctypes.c_void_p * 1)(base + 1024)
    gs = (ctypes.c_void_p * 1)(base + (3 << 30))
    sizes = (ctypes.c_int * 1)(1)
    ws = base + (4 << 30)
    assert lib.nvfp4_quant_grouped_mma(1, sizes, x, pk, sb_over_x, gs, ws, 256, None) == L.PWQ_ERR_OVERLAP
    x24 = (L.PwqTensor * 1)(T(L, base, 1, 4, 48, 4 * 48, 48))
    q24 = (L.PwqTensor * 1)(T(L, base + (1 << 30), 1, 4, 48, 4 * 48, 48))
    sc = (ctypes.c_void_p * 1)(base + (2 << 30))
    assert lib.mxfp8_quant_grouped_mma(1, x24, q24, sc, None) == L.PWQ_ERR_SHAPE


def test_4over6_validation_without_gpu():
    """nvfp4_4over6_quant / _fake_quant: e4m3_max, siblings, workspace and
    overlap rules, all decided before any CUDA call."""
    L = _lib()
    lib = L.lib
    base = 1 << 40
    xs = (L.PwqTensor * 2)(T(L, base, 3, 64, 256, 64 * 256, 256),
                           T(L, base + (1 << 24), 3, 32, 256, 32 * 256, 256))
    qs = (L.PwqTensor * 2)(T(L, base + (1 << 30), 3, 64, 256, 64 * 128, 128),
                           T(L, base + (1 << 30) + (1 << 24), 3, 32, 256, 32 * 128, 128))
    sb = (ctypes.c_void_p * 2)(base + (2 << 30), base + (2 << 30) + (1 << 24))
    gs = base + (3 << 30)
    ws = base + (4 << 30)
    assert lib.nvfp4_4over6_workspace_size(2, xs) == 256
    big = T(L, base, 100, 16, 16, 256, 16)
    assert lib.nvfp4_4over6_workspace_size(1, ctypes.byref(big)) == 512
    assert lib.nvfp4_4over6_workspace_size(0, xs) == 0
    for E in (0, 255, 257, 447, 449, 1000):
        assert lib.nvfp4_4over6_quant(xs, 2, qs, sb, gs, None, E, ws, 256, None) == L.PWQ_ERR_ARG
        assert lib.nvfp4_4over6_fake_quant(xs, xs, 2, None, None, E, ws, 256, None) == L.PWQ_ERR_ARG
    assert "e4m3_max" in lib.pwq_last_error_detail().decode()
    assert lib.nvfp4_4over6_quant(xs, 0, qs, sb, gs, None, 256, ws, 256, None) == L.PWQ_ERR_ARG
    assert lib.nvfp4_4over6_quant(xs, 9, qs, sb, gs, None, 256, ws, 256, None) == L.PWQ_ERR_ARG
    # workspace: required without amax_in, at least 4 bytes per batch index
    assert lib.nvfp4_4over6_quant(xs, 2, qs, sb, gs, None, 256, None, 0, None) == L.PWQ_ERR_WORKSPACE
    assert lib.nvfp4_4over6_quant(xs, 2, qs, sb, gs, None, 256, ws, 8, None) == L.PWQ_ERR_WORKSPACE
    assert lib.nvfp4_4over6_quant(xs, 2, qs, sb, gs, None, 256, ws + 2, 256, None) == L.PWQ_ERR_WORKSPACE
    # null global scale, misaligned amax_in
    assert lib.nvfp4_4over6_quant(xs, 2, qs, sb, None, None, 256, ws, 256, None) == L.PWQ_ERR_NULL
    assert lib.nvfp4_4over6_quant(xs, 2, qs, sb, gs, gs + 66, 448, None, 0, None) == L.PWQ_ERR_ALIGN
    # overlaps: block scales over an input, workspace over an output, y over the other input
    sbo = (ctypes.c_void_p * 2)(base + 64, base + (2 << 30) + (1 << 24))
    assert lib.nvfp4_4over6_quant(xs, 2, qs, sbo, gs, None, 256, ws, 256, None) == L.PWQ_ERR_OVERLAP
    assert lib.nvfp4_4over6_quant(xs, 2, qs, sb, gs, None, 256, gs, 256, None) == L.PWQ_ERR_OVERLAP
    xe = (L.PwqTensor * 2)(T(L, base, 1, 64, 256, 64 * 256, 256), T(L, base + (1 << 24), 1, 64, 256, 64 * 256, 256))
    ys = (L.PwqTensor * 2)(xe[1], xe[0])
    assert lib.nvfp4_4over6_fake_quant(xe, ys, 2, None, None, 256, ws, 256, None) == L.PWQ_ERR_OVERLAP
    # N % 16 and shape mismatch
    x24 = T(L, base, 1, 4, 24, 4 * 32, 32)
    y24 = T(L, base + (1 << 30), 1, 4, 24, 4 * 32, 32)
    assert lib.nvfp4_4over6_fake_quant(ctypes.byref(x24), ctypes.byref(y24), 1, None, None, 256, ws, 256,
                                       None) == L.PWQ_ERR_SHAPE
    # empty tensors: a no-op that succeeds without a CUDA call
    xz = T(L, None, 1, 0, 256, 0, 256)
    assert lib.nvfp4_4over6_fake_quant(ctypes.byref(xz), ctypes.byref(xz), 1, None, None, 256, None, 0,
                                       None) == L.PWQ_OK


def test_4over6_grouped_validation_without_gpu():
    L = _lib()
    lib = L.lib
    base = 1 << 40
    IP = ctypes.c_int * 2
    xs = (L.PwqTensor * 3)(T(L, base, 4, 64, 256, 64 * 256, 256), T(L, base + (1 << 24), 4, 32, 256, 32 * 256, 256),
                           T(L, base + (1 << 26), 2, 16, 512, 16 * 512, 512))
    ys = (L.PwqTensor * 3)(T(L, base + (1 << 30), 4, 64, 256, 64 * 256, 256),
                           T(L, base + (1 << 30) + (1 << 24), 4, 32, 256, 32 * 256, 256),
                           T(L, base + (1 << 30) + (1 << 26), 2, 16, 512, 16 * 512, 512))
    sizes = IP(2, 1)
    # 4 + 2 instances: 24 bytes, rounded up to 256
    assert lib.nvfp4_4over6_workspace_size_grouped(2, sizes, xs) == 256
    assert lib.nvfp4_4over6_workspace_size_grouped(2, IP(2, 9), xs) == 0
    ws = base + (4 << 30)
    ao = (ctypes.c_void_p * 2)(None, None)
    assert lib.nvfp4_4over6_fake_quant_grouped(2, sizes, xs, ys, ao, 300, ws, 256, None) == L.PWQ_ERR_ARG
    assert lib.nvfp4_4over6_fake_quant_grouped(2, sizes, xs, ys, ao, 256, None, 0, None) == L.PWQ_ERR_WORKSPACE
    assert lib.nvfp4_4over6_fake_quant_grouped(0, sizes, xs, ys, ao, 256, ws, 256, None) == L.PWQ_ERR_ARG
    assert lib.nvfp4_4over6_fake_quant_grouped(2, IP(2, 0), xs, ys, ao, 256, ws, 256, None) == L.PWQ_ERR_ARG
    # an output of group 1 over an input of group 0
    ys2 = (L.PwqTensor * 3)(ys[0], ys[1], T(L, base + 512, 2, 16, 512, 16 * 512, 512))
    assert lib.nvfp4_4over6_fake_quant_grouped(2, sizes, xs, ys2, ao, 256, ws, 256, None) == L.PWQ_ERR_OVERLAP
    # quantise: a missing global scale of the second group
    qs = (L.PwqTensor * 3)(T(L, base + (1 << 30), 4, 64, 256, 64 * 128, 128),
                           T(L, base + (1 << 30) + (1 << 24), 4, 32, 256, 32 * 128, 128),
                           T(L, base + (1 << 30) + (1 << 26), 2, 16, 512, 16 * 256, 256))
    sb = (ctypes.c_void_p * 3)(base + (2 << 30), base + (2 << 30) + (1 << 24), base + (2 << 30) + (1 << 26))
    gs = (ctypes.c_void_p * 2)(base + (3 << 30), None)
    assert lib.nvfp4_4over6_quant_grouped(2, sizes, xs, qs, sb, gs, 256, ws, 256, None) == L.PWQ_ERR_NULL
