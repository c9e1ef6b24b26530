"""B200-native block-scaled quantisation of BF16 tensors: FP8 block-wise
(128x128, FP32 scales), MXFP8 (1x32, UE8M0) and NVFP4 (1x16, E4M3 block
scale + FP32 global scale), quantise / dequantise / fake-quantise.

Formats as listed on "Low Precision RL" ("Choose a precision" table); NVFP4
fake-quantisation with sibling-shared global amax and the straight-through
backward as described in the verl NVFP4 QAT article (sections 2.3, 2.4).

This module is argument marshalling only: every step runs in libpwq's CUDA
kernels (include/pwq.h).  PyTorch supplies device memory and the stream.
Functions take CUDA tensors ([M, N] or batched [B, M, N], last dimension
contiguous) and return newly allocated outputs unless ``out=`` buffers are
given.  Nothing synchronises.
"""
import ctypes
from typing import List, Optional, Sequence, Tuple

import torch

from ._lib import (LIB_PATH, PWQ_MAX_SIBLINGS, PwqError, PwqTensor, check, lib,  # noqa: F401
                   status_string)

__all__ = [
    "fp8_block_quant", "fp8_block_dequant", "mxfp8_quant", "mxfp8_dequant",
    "nvfp4_group_amax", "nvfp4_quant", "nvfp4_dequant", "nvfp4_fake_quant",
    "nvfp4_workspace_size", "NVFP4FakeQuantSTE", "nvfp4_fake_quant_ste", "build_info",
    "device_error", "PwqError", "LIB_PATH", "fp8_block_quant_grouped", "fp8_block_dequant_grouped",
    "mxfp8_quant_grouped", "mxfp8_dequant_grouped", "nvfp4_dequant_grouped", "nvfp4_quant_grouped",
    "nvfp4_fake_quant_grouped", "fp8_block_requant", "fp8_block_requant_mxfp8", "fp8_block_requant_nvfp4",
    "fp8_block_requant_nvfp4_grouped", "fp8_block_requant_grouped", "fp8_block_requant_mxfp8_grouped",
    "NVFP4ActivationObserver", "nvfp4_w4a4_fake_quant_ste", "OBSERVERS", "mma_scale_bytes", "scales_to_mma",
    "scales_from_mma", "mxfp8_quant_grouped_mma", "nvfp4_quant_grouped_mma",
]

_CODE_DTYPES = (torch.uint8, torch.float8_e4m3fn)


def _stream(t: torch.Tensor):
    return ctypes.c_void_p(torch.cuda.current_stream(t.device).cuda_stream)


def _bmn(t: torch.Tensor, name: str):
    if t.dim() == 2:
        M, N = t.shape
        return 1, M, N, M * t.stride(0), t.stride(0)
    if t.dim() == 3:
        B, M, N = t.shape
        return B, M, N, t.stride(0), t.stride(1)
    raise ValueError("%s must be 2-D [M, N] or 3-D [B, M, N], got shape %s" % (name, tuple(t.shape)))


def _desc(t: torch.Tensor, name: str, packed: bool = False) -> PwqTensor:
    """pwq_tensor for a [M, N] / [B, M, N] CUDA tensor.  For packed E2M1 codes
    (uint8, two per byte) the logical column count is twice the byte count."""
    if not t.is_cuda:
        raise ValueError("%s must be a CUDA tensor" % name)
    B, M, N, bs, rs = _bmn(t, name)
    if t.numel() == 0:
        # an empty tensor's strides are arbitrary; the library launches nothing for it
        return PwqTensor(t.data_ptr(), B, M, 2 * N if packed else N, M * N, N)
    if N > 1 and t.stride(-1) != 1:
        raise ValueError("%s: last dimension must be contiguous" % name)
    return PwqTensor(t.data_ptr(), B, M, 2 * N if packed else N, bs, rs)


def _lead(x: torch.Tensor):
    return tuple(x.shape[:-2]) if x.dim() == 3 else ()


def _check_dtype(t, dtypes, name):
    if t.dtype not in dtypes:
        raise TypeError("%s must have dtype in %s, got %s" % (name, dtypes, t.dtype))


# ---------------------------------------------------------------- FP8 block-wise

def fp8_block_quant(x: torch.Tensor, out: Optional[torch.Tensor] = None,
                    scale: Optional[torch.Tensor] = None) -> Tuple[torch.Tensor, torch.Tensor]:
    """128x128 block-wise FP8: returns (codes float8_e4m3fn [.., M, N],
    scale float32 [.., ceil(M/128), ceil(N/128)]) with s = fl(amax/448)."""
    _check_dtype(x, (torch.bfloat16,), "x")
    M, N = x.shape[-2:]
    if out is None:
        out = torch.empty(x.shape, dtype=torch.float8_e4m3fn, device=x.device)
    if scale is None:
        scale = torch.empty(_lead(x) + (-(-M // 128), -(-N // 128)), dtype=torch.float32, device=x.device)
    _check_dtype(out, _CODE_DTYPES, "out")
    dx, dq = _desc(x, "x"), _desc(out, "out")
    check(lib.fp8_block_quant(ctypes.byref(dx), ctypes.byref(dq), scale.data_ptr(), _stream(x)),
          "fp8_block_quant")
    return out, scale


def fp8_block_dequant(q: torch.Tensor, scale: torch.Tensor,
                      out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """BF16 y = bf16(fl(dec(q) * s)) for FP8 block-wise codes and scales."""
    _check_dtype(q, _CODE_DTYPES, "q")
    if out is None:
        out = torch.empty(q.shape, dtype=torch.bfloat16, device=q.device)
    if not scale.is_contiguous() or scale.dtype != torch.float32:
        raise ValueError("scale must be a contiguous float32 tensor")
    dq, dy = _desc(q, "q"), _desc(out, "out")
    check(lib.fp8_block_dequant(ctypes.byref(dq), scale.data_ptr(), ctypes.byref(dy), _stream(q)),
          "fp8_block_dequant")
    return out


# ---------------------------------------------------------------- MXFP8

def mxfp8_quant(x: torch.Tensor, out: Optional[torch.Tensor] = None,
                scale: Optional[torch.Tensor] = None) -> Tuple[torch.Tensor, torch.Tensor]:
    """MXFP8 1x32: returns (codes float8_e4m3fn [.., M, N], UE8M0 scale bytes
    uint8 [.., M, N/32])."""
    _check_dtype(x, (torch.bfloat16,), "x")
    if out is None:
        out = torch.empty(x.shape, dtype=torch.float8_e4m3fn, device=x.device)
    if scale is None:
        scale = torch.empty(x.shape[:-1] + (x.shape[-1] // 32,), dtype=torch.uint8, device=x.device)
    dx, dq = _desc(x, "x"), _desc(out, "out")
    check(lib.mxfp8_quant(ctypes.byref(dx), ctypes.byref(dq), scale.data_ptr(), _stream(x)), "mxfp8_quant")
    return out, scale


def mxfp8_dequant(q: torch.Tensor, scale: torch.Tensor, out: Optional[torch.Tensor] = None) -> torch.Tensor:
    _check_dtype(q, _CODE_DTYPES, "q")
    if out is None:
        out = torch.empty(q.shape, dtype=torch.bfloat16, device=q.device)
    if not scale.is_contiguous():
        raise ValueError("scale must be contiguous")
    dq, dy = _desc(q, "q"), _desc(out, "out")
    check(lib.mxfp8_dequant(ctypes.byref(dq), scale.data_ptr(), ctypes.byref(dy), _stream(q)),
          "mxfp8_dequant")
    return out


# ---------------------------------------------------------------- NVFP4

def _siblings(xs) -> List[torch.Tensor]:
    if isinstance(xs, torch.Tensor):
        xs = [xs]
    xs = list(xs)
    if not 1 <= len(xs) <= PWQ_MAX_SIBLINGS:
        raise ValueError("1..%d sibling tensors expected" % PWQ_MAX_SIBLINGS)
    for i, x in enumerate(xs):
        _check_dtype(x, (torch.bfloat16,), "x[%d]" % i)
    return xs


def _desc_array(ts, name, packed=False):
    arr = (PwqTensor * len(ts))()
    for i, t in enumerate(ts):
        arr[i] = _desc(t, "%s[%d]" % (name, i), packed)
    return arr


def _batch(x: torch.Tensor) -> int:
    return x.shape[0] if x.dim() == 3 else 1


def nvfp4_workspace_size(xs) -> int:
    xs = _siblings(xs)
    return int(lib.nvfp4_workspace_size(len(xs), _desc_array(xs, "x")))


def _workspace(xs, arr) -> torch.Tensor:
    n = int(lib.nvfp4_workspace_size(len(xs), arr))
    return torch.empty(max(n, 256), dtype=torch.uint8, device=xs[0].device)


def nvfp4_group_amax(xs, out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Group amax A_b = max |x| over all siblings' batch slice b, float32 [B].
    This is the value to all-reduce (MAX) when a group is sharded."""
    xs = _siblings(xs)
    if out is None:
        out = torch.empty(_batch(xs[0]), dtype=torch.float32, device=xs[0].device)
    arr = _desc_array(xs, "x")
    check(lib.nvfp4_group_amax(arr, len(xs), out.data_ptr(), _stream(xs[0])), "nvfp4_group_amax")
    return out


def nvfp4_quant(xs, amax: Optional[torch.Tensor] = None, out=None, sb=None,
                global_scale: Optional[torch.Tensor] = None):
    """NVFP4 quantisation of a sibling group (one tensor or a list sharing
    one global amax per batch index).  Returns (packed codes list uint8
    [.., M, N/2], block scales list float8_e4m3fn [.., M, N/16], global
    scales float32 [B]).  ``amax`` (float32 [B]) replaces the on-device
    group amax reduction (cached or all-reduced value)."""
    single = isinstance(xs, torch.Tensor)
    xs = _siblings(xs)
    dev = xs[0].device
    B = _batch(xs[0])
    if out is None:
        out = [torch.empty(x.shape[:-1] + (x.shape[-1] // 2,), dtype=torch.uint8, device=dev) for x in xs]
    if sb is None:
        sb = [torch.empty(x.shape[:-1] + (x.shape[-1] // 16,), dtype=torch.float8_e4m3fn, device=dev)
              for x in xs]
    if global_scale is None:
        global_scale = torch.empty(B, dtype=torch.float32, device=dev)
    for t in sb:
        if not t.is_contiguous():
            raise ValueError("block scale tensors must be contiguous")
    ax = _desc_array(xs, "x")
    aq = _desc_array(out, "out", packed=True)
    sbp = (ctypes.c_void_p * len(xs))(*[t.data_ptr() for t in sb])
    ws = None if amax is not None else _workspace(xs, ax)
    check(lib.nvfp4_quant(ax, len(xs), aq, sbp, global_scale.data_ptr(),
                          amax.data_ptr() if amax is not None else None,
                          ws.data_ptr() if ws is not None else None,
                          ws.numel() if ws is not None else 0, _stream(xs[0])), "nvfp4_quant")
    if single:
        return out[0], sb[0], global_scale
    return out, sb, global_scale


def nvfp4_dequant(packed: torch.Tensor, sb: torch.Tensor, global_scale: torch.Tensor,
                  out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """BF16 y = bf16(fl((dec(c) * dec(sb)) * gs)) for one NVFP4 tensor."""
    _check_dtype(packed, (torch.uint8,), "packed")
    if out is None:
        out = torch.empty(packed.shape[:-1] + (packed.shape[-1] * 2,), dtype=torch.bfloat16,
                          device=packed.device)
    if not sb.is_contiguous() or not global_scale.is_contiguous():
        raise ValueError("sb and global_scale must be contiguous")
    dq, dy = _desc(packed, "packed", packed=True), _desc(out, "out")
    check(lib.nvfp4_dequant(ctypes.byref(dq), sb.data_ptr(), global_scale.data_ptr(), ctypes.byref(dy),
                            _stream(packed)), "nvfp4_dequant")
    return out


def nvfp4_fake_quant(xs, amax: Optional[torch.Tensor] = None, out=None, inplace: bool = False,
                     amax_out: Optional[torch.Tensor] = None):
    """NVFP4 QDQ of a sibling group: BF16 outputs equal to
    nvfp4_dequant(nvfp4_quant(x)), without materialising codes.  Returns the
    output tensor (single input) or list of outputs."""
    single = isinstance(xs, torch.Tensor)
    xs = _siblings(xs)
    if out is None:
        out = xs if inplace else [torch.empty_like(x) for x in xs]
    elif isinstance(out, torch.Tensor):
        out = [out]
    ax = _desc_array(xs, "x")
    ay = _desc_array(out, "out")
    ws = None if amax is not None else _workspace(xs, ax)
    check(lib.nvfp4_fake_quant(ax, ay, len(xs), amax.data_ptr() if amax is not None else None,
                               amax_out.data_ptr() if amax_out is not None else None,
                               ws.data_ptr() if ws is not None else None,
                               ws.numel() if ws is not None else 0, _stream(xs[0])), "nvfp4_fake_quant")
    return out[0] if single else out


class NVFP4FakeQuantSTE(torch.autograd.Function):
    """Fake-quantised forward, straight-through backward: grad_x = grad_y and
    no gradient for the amax (verl NVFP4 QAT article, section 2.3)."""

    @staticmethod
    def forward(ctx, x: torch.Tensor, amax: Optional[torch.Tensor] = None):
        return nvfp4_fake_quant(x, amax=amax)

    @staticmethod
    def backward(ctx, grad_y):
        return grad_y, None


class _SiblingSTE(torch.autograd.Function):
    @staticmethod
    def forward(ctx, amax, *xs):
        return tuple(nvfp4_fake_quant(list(xs), amax=amax))

    @staticmethod
    def backward(ctx, *grads):
        return (None,) + tuple(grads)


def nvfp4_fake_quant_ste(xs: Sequence[torch.Tensor], amax: Optional[torch.Tensor] = None):
    """Sibling-group fake-quantisation with the straight-through backward."""
    if isinstance(xs, torch.Tensor):
        return NVFP4FakeQuantSTE.apply(xs, amax)
    return list(_SiblingSTE.apply(amax, *xs))


# ---------------------------------------------------------------- NVFP4 4over6

def nvfp4_4over6_quant(xs, e4m3_max: int = 256, amax: Optional[torch.Tensor] = None, out=None, sb=None,
                       global_scale: Optional[torch.Tensor] = None):
    """NVFP4 "4over6" quantisation of a sibling group (vime pull request
    #503, NVFP4 QDQ config: NVTE_NVFP4_4OVER6, E4M3 maximum 256 by default).
    Every block keeps the candidate -- its amax mapped to 6 or to 4 -- whose
    dequantised values have the smaller squared error; gs = fl(A / (6 E)).
    Returns what nvfp4_quant returns; nvfp4_dequant reads the result."""
    single = isinstance(xs, torch.Tensor)
    xs = _siblings(xs)
    dev = xs[0].device
    B = _batch(xs[0])
    if out is None:
        out = [torch.empty(x.shape[:-1] + (x.shape[-1] // 2,), dtype=torch.uint8, device=dev) for x in xs]
    if sb is None:
        sb = [torch.empty(x.shape[:-1] + (x.shape[-1] // 16,), dtype=torch.float8_e4m3fn, device=dev)
              for x in xs]
    if global_scale is None:
        global_scale = torch.empty(B, dtype=torch.float32, device=dev)
    for t in sb:
        if not t.is_contiguous():
            raise ValueError("block scale tensors must be contiguous")
    ax = _desc_array(xs, "x")
    aq = _desc_array(out, "out", packed=True)
    sbp = (ctypes.c_void_p * len(xs))(*[t.data_ptr() for t in sb])
    ws = None
    if amax is None:
        ws = torch.empty(max(int(lib.nvfp4_4over6_workspace_size(len(xs), ax)), 256), dtype=torch.uint8, device=dev)
    check(lib.nvfp4_4over6_quant(ax, len(xs), aq, sbp, global_scale.data_ptr(),
                                 amax.data_ptr() if amax is not None else None, int(e4m3_max),
                                 ws.data_ptr() if ws is not None else None,
                                 ws.numel() if ws is not None else 0, _stream(xs[0])), "nvfp4_4over6_quant")
    if single:
        return out[0], sb[0], global_scale
    return out, sb, global_scale


def nvfp4_4over6_fake_quant(xs, e4m3_max: int = 256, amax: Optional[torch.Tensor] = None, out=None,
                            inplace: bool = False, amax_out: Optional[torch.Tensor] = None):
    """BF16 outputs equal to nvfp4_dequant(nvfp4_4over6_quant(x)), without
    materialising codes.  Returns the output tensor or list of outputs."""
    single = isinstance(xs, torch.Tensor)
    xs = _siblings(xs)
    if out is None:
        out = xs if inplace else [torch.empty_like(x) for x in xs]
    elif isinstance(out, torch.Tensor):
        out = [out]
    ax = _desc_array(xs, "x")
    ay = _desc_array(out, "out")
    ws = None
    if amax is None:
        ws = torch.empty(max(int(lib.nvfp4_4over6_workspace_size(len(xs), ax)), 256), dtype=torch.uint8,
                         device=xs[0].device)
    check(lib.nvfp4_4over6_fake_quant(ax, ay, len(xs), amax.data_ptr() if amax is not None else None,
                                      amax_out.data_ptr() if amax_out is not None else None, int(e4m3_max),
                                      ws.data_ptr() if ws is not None else None,
                                      ws.numel() if ws is not None else 0, _stream(xs[0])),
          "nvfp4_4over6_fake_quant")
    return out[0] if single else out


# ---------------------------------------------------------------- grouped calls (one launch per list)

def _ptrs(ts):
    return (ctypes.c_void_p * len(ts))(*[t.data_ptr() for t in ts])


def fp8_block_quant_grouped(xs: Sequence[torch.Tensor], out=None, scale=None):
    """fp8_block_quant of every tensor of a list (a layer's weights) in one
    launch.  Returns (codes list, scales list)."""
    xs = list(xs)
    for i, x in enumerate(xs):
        _check_dtype(x, (torch.bfloat16,), "x[%d]" % i)
    if out is None:
        out = [torch.empty(x.shape, dtype=torch.float8_e4m3fn, device=x.device) for x in xs]
    if scale is None:
        scale = [torch.empty(_lead(x) + (-(-x.shape[-2] // 128), -(-x.shape[-1] // 128)), dtype=torch.float32,
                             device=x.device) for x in xs]
    if xs:
        check(lib.fp8_block_quant_grouped(len(xs), _desc_array(xs, "x"), _desc_array(out, "out"), _ptrs(scale),
                                          _stream(xs[0])), "fp8_block_quant_grouped")
    return out, scale


def fp8_block_dequant_grouped(qs: Sequence[torch.Tensor], scales: Sequence[torch.Tensor], out=None):
    qs = list(qs)
    if out is None:
        out = [torch.empty(q.shape, dtype=torch.bfloat16, device=q.device) for q in qs]
    if qs:
        check(lib.fp8_block_dequant_grouped(len(qs), _desc_array(qs, "q"), _ptrs(scales), _desc_array(out, "out"),
                                            _stream(qs[0])), "fp8_block_dequant_grouped")
    return out


def mxfp8_quant_grouped(xs: Sequence[torch.Tensor], out=None, scale=None):
    xs = list(xs)
    if out is None:
        out = [torch.empty(x.shape, dtype=torch.float8_e4m3fn, device=x.device) for x in xs]
    if scale is None:
        scale = [torch.empty(x.shape[:-1] + (x.shape[-1] // 32,), dtype=torch.uint8, device=x.device) for x in xs]
    if xs:
        check(lib.mxfp8_quant_grouped(len(xs), _desc_array(xs, "x"), _desc_array(out, "out"), _ptrs(scale),
                                      _stream(xs[0])), "mxfp8_quant_grouped")
    return out, scale


def mxfp8_dequant_grouped(qs: Sequence[torch.Tensor], scales: Sequence[torch.Tensor], out=None):
    qs = list(qs)
    if out is None:
        out = [torch.empty(q.shape, dtype=torch.bfloat16, device=q.device) for q in qs]
    if qs:
        check(lib.mxfp8_dequant_grouped(len(qs), _desc_array(qs, "q"), _ptrs(scales), _desc_array(out, "out"),
                                        _stream(qs[0])), "mxfp8_dequant_grouped")
    return out


def nvfp4_dequant_grouped(packed: Sequence[torch.Tensor], sb: Sequence[torch.Tensor],
                          global_scale: Sequence[torch.Tensor], out=None):
    packed = list(packed)
    if out is None:
        out = [torch.empty(p.shape[:-1] + (p.shape[-1] * 2,), dtype=torch.bfloat16, device=p.device)
               for p in packed]
    if packed:
        check(lib.nvfp4_dequant_grouped(len(packed), _desc_array(packed, "packed", packed=True), _ptrs(sb),
                                        _ptrs(global_scale), _desc_array(out, "out"), _stream(packed[0])),
              "nvfp4_dequant_grouped")
    return out


def _groups(groups):
    groups = [_siblings(g) for g in groups]
    flat = [x for g in groups for x in g]
    sizes = (ctypes.c_int * len(groups))(*[len(g) for g in groups])
    return groups, flat, sizes


def nvfp4_quant_grouped(groups: Sequence[Sequence[torch.Tensor]], out=None, sb=None, global_scale=None):
    """NVFP4 quantisation of several sibling groups (e.g. a layer's {q,k,v},
    {o}, {gate,up}, {down}) in one single-pass launch.  Returns (packed
    codes per group, block scales per group, global scales per group)."""
    groups, flat, sizes = _groups(groups)
    dev = flat[0].device
    if out is None:
        out = [[torch.empty(x.shape[:-1] + (x.shape[-1] // 2,), dtype=torch.uint8, device=dev) for x in g]
               for g in groups]
    if sb is None:
        sb = [[torch.empty(x.shape[:-1] + (x.shape[-1] // 16,), dtype=torch.float8_e4m3fn, device=dev) for x in g]
              for g in groups]
    if global_scale is None:
        global_scale = [torch.empty(_batch(g[0]), dtype=torch.float32, device=dev) for g in groups]
    ax = _desc_array(flat, "x")
    ws_bytes = int(lib.nvfp4_workspace_size_grouped(len(groups), sizes, ax))
    ws = torch.empty(max(ws_bytes, 256), dtype=torch.uint8, device=dev)
    check(lib.nvfp4_quant_grouped(len(groups), sizes, ax, _desc_array([p for g in out for p in g], "out", packed=True),
                                  _ptrs([s for g in sb for s in g]), _ptrs(global_scale), ws.data_ptr(), ws.numel(),
                                  _stream(flat[0])), "nvfp4_quant_grouped")
    return out, sb, global_scale


def nvfp4_fake_quant_grouped(groups: Sequence[Sequence[torch.Tensor]], out=None, inplace: bool = False,
                             amax_out=None):
    """NVFP4 fake-quantisation of several sibling groups in one single-pass
    launch.  Returns the BF16 outputs per group."""
    groups, flat, sizes = _groups(groups)
    dev = flat[0].device
    if out is None:
        out = groups if inplace else [[torch.empty_like(x) for x in g] for g in groups]
    ax = _desc_array(flat, "x")
    ws_bytes = int(lib.nvfp4_workspace_size_grouped(len(groups), sizes, ax))
    ws = torch.empty(max(ws_bytes, 256), dtype=torch.uint8, device=dev)
    ao = None
    if amax_out is not None:
        ao = (ctypes.c_void_p * len(groups))(*[a.data_ptr() if a is not None else None for a in amax_out])
    check(lib.nvfp4_fake_quant_grouped(len(groups), sizes, ax, _desc_array([y for g in out for y in g], "out"), ao,
                                       ws.data_ptr(), ws.numel(), _stream(flat[0])), "nvfp4_fake_quant_grouped")
    return out


def nvfp4_4over6_quant_grouped(groups: Sequence[Sequence[torch.Tensor]], e4m3_max: int = 256, out=None, sb=None,
                               global_scale=None):
    """NVFP4 "4over6" quantisation of several sibling groups (two launches per
    16 members).  Returns what nvfp4_quant_grouped returns."""
    groups, flat, sizes = _groups(groups)
    dev = flat[0].device
    if out is None:
        out = [[torch.empty(x.shape[:-1] + (x.shape[-1] // 2,), dtype=torch.uint8, device=dev) for x in g]
               for g in groups]
    if sb is None:
        sb = [[torch.empty(x.shape[:-1] + (x.shape[-1] // 16,), dtype=torch.float8_e4m3fn, device=dev) for x in g]
              for g in groups]
    if global_scale is None:
        global_scale = [torch.empty(_batch(g[0]), dtype=torch.float32, device=dev) for g in groups]
    ax = _desc_array(flat, "x")
    ws_bytes = int(lib.nvfp4_4over6_workspace_size_grouped(len(groups), sizes, ax))
    ws = torch.empty(max(ws_bytes, 256), dtype=torch.uint8, device=dev)
    check(lib.nvfp4_4over6_quant_grouped(len(groups), sizes, ax,
                                         _desc_array([p for g in out for p in g], "out", packed=True),
                                         _ptrs([s for g in sb for s in g]), _ptrs(global_scale), int(e4m3_max),
                                         ws.data_ptr(), ws.numel(), _stream(flat[0])), "nvfp4_4over6_quant_grouped")
    return out, sb, global_scale


def nvfp4_4over6_fake_quant_grouped(groups: Sequence[Sequence[torch.Tensor]], e4m3_max: int = 256, out=None,
                                    inplace: bool = False, amax_out=None):
    """NVFP4 "4over6" fake-quantisation of several sibling groups.  Returns
    the BF16 outputs per group."""
    groups, flat, sizes = _groups(groups)
    dev = flat[0].device
    if out is None:
        out = groups if inplace else [[torch.empty_like(x) for x in g] for g in groups]
    ax = _desc_array(flat, "x")
    ws_bytes = int(lib.nvfp4_4over6_workspace_size_grouped(len(groups), sizes, ax))
    ws = torch.empty(max(ws_bytes, 256), dtype=torch.uint8, device=dev)
    ao = None
    if amax_out is not None:
        ao = (ctypes.c_void_p * len(groups))(*[a.data_ptr() if a is not None else None for a in amax_out])
    check(lib.nvfp4_4over6_fake_quant_grouped(len(groups), sizes, ax, _desc_array([y for g in out for y in g], "out"),
                                              ao, int(e4m3_max), ws.data_ptr(), ws.numel(), _stream(flat[0])),
          "nvfp4_4over6_fake_quant_grouped")
    return out


# ---------------------------------------------------------------- block scales in the tensor-core layout

def mma_scale_bytes(batch: int, rows: int, scale_cols: int) -> int:
    """Bytes of an [B][M][S] scale array in the tensor-core tile layout
    (include/pwq.h: 128 x 4 tiles of 512 bytes, zero padding)."""
    return int(lib.pwq_mma_scale_bytes(batch, rows, scale_cols))


def _scale_shape(dense_or_shape):
    shape = tuple(dense_or_shape.shape) if isinstance(dense_or_shape, torch.Tensor) else tuple(dense_or_shape)
    return (1,) + shape if len(shape) == 2 else shape


def scales_to_mma(dense: torch.Tensor, out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Dense scale bytes [.., M, S] (uint8 or float8_e4m3fn) -> the tile
    layout, a flat uint8 tensor of mma_scale_bytes(B, M, S) bytes."""
    if not dense.is_contiguous():
        raise ValueError("dense scales must be contiguous")
    B, M, S = _scale_shape(dense)
    if out is None:
        out = torch.empty(mma_scale_bytes(B, M, S), dtype=torch.uint8, device=dense.device)
    check(lib.pwq_scales_to_mma(dense.data_ptr(), B, M, S, out.data_ptr(), _stream(dense)), "pwq_scales_to_mma")
    return out


def scales_from_mma(mma: torch.Tensor, shape, out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """The tile layout back to dense uint8 scale bytes of `shape` ([M, S] or [B, M, S])."""
    B, M, S = _scale_shape(shape)
    if out is None:
        out = torch.empty(tuple(shape), dtype=torch.uint8, device=mma.device)
    check(lib.pwq_scales_from_mma(mma.data_ptr(), B, M, S, out.data_ptr(), _stream(mma)), "pwq_scales_from_mma")
    return out


def mxfp8_quant_grouped_mma(xs: Sequence[torch.Tensor], out=None, scale=None):
    """mxfp8_quant_grouped with every tensor's UE8M0 scales written in the
    tensor-core tile layout.  Returns (codes list, flat uint8 scale arrays)."""
    xs = list(xs)
    if out is None:
        out = [torch.empty(x.shape, dtype=torch.float8_e4m3fn, device=x.device) for x in xs]
    if scale is None:
        scale = [torch.empty(mma_scale_bytes(*_scale_shape(x.shape[:-1] + (x.shape[-1] // 32,))), dtype=torch.uint8,
                             device=x.device) for x in xs]
    if xs:
        check(lib.mxfp8_quant_grouped_mma(len(xs), _desc_array(xs, "x"), _desc_array(out, "out"), _ptrs(scale),
                                          _stream(xs[0])), "mxfp8_quant_grouped_mma")
    return out, scale


def nvfp4_quant_grouped_mma(groups: Sequence[Sequence[torch.Tensor]], out=None, sb=None, global_scale=None):
    """nvfp4_quant_grouped with the E4M3 block scales written in the
    tensor-core tile layout (flat uint8 arrays, one per member)."""
    groups, flat, sizes = _groups(groups)
    dev = flat[0].device
    if out is None:
        out = [[torch.empty(x.shape[:-1] + (x.shape[-1] // 2,), dtype=torch.uint8, device=dev) for x in g]
               for g in groups]
    if sb is None:
        sb = [[torch.empty(mma_scale_bytes(*_scale_shape(x.shape[:-1] + (x.shape[-1] // 16,))), dtype=torch.uint8,
                           device=dev) for x in g] for g in groups]
    if global_scale is None:
        global_scale = [torch.empty(_batch(g[0]), dtype=torch.float32, device=dev) for g in groups]
    ax = _desc_array(flat, "x")
    ws_bytes = int(lib.nvfp4_workspace_size_grouped(len(groups), sizes, ax))
    ws = torch.empty(max(ws_bytes, 256), dtype=torch.uint8, device=dev)
    check(lib.nvfp4_quant_grouped_mma(len(groups), sizes, ax,
                                      _desc_array([p for g in out for p in g], "out", packed=True),
                                      _ptrs([s for g in sb for s in g]), _ptrs(global_scale), ws.data_ptr(),
                                      ws.numel(), _stream(flat[0])), "nvfp4_quant_grouped_mma")
    return out, sb, global_scale


# ---------------------------------------------------------------- diagnostics

# ---------------------------------------------------------------- FP8 block-wise -> rollout formats

def _fp8_input(q, scale, name="q"):
    _check_dtype(q, _CODE_DTYPES, name)
    if not scale.is_contiguous() or scale.dtype != torch.float32:
        raise ValueError("scale must be a contiguous float32 tensor")


def fp8_block_requant(q: torch.Tensor, scale: torch.Tensor, out: Optional[torch.Tensor] = None,
                      scale_out: Optional[torch.Tensor] = None, inplace: bool = False):
    """FP8 block-wise codes + tile scales -> the FP8 block-wise codes and
    scales of their dequantised BF16 values, in one pass (no BF16 tensor):
    fp8_block_quant(fp8_block_dequant(q, scale)).  inplace=True overwrites
    q and scale."""
    _fp8_input(q, scale)
    if out is None:
        out = q if inplace else torch.empty(q.shape, dtype=torch.float8_e4m3fn, device=q.device)
    if scale_out is None:
        scale_out = scale if inplace else torch.empty_like(scale)
    _check_dtype(out, _CODE_DTYPES, "out")
    dq, do = _desc(q, "q"), _desc(out, "out")
    check(lib.fp8_block_requant(ctypes.byref(dq), scale.data_ptr(), ctypes.byref(do), scale_out.data_ptr(),
                                _stream(q)), "fp8_block_requant")
    return out, scale_out


def fp8_block_requant_mxfp8(q: torch.Tensor, scale: torch.Tensor, out: Optional[torch.Tensor] = None,
                            scale_out: Optional[torch.Tensor] = None, inplace: bool = False):
    """FP8 block-wise -> MXFP8 in one pass: mxfp8_quant(fp8_block_dequant(q,
    scale)).  Returns (codes, UE8M0 bytes [.., M, N/32]); inplace=True
    writes the codes over q."""
    _fp8_input(q, scale)
    if out is None:
        out = q if inplace else torch.empty(q.shape, dtype=torch.float8_e4m3fn, device=q.device)
    if scale_out is None:
        scale_out = torch.empty(q.shape[:-1] + (q.shape[-1] // 32,), dtype=torch.uint8, device=q.device)
    _check_dtype(out, _CODE_DTYPES, "out")
    dq, do = _desc(q, "q"), _desc(out, "out")
    check(lib.fp8_block_requant_mxfp8(ctypes.byref(dq), scale.data_ptr(), ctypes.byref(do),
                                      scale_out.data_ptr(), _stream(q)), "fp8_block_requant_mxfp8")
    return out, scale_out


def fp8_block_requant_nvfp4(qs, scales, amax: Optional[torch.Tensor] = None, out=None, sb=None,
                            global_scale: Optional[torch.Tensor] = None):
    """A sibling group of FP8 block-wise members -> NVFP4 in one pass (amax
    over the dequantised members, then encode): nvfp4_quant of the
    dequantised group.  Returns (packed codes list, block scales list,
    global scales [B]) like nvfp4_quant; ``amax`` replaces the reduction."""
    single = isinstance(qs, torch.Tensor)
    qs = [qs] if single else list(qs)
    scales = [scales] if isinstance(scales, torch.Tensor) else list(scales)
    if not 1 <= len(qs) <= PWQ_MAX_SIBLINGS or len(scales) != len(qs):
        raise ValueError("1..%d members, one scale tensor each" % PWQ_MAX_SIBLINGS)
    for i, (q, s_) in enumerate(zip(qs, scales)):
        _fp8_input(q, s_, "q[%d]" % i)
    dev = qs[0].device
    B = _batch(qs[0])
    if out is None:
        out = [torch.empty(q.shape[:-1] + (q.shape[-1] // 2,), dtype=torch.uint8, device=dev) for q in qs]
    if sb is None:
        sb = [torch.empty(q.shape[:-1] + (q.shape[-1] // 16,), dtype=torch.float8_e4m3fn, device=dev) for q in qs]
    if global_scale is None:
        global_scale = torch.empty(B, dtype=torch.float32, device=dev)
    aq = _desc_array(qs, "q")
    ao = _desc_array(out, "out", packed=True)
    sp = (ctypes.c_void_p * len(qs))(*[t.data_ptr() for t in scales])
    sbp = (ctypes.c_void_p * len(qs))(*[t.data_ptr() for t in sb])
    ws = None
    if amax is None:
        n = int(lib.fp8_block_requant_nvfp4_workspace_size(len(qs), aq))
        ws = torch.empty(max(n, 256), dtype=torch.uint8, device=dev)
    check(lib.fp8_block_requant_nvfp4(aq, sp, len(qs), ao, sbp, global_scale.data_ptr(),
                                      amax.data_ptr() if amax is not None else None,
                                      ws.data_ptr() if ws is not None else None,
                                      ws.numel() if ws is not None else 0, _stream(qs[0])),
          "fp8_block_requant_nvfp4")
    if single:
        return out[0], sb[0], global_scale
    return out, sb, global_scale


def fp8_block_requant_grouped(qs: Sequence[torch.Tensor], scales: Sequence[torch.Tensor], out=None,
                              scale_out=None, inplace: bool = False):
    """fp8_block_requant over a list of tensors in one launch per 16."""
    qs, scales = list(qs), list(scales)
    for i, (q, s_) in enumerate(zip(qs, scales)):
        _fp8_input(q, s_, "q[%d]" % i)
    if out is None:
        out = qs if inplace else [torch.empty(q.shape, dtype=torch.float8_e4m3fn, device=q.device) for q in qs]
    if scale_out is None:
        scale_out = scales if inplace else [torch.empty_like(s_) for s_ in scales]
    check(lib.fp8_block_requant_grouped(len(qs), _desc_array(qs, "q"), _ptrs(scales), _desc_array(out, "out"),
                                        _ptrs(scale_out), _stream(qs[0])), "fp8_block_requant_grouped")
    return out, scale_out


def fp8_block_requant_mxfp8_grouped(qs: Sequence[torch.Tensor], scales: Sequence[torch.Tensor], out=None,
                                    scale_out=None, inplace: bool = False):
    """fp8_block_requant_mxfp8 over a list of tensors in one launch per 16."""
    qs, scales = list(qs), list(scales)
    for i, (q, s_) in enumerate(zip(qs, scales)):
        _fp8_input(q, s_, "q[%d]" % i)
    if out is None:
        out = qs if inplace else [torch.empty(q.shape, dtype=torch.float8_e4m3fn, device=q.device) for q in qs]
    if scale_out is None:
        scale_out = [torch.empty(q.shape[:-1] + (q.shape[-1] // 32,), dtype=torch.uint8, device=q.device)
                     for q in qs]
    check(lib.fp8_block_requant_mxfp8_grouped(len(qs), _desc_array(qs, "q"), _ptrs(scales),
                                              _desc_array(out, "out"), _ptrs(scale_out), _stream(qs[0])),
          "fp8_block_requant_mxfp8_grouped")
    return out, scale_out


def fp8_block_requant_nvfp4_grouped(groups, scales, out=None, sb=None, global_scale=None):
    """Several sibling groups of FP8 block-wise members (codes; `scales`
    mirrors `groups` with their tile scales) -> NVFP4 in one single-pass
    launch.  Returns (packed codes per group, block scales per group, global
    scales per group)."""
    groups = [list(g) for g in groups]
    scales = [list(g) for g in scales]
    if [len(g) for g in groups] != [len(g) for g in scales]:
        raise ValueError("scales must mirror groups")
    for gi, g in enumerate(groups):
        if not 1 <= len(g) <= PWQ_MAX_SIBLINGS:
            raise ValueError("1..%d members per group" % PWQ_MAX_SIBLINGS)
        for i, (q, s_) in enumerate(zip(g, scales[gi])):
            _fp8_input(q, s_, "groups[%d][%d]" % (gi, i))
    flat = [q for g in groups for q in g]
    sizes = (ctypes.c_int * len(groups))(*[len(g) for g in groups])
    dev = flat[0].device
    if out is None:
        out = [[torch.empty(q.shape[:-1] + (q.shape[-1] // 2,), dtype=torch.uint8, device=dev) for q in g]
               for g in groups]
    if sb is None:
        sb = [[torch.empty(q.shape[:-1] + (q.shape[-1] // 16,), dtype=torch.float8_e4m3fn, device=dev) for q in g]
              for g in groups]
    if global_scale is None:
        global_scale = [torch.empty(_batch(g[0]), dtype=torch.float32, device=dev) for g in groups]
    aq = _desc_array(flat, "q")
    ws_bytes = int(lib.fp8_block_requant_nvfp4_workspace_size_grouped(len(groups), sizes, aq))
    ws = torch.empty(max(ws_bytes, 256), dtype=torch.uint8, device=dev)
    check(lib.fp8_block_requant_nvfp4_grouped(len(groups), sizes, aq, _ptrs([t for g in scales for t in g]),
                                              _desc_array([p_ for g in out for p_ in g], "out", packed=True),
                                              _ptrs([t for g in sb for t in g]), _ptrs(global_scale),
                                              ws.data_ptr(), ws.numel(), _stream(flat[0])),
          "fp8_block_requant_nvfp4_grouped")
    return out, sb, global_scale


# ---------------------------------------------------------------- W4A4 activation observers

OBSERVERS = {"memoryless_minmax": 0, "static_minmax": 1, "minmax": 2}


class NVFP4ActivationObserver:
    """An activation observer of W4A4 NVFP4 fake-quantisation (verl NVFP4 QAT
    article 2.2 / 3.1): keeps the running extremes (lo, hi) of the activations
    it sees on the device and gives the activation's amax and
    input_global_scale = fl(amax / 2688).  kind: "static_minmax" (default),
    "memoryless_minmax" or "minmax" (moving average with constant
    `averaging_constant`); the exact rules are those of nvfp4_activation_observe
    in include/pwq.h.  No host synchronisation."""

    def __init__(self, kind: str = "static_minmax", averaging_constant: float = 0.01, device="cuda"):
        if kind not in OBSERVERS:
            raise ValueError("observer kind must be one of %s" % sorted(OBSERVERS))
        self.kind = kind
        self.averaging_constant = float(averaging_constant)
        self.state = torch.tensor([float("inf"), float("-inf")], dtype=torch.float32, device=device)
        self.amax = torch.zeros(1, dtype=torch.float32, device=device)
        self.input_global_scale = torch.zeros(1, dtype=torch.float32, device=device)
        self._ws = torch.empty(int(lib.nvfp4_observe_workspace_size()), dtype=torch.uint8, device=device)

    def reset(self):
        self.state.copy_(torch.tensor([float("inf"), float("-inf")], dtype=torch.float32))

    def observe(self, x: torch.Tensor) -> torch.Tensor:
        """One observer step over x (BF16, last dim % 16 == 0); returns the
        amax tensor (float32 [1], on the device)."""
        _check_dtype(x, (torch.bfloat16,), "x")
        dx = _desc(x, "x")
        check(lib.nvfp4_activation_observe(ctypes.byref(dx), OBSERVERS[self.kind], self.averaging_constant,
                                           self.state.data_ptr(), self.amax.data_ptr(),
                                           self.input_global_scale.data_ptr(), self._ws.data_ptr(),
                                           self._ws.numel(), _stream(x)), "nvfp4_activation_observe")
        return self.amax

    def fake_quant(self, x: torch.Tensor, out=None) -> torch.Tensor:
        """Observe x, then NVFP4 fake-quantise it with the observed amax (one
        global scale for the whole tensor: a 3-D x gets the amax once per
        batch index, as nvfp4_fake_quant expects amax[B])."""
        amax = self.observe(x)
        if x.dim() == 3 and x.shape[0] != 1:
            amax = amax.expand(x.shape[0]).contiguous()
        return nvfp4_fake_quant(x, amax=amax, out=out)


class _W4A4STE(torch.autograd.Function):
    @staticmethod
    def forward(ctx, x, observer):
        return observer.fake_quant(x)

    @staticmethod
    def backward(ctx, grad_out):
        return grad_out, None


def nvfp4_w4a4_fake_quant_ste(x: torch.Tensor, observer: NVFP4ActivationObserver) -> torch.Tensor:
    """W4A4 activation fake-quantisation with the straight-through backward
    (the gradient passes unchanged, verl NVFP4 QAT article 2.3)."""
    return _W4A4STE.apply(x, observer)


def build_info() -> str:
    return lib.pwq_build_info().decode()


def device_error() -> int:
    """Reads and clears the device-side error word (synchronous)."""
    code = ctypes.c_uint32(0)
    check(lib.pwq_device_error(ctypes.byref(code)), "pwq_device_error")
    return int(code.value)
