"""numpy-level wrapper around the scalar C oracle (test infrastructure only).

Every function takes and returns dense numpy arrays; BF16 values travel as
their uint16 bit patterns.  The arithmetic is all in ``pwq_oracle.c``; this
module only allocates outputs and composes the per-format calls (for NVFP4:
the group amax over sibling tensors, then quantisation with that amax).

Formats and readings: see the header of ``pwq_oracle.c`` (block-scaled FP8,
MXFP8 and NVFP4 as defined on "Low Precision RL", "Choose a precision", and
the verl NVFP4 QAT article, sections 2.3-2.4 and 3.3).
"""
import ctypes
import os

import numpy as np

from . import build as _build

_LIB = None


def lib():
    global _LIB
    if _LIB is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        P = ctypes.c_void_p
        I64 = ctypes.c_int64
        F = ctypes.c_float
        L.or_fp_env_ok.restype = ctypes.c_int
        L.or_bf16_round.restype = ctypes.c_uint16
        L.or_bf16_round.argtypes = [F]
        L.or_e4m3_encode.restype = ctypes.c_uint8
        L.or_e4m3_encode.argtypes = [ctypes.c_double]
        L.or_e4m3_decode.restype = ctypes.c_double
        L.or_e4m3_decode.argtypes = [ctypes.c_uint8]
        L.or_e2m1_encode.restype = ctypes.c_uint8
        L.or_e2m1_encode.argtypes = [ctypes.c_double]
        L.or_e2m1_decode.restype = ctypes.c_double
        L.or_e2m1_decode.argtypes = [ctypes.c_uint8]
        L.or_ue8m0_exponent.restype = ctypes.c_int
        L.or_ue8m0_exponent.argtypes = [F]
        for name in ("or_bf16_round_array", "or_e4m3_encode_array",
                     "or_e2m1_encode_array", "or_ue8m0_byte_array"):
            getattr(L, name).argtypes = [P, P, I64]
            getattr(L, name).restype = None
        L.or_fp8_block_quant.argtypes = [P, I64, I64, I64, P, P]
        L.or_fp8_block_dequant.argtypes = [P, P, I64, I64, I64, P]
        L.or_mxfp8_quant.argtypes = [P, I64, I64, I64, P, P]
        L.or_mxfp8_dequant.argtypes = [P, P, I64, I64, I64, P]
        L.or_amax_bf16.argtypes = [P, I64]
        L.or_amax_bf16.restype = F
        L.or_nvfp4_global_scale.argtypes = [F]
        L.or_nvfp4_global_scale.restype = F
        L.or_nvfp4_quant.argtypes = [P, I64, I64, F, P, P]
        L.or_nvfp4_dequant.argtypes = [P, P, F, I64, I64, P]
        L.or_nvfp4_fake_quant.argtypes = [P, I64, I64, F, P]
        L.or_nvfp4_4over6_global_scale.argtypes = [F, ctypes.c_int]
        L.or_nvfp4_4over6_global_scale.restype = F
        L.or_nvfp4_4over6_quant.argtypes = [P, I64, I64, F, ctypes.c_int, P, P, P, P]
        L.or_nvfp4_4over6_fake_quant.argtypes = [P, I64, I64, F, ctypes.c_int, P]
        for name in ("or_fp8_block_quant", "or_fp8_block_dequant", "or_mxfp8_quant",
                     "or_mxfp8_dequant", "or_nvfp4_quant", "or_nvfp4_dequant",
                     "or_nvfp4_fake_quant", "or_nvfp4_4over6_quant", "or_nvfp4_4over6_fake_quant"):
            getattr(L, name).restype = None
        _LIB = L
    return _LIB


def _p(a):
    return a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    a = np.ascontiguousarray(a)
    assert a.dtype == dtype, (a.dtype, dtype)
    return a


def fp_env_ok():
    return bool(lib().or_fp_env_ok())


# ---------------------------------------------------------------- codecs

def bf16_round(v):
    v = _c(np.asarray(v, dtype=np.float32), np.float32)
    out = np.empty(v.shape, np.uint16)
    lib().or_bf16_round_array(_p(v), _p(out), v.size)
    return out


def e4m3_encode(v):
    v = _c(np.asarray(v, dtype=np.float32), np.float32)
    out = np.empty(v.shape, np.uint8)
    lib().or_e4m3_encode_array(_p(v), _p(out), v.size)
    return out


def e2m1_encode(v):
    v = _c(np.asarray(v, dtype=np.float32), np.float32)
    out = np.empty(v.shape, np.uint8)
    lib().or_e2m1_encode_array(_p(v), _p(out), v.size)
    return out


def ue8m0_byte(amax):
    a = _c(np.asarray(amax, dtype=np.float32), np.float32)
    out = np.empty(a.shape, np.uint8)
    lib().or_ue8m0_byte_array(_p(a), _p(out), a.size)
    return out


def e4m3_decode(code):
    return float(lib().or_e4m3_decode(int(code)))


def e2m1_decode(code):
    return float(lib().or_e2m1_decode(int(code)))


def bf16_to_f32(bits):
    bits = np.asarray(bits, dtype=np.uint16)
    return (bits.astype(np.uint32) << 16).view(np.float32)


# ---------------------------------------------------------------- FP8 block

def _bmn(x):
    if x.ndim == 2:
        return 1, x.shape[0], x.shape[1]
    assert x.ndim == 3
    return x.shape


def fp8_block_quant(x_bits):
    """x_bits: uint16 [M][N] or [B][M][N].  Returns (codes u8, scales f32
    [B][ceil(M/128)][ceil(N/128)]) with the input's leading shape."""
    x = _c(x_bits, np.uint16)
    B, M, N = _bmn(x)
    q = np.empty(x.shape, np.uint8)
    s = np.empty((B, -(-M // 128), -(-N // 128)), np.float32)
    if x.size:
        lib().or_fp8_block_quant(_p(x), B, M, N, _p(q), _p(s))
    if x.ndim == 2:
        s = s[0]
    return q, s


def fp8_block_dequant(q, s):
    q = _c(q, np.uint8)
    s = _c(s, np.float32)
    B, M, N = _bmn(q)
    y = np.empty(q.shape, np.uint16)
    if q.size:
        lib().or_fp8_block_dequant(_p(q), _p(s), B, M, N, _p(y))
    return y


# ---------------------------------------------------------------- MXFP8

def mxfp8_quant(x_bits):
    x = _c(x_bits, np.uint16)
    B, M, N = _bmn(x)
    assert N % 32 == 0
    q = np.empty(x.shape, np.uint8)
    e = np.empty(x.shape[:-1] + (N // 32,), np.uint8)
    if x.size:
        lib().or_mxfp8_quant(_p(x), B, M, N, _p(q), _p(e))
    return q, e


def mxfp8_dequant(q, e):
    q = _c(q, np.uint8)
    e = _c(e, np.uint8)
    B, M, N = _bmn(q)
    y = np.empty(q.shape, np.uint16)
    if q.size:
        lib().or_mxfp8_dequant(_p(q), _p(e), B, M, N, _p(y))
    return y


# ---------------------------------------------------------------- NVFP4

def amax_bf16(x_bits):
    x = _c(x_bits, np.uint16)
    return float(np.float32(lib().or_amax_bf16(_p(x), x.size)))


def nvfp4_group_amax(members):
    """A = max |x| over every element of every member of a sibling group."""
    return float(np.float32(max([amax_bf16(m) for m in members] + [0.0])))


def nvfp4_global_scale(group_amax):
    return float(np.float32(lib().or_nvfp4_global_scale(np.float32(group_amax))))


def _as_2d(x):
    return x.reshape(-1, x.shape[-1])


def nvfp4_quant(x_bits, group_amax):
    """One member tensor [..., M, N] with its group's amax.  Returns
    (packed u8 [..., N/2], sb u8 [..., N/16], gs f32)."""
    x = _c(x_bits, np.uint16)
    N = x.shape[-1]
    assert N % 16 == 0
    x2 = _as_2d(x)
    packed = np.empty(x.shape[:-1] + (N // 2,), np.uint8)
    sb = np.empty(x.shape[:-1] + (N // 16,), np.uint8)
    if x.size:
        lib().or_nvfp4_quant(_p(x2), x2.shape[0], N, np.float32(group_amax), _p(packed), _p(sb))
    return packed, sb, nvfp4_global_scale(group_amax)


def nvfp4_dequant(packed, sb, gs, N):
    packed = _c(packed, np.uint8)
    sb = _c(sb, np.uint8)
    M = packed.size // (N // 2) if N else 0
    y = np.empty(packed.shape[:-1] + (N,), np.uint16)
    if y.size:
        lib().or_nvfp4_dequant(_p(packed), _p(sb), np.float32(gs), M, N, _p(y))
    return y


def nvfp4_fake_quant(x_bits, group_amax):
    x = _c(x_bits, np.uint16)
    N = x.shape[-1]
    x2 = _as_2d(x)
    y = np.empty(x.shape, np.uint16)
    if x.size:
        lib().or_nvfp4_fake_quant(_p(x2), x2.shape[0], N, np.float32(group_amax), _p(y))
    return y


def nvfp4_quant_group(members):
    """Quantise a sibling group (list of member arrays sharing one amax)."""
    A = nvfp4_group_amax(members)
    return A, [nvfp4_quant(m, A) for m in members]


def unpack_e2m1(packed):
    """Packed bytes -> one code per element (element 2j from the low nibble)."""
    packed = np.asarray(packed, np.uint8)
    out = np.empty(packed.shape[:-1] + (packed.shape[-1] * 2,), np.uint8)
    out[..., 0::2] = packed & 0xF
    out[..., 1::2] = packed >> 4
    return out


# ---------------------------------------------------------------- NVFP4 "4over6"
#
# vime pull request #503, NVFP4 QDQ config thread: NVTE_NVFP4_4OVER6 and
# NVTE_NVFP4_4OVER6_E4M3_USE_256 (E4M3 maximum 256 instead of 448).  Each
# block is scaled so its amax maps to 6 or to 4 and keeps the candidate with
# the smaller squared error (readings R19-R21 of pwq_oracle.c; parity
# unpinned against the pages, which give no selection rule).  The result is
# plain NVFP4: nvfp4_dequant reads it.

def nvfp4_4over6_global_scale(group_amax, e4m3_max=256):
    return float(np.float32(lib().or_nvfp4_4over6_global_scale(np.float32(group_amax), int(e4m3_max))))


def nvfp4_4over6_quant(x_bits, group_amax, e4m3_max=256, details=False):
    """One member tensor [..., M, N] with its group's amax.  Returns (packed,
    sb, gs), plus (choice u8 [..., N/16] of 4 / 6, err f32 [..., N/16, 2]
    with the t = 6 error first) when ``details``."""
    x = _c(x_bits, np.uint16)
    N = x.shape[-1]
    assert N % 16 == 0
    x2 = _as_2d(x)
    packed = np.empty(x.shape[:-1] + (N // 2,), np.uint8)
    sb = np.empty(x.shape[:-1] + (N // 16,), np.uint8)
    choice = np.empty(x.shape[:-1] + (N // 16,), np.uint8)
    err = np.empty(x.shape[:-1] + (N // 16, 2), np.float32)
    if x.size:
        lib().or_nvfp4_4over6_quant(_p(x2), x2.shape[0], N, np.float32(group_amax), int(e4m3_max),
                                    _p(packed), _p(sb), _p(choice), _p(err))
    gs = nvfp4_4over6_global_scale(group_amax, e4m3_max)
    if details:
        return packed, sb, gs, choice, err
    return packed, sb, gs


def nvfp4_4over6_fake_quant(x_bits, group_amax, e4m3_max=256):
    x = _c(x_bits, np.uint16)
    N = x.shape[-1]
    x2 = _as_2d(x)
    y = np.empty(x.shape, np.uint16)
    if x.size:
        lib().or_nvfp4_4over6_fake_quant(_p(x2), x2.shape[0], N, np.float32(group_amax), int(e4m3_max), _p(y))
    return y


def nvfp4_4over6_quant_group(members, e4m3_max=256):
    """A sibling group under 4over6: (A, [(packed, sb, gs) per member])."""
    A = nvfp4_group_amax(members)
    return A, [nvfp4_4over6_quant(m, A, e4m3_max) for m in members]


# ---------------------------------------------------------------- FP8 block -> rollout formats
#
# "低精度训练与 Rollout", "FP8 训练 + FP8 Rollout" / "实现说明" item 3: on a
# weight update the FP8 training weights are dequantised to BF16 and the BF16
# weights are quantised into the rollout format.  The re-quantisation is
# defined as exactly that composition; the functions below are the plain
# composition of the pinned per-format functions above, with no shortcut.

def fp8_block_requant(q, s):
    """FP8 block codes + tile scales -> the FP8 block codes and scales of the
    dequantised BF16 tensor: fp8_block_quant(fp8_block_dequant(q, s))."""
    return fp8_block_quant(fp8_block_dequant(q, s))


def fp8_block_requant_mxfp8(q, s):
    """mxfp8_quant(fp8_block_dequant(q, s)); N % 32 == 0."""
    return mxfp8_quant(fp8_block_dequant(q, s))


def fp8_block_requant_nvfp4(qs, ss):
    """A sibling group given as FP8 block members (codes [M][N] or
    [B][M][N], tile scales): dequantise every member, then NVFP4-quantise
    the group with the amax of the dequantised members, per batch index.
    Returns (A [B], [(packed, sb)] per member, gs [B])."""
    ys = [fp8_block_dequant(q, s) for q, s in zip(qs, ss)]
    batched = ys[0].ndim == 3
    y3 = [y if batched else y[None] for y in ys]
    B = y3[0].shape[0]
    A = np.array([nvfp4_group_amax([y[b] for y in y3]) for b in range(B)], np.float32)
    gs = np.array([nvfp4_global_scale(a) for a in A], np.float32)
    out = []
    for y in y3:
        pk, sb = [], []
        for b in range(B):
            p, s_, _ = nvfp4_quant(y[b], A[b])
            pk.append(p)
            sb.append(s_)
        pk, sb = np.stack(pk), np.stack(sb)
        out.append((pk if batched else pk[0], sb if batched else sb[0]))
    return A, out, gs


# ---------------------------------------------------------------- W4A4 activation observers
#
# verl NVFP4 QAT article, 2.2 and 3.1: in W4A4 mode the activation has its own
# global scale (input_global_scale), kept by an activation observer named
# static_minmax (default), memoryless_minmax or minmax.  The names are all
# the pages give; the readings (stated with the library's C ABI) are:
#   state (lo, hi): binary32 minimum and maximum of the values observed,
#     empty = (+inf, -inf); the order on values is the numeric one with
#     -0 < +0, so the extremes of a tensor are unique;
#   memoryless_minmax: (lo, hi) = (min x, max x) of this tensor;
#   static_minmax:     (lo, hi) = (min(lo, min x), max(hi, max x));
#   minmax:            moving average with constant c: an empty state takes
#     (min x, max x); otherwise lo = fl(fl(fl(1 - c) * lo) + fl(c * min x)),
#     hi likewise;
# then A = max(|lo|, |hi|) and input_global_scale = fl(A / 2688) (as the
# weight global scale).  The state is updated before the tensor is
# quantised with A.

MEMORYLESS_MINMAX, STATIC_MINMAX, MINMAX = 0, 1, 2


def _bf16_key(bits):
    """BF16 bits -> unsigned keys in the order of the values (-0 < +0)."""
    b = np.asarray(bits, np.uint32)
    return np.where(b & 0x8000, (~b) & 0xFFFF, b | 0x8000)


def _key_bf16(key):
    k = int(key)
    return (k & 0x7FFF) if k & 0x8000 else ((~k) & 0xFFFF)


def activation_minmax(x_bits):
    """(min, max) of a BF16 tensor in the value order with -0 < +0."""
    k = _bf16_key(np.asarray(x_bits, np.uint16).ravel())
    lo = np.float32(bf16_to_f32(np.array([_key_bf16(k.min())], np.uint16))[0])
    hi = np.float32(bf16_to_f32(np.array([_key_bf16(k.max())], np.uint16))[0])
    return lo, hi


def _minf(a, b):
    # value order with -0 < +0 on binary32
    if a == b:
        return a if np.signbit(a) else b
    return a if a < b else b


def _maxf(a, b):
    if a == b:
        return b if np.signbit(a) else a
    return a if a > b else b


def observe(state, x_bits, kind, c=np.float32(0.01)):
    """One observer step.  state: float32 [2] (lo, hi).  Returns (new state,
    A, input_global_scale)."""
    lo, hi = np.float32(state[0]), np.float32(state[1])
    mn, mx = activation_minmax(x_bits)
    empty = lo > hi
    if kind == MEMORYLESS_MINMAX or (kind == MINMAX and empty):
        lo, hi = mn, mx
    elif kind == STATIC_MINMAX:
        lo, hi = _minf(lo, mn), _maxf(hi, mx)
    elif kind == MINMAX:
        c = np.float32(c)
        w = np.float32(np.float32(1) - c)
        lo = np.float32(np.float32(w * lo) + np.float32(c * mn))
        hi = np.float32(np.float32(w * hi) + np.float32(c * mx))
    else:
        raise ValueError("observer kind")
    A = np.float32(max(abs(lo), abs(hi)))
    return np.array([lo, hi], np.float32), A, np.float32(nvfp4_global_scale(A))

OBSERVERS_BY_NAME = {"memoryless_minmax": MEMORYLESS_MINMAX, "static_minmax": STATIC_MINMAX, "minmax": MINMAX}


# ---------------------------------------------------------------- tensor-core block-scale layout
#
# The block-scaled tensor-core MMA of sm_100 (PTX ISA, tcgen05.mma with
# block scaling; the scale factors reach tensor memory with tcgen05.cp's
# 32x128b.warpx4 shape, i.e. 32 rows of 16 bytes fanned out to four warps)
# and cuBLAS's 1D block-scaling-factor layout take the scale bytes of an
# [M][S] scale matrix (S = K / 32 for MXFP8, K / 16 for NVFP4) in tiles of
# 128 rows x 4 scale columns.  Each tile is 512 contiguous bytes, the tiles
# of one 128-row band follow each other along S, the bands follow each
# other along M, and inside a tile the scale of tile row r (0..127) and
# column c (0..3) sits at byte (r % 32) * 16 + (r // 32) * 4 + c.  Rows
# are padded to a multiple of 128 and columns to a multiple of 4 with zero
# bytes.  A batch [B][M][S] is B such slabs one after the other.  (The
# pages name the consumer -- the rollout GEMM takes the quantised weights,
# "Low Precision RL", "Modes" 3; the exporter repacks NVFP4 scales for the
# inference kernels, verl NVFP4 QAT article 2.5 -- but not the layout.)

def mma_scale_bytes(B, M, S):
    return B * (-(-M // 128)) * (-(-S // 4)) * 512


def mma_scale_offset(M, S, b, r, c):
    """Byte offset of the scale of (batch b, row r, scale column c)."""
    ct = -(-S // 4)
    slab = (-(-M // 128)) * ct * 512
    return b * slab + ((r // 128) * ct + c // 4) * 512 + (r % 32) * 16 + ((r % 128) // 32) * 4 + c % 4


def mma_scale_layout(dense):
    """Dense scale bytes [M][S] or [B][M][S] -> the tile layout (uint8, flat)."""
    d = np.asarray(dense, np.uint8)
    d3 = d if d.ndim == 3 else d[None]
    B, M, S = d3.shape
    out = np.zeros(mma_scale_bytes(B, M, S), np.uint8)
    b, r, c = np.meshgrid(np.arange(B), np.arange(M), np.arange(S), indexing="ij")
    out[mma_scale_offset(M, S, b, r, c)] = d3
    return out


def mma_scale_dense(mma, B, M, S):
    """The tile layout back to dense [B][M][S] scale bytes."""
    m = np.asarray(mma, np.uint8).reshape(-1)
    b, r, c = np.meshgrid(np.arange(B), np.arange(M), np.arange(S), indexing="ij")
    return m[mma_scale_offset(M, S, b, r, c)]
