"""Multi-threaded driver of the scalar C oracle (test infrastructure only).

The arithmetic is exactly that of ``pwq_oracle.c``: this module only splits
a tensor into row ranges and calls the same C entry points on them from a
pool of host threads (ctypes releases the interpreter lock for the length
of each foreign call, so the pieces run in parallel).  Splits never cut a
unit of the formats: FP8 block-wise pieces are bands of whole 128-row tile
rows of one batch matrix; MXFP8 and NVFP4 pieces are whole rows; the NVFP4
group amax is the maximum of the pieces' maxima (max is exact and
order-free).  Results are therefore identical to the single-threaded
oracle's, which ``tests/test_oracle_parallel.py`` checks.

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may use it.
"""
import concurrent.futures
import ctypes
import os

import numpy as np

from . import oracle as O


def host_threads() -> int:
    """Threads this process may run on (its CPU affinity mask)."""
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


_POOLS = {}


def _pool(threads):
    if threads not in _POOLS:
        _POOLS[threads] = concurrent.futures.ThreadPoolExecutor(max_workers=threads)
    return _POOLS[threads]


def _run(threads, tasks):
    """Run the zero-argument callables in `tasks` on `threads` threads."""
    lib = O.lib()
    lib.or_e4m3_encode(0.0)      # fills the E4M3 value table before any worker reads it
    if threads <= 1 or len(tasks) <= 1:
        return [t() for t in tasks]
    return list(_pool(threads).map(lambda t: t(), tasks))


def _ptr(a, byte_offset=0):
    return ctypes.c_void_p(a.ctypes.data + int(byte_offset))


def _ranges(n, parts):
    """n items cut into at most `parts` contiguous ranges of nearly equal size."""
    parts = max(1, min(parts, n))
    step = -(-n // parts)
    return [(i, min(i + step, n)) for i in range(0, n, step)]


def _bmn(x):
    return (1,) + tuple(x.shape) if x.ndim == 2 else tuple(x.shape)


# ---------------------------------------------------------------- FP8 block-wise

def _tile_bands(B, M, threads):
    """(b, r0, r1) bands of whole 128-row tile rows, about 4 per thread."""
    TM = -(-M // 128)
    bands = []
    per = max(1, -(-(B * TM) // (4 * threads)))
    for b in range(B):
        for t0, t1 in _ranges(TM, -(-TM // per)):
            bands.append((b, t0 * 128, min(t1 * 128, M)))
    return bands


def fp8_block_quant(x_bits, threads=None):
    threads = threads or host_threads()
    x = np.ascontiguousarray(x_bits, np.uint16)
    B, M, N = _bmn(x)
    TM, TN = -(-M // 128), -(-N // 128)
    q = np.empty(x.shape, np.uint8)
    s = np.empty((B, TM, TN), np.float32)
    lib = O.lib()
    tasks = []
    for b, r0, r1 in _tile_bands(B, M, threads):
        xo, so = (b * M + r0) * N, (b * TM + r0 // 128) * TN
        tasks.append(lambda xo=xo, so=so, m=r1 - r0: lib.or_fp8_block_quant(
            _ptr(x, 2 * xo), 1, m, N, _ptr(q, xo), _ptr(s, 4 * so)))
    if x.size:
        _run(threads, tasks)
    return q, (s[0] if x.ndim == 2 else s)


def fp8_block_dequant(q, s, threads=None):
    threads = threads or host_threads()
    q = np.ascontiguousarray(q, np.uint8)
    s = np.ascontiguousarray(s, np.float32)
    B, M, N = _bmn(q)
    TM, TN = -(-M // 128), -(-N // 128)
    y = np.empty(q.shape, np.uint16)
    lib = O.lib()
    tasks = []
    for b, r0, r1 in _tile_bands(B, M, threads):
        qo, so = (b * M + r0) * N, (b * TM + r0 // 128) * TN
        tasks.append(lambda qo=qo, so=so, m=r1 - r0: lib.or_fp8_block_dequant(
            _ptr(q, qo), _ptr(s, 4 * so), 1, m, N, _ptr(y, 2 * qo)))
    if q.size:
        _run(threads, tasks)
    return y


# ---------------------------------------------------------------- row-wise formats

def _row_tasks(rows, threads, make):
    return [make(r0, r1) for r0, r1 in _ranges(rows, 4 * threads)]


def mxfp8_quant(x_bits, threads=None):
    threads = threads or host_threads()
    x = np.ascontiguousarray(x_bits, np.uint16)
    N = x.shape[-1]
    assert N % 32 == 0
    R = x.size // N if N else 0
    q = np.empty(x.shape, np.uint8)
    e = np.empty(x.shape[:-1] + (N // 32,), np.uint8)
    lib = O.lib()
    if x.size:
        _run(threads, _row_tasks(R, threads, lambda r0, r1: lambda: lib.or_mxfp8_quant(
            _ptr(x, 2 * r0 * N), 1, r1 - r0, N, _ptr(q, r0 * N), _ptr(e, r0 * (N // 32)))))
    return q, e


def mxfp8_dequant(q, e, threads=None):
    threads = threads or host_threads()
    q = np.ascontiguousarray(q, np.uint8)
    e = np.ascontiguousarray(e, np.uint8)
    N = q.shape[-1]
    R = q.size // N if N else 0
    y = np.empty(q.shape, np.uint16)
    lib = O.lib()
    if q.size:
        _run(threads, _row_tasks(R, threads, lambda r0, r1: lambda: lib.or_mxfp8_dequant(
            _ptr(q, r0 * N), _ptr(e, r0 * (N // 32)), 1, r1 - r0, N, _ptr(y, 2 * r0 * N))))
    return y


def amax_bf16(x_bits, threads=None):
    threads = threads or host_threads()
    x = np.ascontiguousarray(x_bits, np.uint16).reshape(-1)
    lib = O.lib()
    parts = _run(threads, [lambda a=a, b=b: float(np.float32(lib.or_amax_bf16(_ptr(x, 2 * a), b - a)))
                           for a, b in _ranges(x.size, 4 * threads)] if x.size else [])
    return float(np.float32(max(parts + [0.0])))


def nvfp4_group_amax(members, threads=None):
    return float(np.float32(max([amax_bf16(m, threads) for m in members] + [0.0])))


def nvfp4_quant(x_bits, group_amax, threads=None):
    threads = threads or host_threads()
    x = np.ascontiguousarray(x_bits, np.uint16)
    N = x.shape[-1]
    assert N % 16 == 0
    R = x.size // N if N else 0
    packed = np.empty(x.shape[:-1] + (N // 2,), np.uint8)
    sb = np.empty(x.shape[:-1] + (N // 16,), np.uint8)
    lib = O.lib()
    A = np.float32(group_amax)
    if x.size:
        _run(threads, _row_tasks(R, threads, lambda r0, r1: lambda: lib.or_nvfp4_quant(
            _ptr(x, 2 * r0 * N), r1 - r0, N, A, _ptr(packed, r0 * (N // 2)), _ptr(sb, r0 * (N // 16)))))
    return packed, sb, O.nvfp4_global_scale(group_amax)


def nvfp4_dequant(packed, sb, gs, N, threads=None):
    threads = threads or host_threads()
    packed = np.ascontiguousarray(packed, np.uint8)
    sb = np.ascontiguousarray(sb, np.uint8)
    R = packed.size // (N // 2) if N else 0
    y = np.empty(packed.shape[:-1] + (N,), np.uint16)
    lib = O.lib()
    g = np.float32(gs)
    if y.size:
        _run(threads, _row_tasks(R, threads, lambda r0, r1: lambda: lib.or_nvfp4_dequant(
            _ptr(packed, r0 * (N // 2)), _ptr(sb, r0 * (N // 16)), g, r1 - r0, N, _ptr(y, 2 * r0 * N))))
    return y


def nvfp4_fake_quant(x_bits, group_amax, threads=None):
    threads = threads or host_threads()
    x = np.ascontiguousarray(x_bits, np.uint16)
    N = x.shape[-1]
    R = x.size // N if N else 0
    y = np.empty(x.shape, np.uint16)
    lib = O.lib()
    A = np.float32(group_amax)
    if x.size:
        _run(threads, _row_tasks(R, threads, lambda r0, r1: lambda: lib.or_nvfp4_fake_quant(
            _ptr(x, 2 * r0 * N), r1 - r0, N, A, _ptr(y, 2 * r0 * N))))
    return y
