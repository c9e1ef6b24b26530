"""Guard bytes around every GPU output of the parity tests (tests only).

compute-sanitizer is not available to these tests, so out-of-bounds writes
are caught the plain way: every output buffer lives inside a larger device
allocation filled with a sentinel byte, and after the test every byte
outside the output's view must still hold the sentinel.  A guarded buffer
has
  - a head of HEAD bytes before the first element (the view's base stays
    aligned to 512 bytes plus the requested lead),
  - optional gaps before and after each row (lead / pad elements), which
    give strided outputs the row padding the tests need, and
  - a tail of TAIL bytes after the last row, so a vector store or a scale
    write one element past a dense array is seen.

Two ways in:
  - ``empty(shape, dtype, lead=0, pad=0)`` for outputs a test passes with
    ``out=`` (padded or offset views included);
  - ``binding_allocations()`` swaps the ``torch`` name inside the Python
    binding for a proxy whose ``empty`` / ``empty_like`` return guarded
    buffers, so the outputs and workspace the binding allocates itself are
    guarded too.  The library and the binding are unchanged.
``session()`` collects the buffers made while it is open and checks them all
when it closes (the GPU tests' autouse fixture in conftest.py).
"""
import contextlib
import math

import torch

SENTINEL = 0xA7
HEAD = 512
TAIL = 4096

_SESSIONS = []


class Guarded:
    def __init__(self, shape, dtype, device, lead=0, pad=0):
        shape = tuple(int(d) for d in shape)
        if not shape:
            shape = (1,)
        self.shape, self.dtype, self.lead, self.pad = shape, dtype, int(lead), int(pad)
        self.esz = torch.empty((), dtype=dtype).element_size()
        N = shape[-1]
        self.row_elems = self.lead + N + self.pad
        self.rows = math.prod(shape[:-1])
        self.nbytes = self.rows * self.row_elems * self.esz
        self.raw = torch.full((HEAD + self.nbytes + TAIL,), SENTINEL, dtype=torch.uint8, device=device)
        body = self.raw[HEAD:HEAD + self.nbytes].view(dtype).view(shape[:-1] + (self.row_elems,))
        self.view = body[..., self.lead:self.lead + N]

    def violations(self):
        """Descriptions of the guard regions whose bytes changed."""
        bad = []
        S = SENTINEL
        if not bool((self.raw[:HEAD] == S).all()):
            bad.append("head")
        if not bool((self.raw[HEAD + self.nbytes:] == S).all()):
            n = int((self.raw[HEAD + self.nbytes:] != S).nonzero()[0].item())
            bad.append("tail (first changed byte %d past the end)" % n)
        if (self.lead or self.pad) and self.nbytes:
            rows = self.raw[HEAD:HEAD + self.nbytes].view(self.rows, self.row_elems * self.esz)
            if self.lead and not bool((rows[:, :self.lead * self.esz] == S).all()):
                bad.append("row lead gap")
            if self.pad and not bool((rows[:, (self.lead + self.shape[-1]) * self.esz:] == S).all()):
                bad.append("row pad gap")
        return bad

    def describe(self):
        return "%s %s lead=%d pad=%d" % (self.dtype, self.shape, self.lead, self.pad)


def empty(shape, dtype, device="cuda", lead=0, pad=0):
    """A guarded output: a view of `shape` (rows `lead` elements into a row
    of lead + N + pad) inside a sentinel-filled allocation."""
    g = Guarded(shape, dtype, device, lead, pad)
    if _SESSIONS:
        _SESSIONS[-1].append(g)
    return g.view


def check(guards):
    if torch.cuda.is_available():
        torch.cuda.synchronize()
    problems = []
    for g in guards:
        bad = g.violations()
        if bad:
            problems.append("%s: %s" % (g.describe(), ", ".join(bad)))
    assert not problems, "writes outside output views: " + "; ".join(problems)


@contextlib.contextmanager
def session():
    guards = []
    _SESSIONS.append(guards)
    try:
        yield guards
    finally:
        _SESSIONS.pop()
    check(guards)


def _size(size):
    if len(size) == 1 and not isinstance(size[0], int):
        return tuple(size[0])
    return tuple(size)


def _is_cuda(device):
    return device is not None and torch.device(device).type == "cuda"


class _TorchProxy:
    """torch, except that CUDA `empty` / `empty_like` return guarded buffers."""

    def __getattr__(self, name):
        return getattr(torch, name)

    def empty(self, *size, dtype=None, device=None, **kw):
        if _is_cuda(device) and not kw:
            return empty(_size(size), dtype or torch.get_default_dtype(), device)
        return torch.empty(*size, dtype=dtype, device=device, **kw)

    def empty_like(self, x, dtype=None, **kw):
        if x.is_cuda and not kw:
            return empty(x.shape, dtype or x.dtype, x.device)
        return torch.empty_like(x, dtype=dtype, **kw)


@contextlib.contextmanager
def binding_allocations():
    """While open, the binding's own CUDA allocations are guarded buffers."""
    import precision_weight_quantization_b200 as P
    saved = P.torch
    P.torch = _TorchProxy()
    try:
        yield
    finally:
        P.torch = saved
