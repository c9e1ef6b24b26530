"""Static checks on the CUDA sources (no GPU): device code never traps, and
every spin-wait on memory that another thread or CTA releases is bounded
by a time limit after which the kernel records an error and goes on.

  - no __trap, device assert or breakpoint anywhere in csrc/;
  - the mbarrier try-wait is called only by the bounded wait helper;
  - every loop that spins on an acquire load reads the global timer
    within its body.
"""
import os
import re

CSRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                    "precision_weight_quantization_b200", "csrc")


def sources():
    out = {}
    for name in sorted(os.listdir(CSRC)):
        if name.endswith((".cu", ".cuh", ".h")):
            with open(os.path.join(CSRC, name)) as f:
                out[name] = f.read()
    return out


def strip_comments(text):
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return re.sub(r"//[^\n]*", "", text)


def test_device_code_never_traps():
    for name, text in sources().items():
        code = strip_comments(text)
        for pat in (r"\b__trap\s*\(", r"\bassert\s*\(", r"\bbrkpt\b", r'"\s*trap\s*;'):
            assert not re.search(pat, code), (name, pat)


def test_mbarrier_waits_go_through_the_bounded_helper():
    calls = []
    for name, text in sources().items():
        code = strip_comments(text)
        for m in re.finditer(r"\bmbar_try_wait\s*\(", code):
            calls.append((name, code.count("\n", 0, m.start()) + 1))
    # the definition and the calls inside mbar_wait_bounded, all in one header
    assert calls and {n for n, _ in calls} == {"pwq_device.cuh"}, calls
    text = strip_comments(sources()["pwq_device.cuh"])
    body = text[text.index("mbar_wait_bounded("):]
    body = body[:body.index("\n}\n")]
    assert "globaltimer" in body or "clock" in body, "the bounded wait must read a timer"
    assert len(calls) == 1 + body.count("mbar_try_wait("), calls


def test_acquire_spin_loops_read_the_timer():
    loops = 0
    for name, text in sources().items():
        code = strip_comments(text)
        for m in re.finditer(r"while\s*\(\s*ld_acquire_gpu\s*\(", code):
            loops += 1
            body = code[m.end():]
            body = body[:body.index("}")]
            assert "globaltimer_ns" in body and "break" in body, (name, body[:200])
    assert loops >= 1
