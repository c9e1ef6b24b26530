"""Build libpwq.so (the CUDA library behind include/pwq.h) in-tree for sm_100a.

Exact-math flags: no --use_fast_math; -ftz=false -prec-div=true
-prec-sqrt=true -fmad=false, so every binary32 operation the kernels write
is one IEEE round-to-nearest operation and fused multiply-adds appear only
where the source asks for them explicitly.  The CUDA runtime is linked
statically, so the library depends on nothing but the driver at run time.
"""
import concurrent.futures
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD = os.path.join(ROOT, "_build")
LIB = os.path.join(PKG, "libpwq.so")
SOURCES = ["pwq_api.cu", "fp8_block.cu", "mxfp8.cu", "nvfp4.cu", "requant.cu", "observer.cu", "selftest.cu",
           "scale_layout.cu"]
HEADERS = ["pwq_device.cuh", "pwq_internal.h"]

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
EXACT = ["-ftz=false", "-prec-div=true", "-prec-sqrt=true", "-fmad=false"]
NVCC_FLAGS = ARCH + EXACT + ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC",
                             "-Xptxas", "-warn-spills", "-I", INCLUDE, "-I", CSRC]


def nvcc():
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if cand and (os.path.isabs(cand) and os.path.exists(cand) or not os.path.isabs(cand)):
            return cand
    return "nvcc"


def _stale(out, deps):
    if not os.path.exists(out):
        return True
    t = os.path.getmtime(out)
    return any(os.path.getmtime(d) > t for d in deps)


def build(force=False, verbose=False):
    os.makedirs(BUILD, exist_ok=True)
    flags_desc = " ".join(EXACT) + " -O3; no --use_fast_math"
    define = ['-DPWQ_BUILD_FLAGS="%s"' % flags_desc]
    hdrs = [os.path.join(CSRC, h) for h in HEADERS] + [os.path.join(INCLUDE, "pwq.h"),
                                                        os.path.abspath(__file__)]
    objs, jobs = [], []
    for src in SOURCES:
        s = os.path.join(CSRC, src)
        o = os.path.join(BUILD, src + ".o")
        objs.append(o)
        if force or _stale(o, [s] + hdrs):
            jobs.append([nvcc(), *NVCC_FLAGS, *define, "-c", s, "-o", o])
    with concurrent.futures.ThreadPoolExecutor(max_workers=len(SOURCES)) as ex:
        for cmd, res in zip(jobs, ex.map(lambda c: subprocess.run(c, capture_output=True, text=True), jobs)):
            if verbose or res.returncode != 0:
                sys.stderr.write(res.stdout + res.stderr)
            if res.returncode != 0:
                raise RuntimeError("nvcc failed: " + " ".join(cmd))
    if force or jobs or _stale(LIB, objs):
        tmp = LIB + ".tmp%d" % os.getpid()
        cmd = [nvcc(), *ARCH, "-shared", "-cudart", "static", "-Xlinker", "--no-undefined", "-o", tmp, *objs]
        res = subprocess.run(cmd, capture_output=True, text=True)
        if res.returncode != 0:
            sys.stderr.write(res.stdout + res.stderr)
            raise RuntimeError("link failed: " + " ".join(cmd))
        os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
