"""Builds libkvrq.so in-tree with nvcc for sm_100a.

Each translation unit is compiled to an object in parallel, then linked into
one shared library next to this file. The CUDA runtime is linked statically,
so the library needs only the NVIDIA driver at run time.
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
LIB = os.path.join(PKG, "libkvrq.so")

SOURCES = ["setup.cpp", "pages.cpp", "params.cpp", "api.cu", "rq_kernels.cu", "tq_kernels.cu", "tqg_kernels.cu",
           "score_kernels.cu", "attn_kernels.cu", "attn_tc_kernels.cu", "pq_kernels.cu"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
COMMON = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "-I" + INCLUDE, "-I" + CSRC]


def nvcc():
    home = os.environ.get("CUDA_HOME", "/usr/local/cuda")
    exe = os.path.join(home, "bin", "nvcc")
    return exe if os.path.exists(exe) else "nvcc"


def _obj(src):
    return os.path.join(BUILD, src.replace("/", "_") + ".o")


def _compile(src, extra):
    out = _obj(src)
    cmd = [nvcc()] + ARCH + COMMON + extra + ["-c", os.path.join(CSRC, src), "-o", out]
    r = subprocess.run(cmd, capture_output=True, text=True)
    return src, r.returncode, r.stdout + r.stderr, cmd


def _stale(src):
    out = _obj(src)
    if not os.path.exists(out):
        return True
    t = os.path.getmtime(out)
    deps = [os.path.join(CSRC, f) for f in os.listdir(CSRC)] + [os.path.join(INCLUDE, f) for f in os.listdir(INCLUDE)]
    deps.append(os.path.abspath(__file__))
    return any(os.path.getmtime(p) > t for p in deps)


def build(verbose=False, ptxas_info=False, force=False):
    """Compile and link libkvrq.so; returns its path. Raises on failure."""
    os.makedirs(BUILD, exist_ok=True)
    extra = ["-Xptxas", "-v"] if ptxas_info else []
    todo = [s for s in SOURCES if force or ptxas_info or _stale(s)]
    with concurrent.futures.ThreadPoolExecutor(max_workers=min(8, len(todo) or 1)) as ex:
        for src, rc, log, cmd in ex.map(lambda s: _compile(s, extra), todo):
            if verbose or rc != 0 or ptxas_info:
                sys.stderr.write("== %s\n%s\n" % (src, log))
            if rc != 0:
                raise RuntimeError("nvcc failed for %s:\n%s\n%s" % (src, " ".join(cmd), log))
    if todo or not os.path.exists(LIB):
        cmd = [nvcc()] + ARCH + ["-shared", "-cudart", "static", "-o", LIB] + [_obj(s) for s in SOURCES] + ["-lpthread"]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError("link failed:\n%s\n%s" % (" ".join(cmd), r.stdout + r.stderr))
    return LIB


if __name__ == "__main__":
    print(build(verbose=True, ptxas_info="--ptxas" in sys.argv, force="--force" in sys.argv))
