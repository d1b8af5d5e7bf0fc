"""Build libpagedkv.so for sm_100a, in the package directory.

    python -m paged_kv_cache_440_b200.build [--force]

Extra nvcc flags (for example -lineinfo variants or -Xptxas options) come
from the environment variable PAGEDKV_NVCC_FLAGS; pass --force after changing
them.

Each source under csrc/ is compiled by nvcc to an object in _build/ (rebuilt
only when it or a header is newer), then linked with the static CUDA runtime
into paged_kv_cache_440_b200/libpagedkv.so. No GPU is needed to build.
"""
import argparse
import concurrent.futures
import glob
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD = os.path.join(ROOT, "_build")
LIB = os.path.join(PKG, "libpagedkv.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
# No fast-math and no flush-to-zero: the quantizer's fp32 divisions and
# rounding must be IEEE-exact to reproduce bit for bit.
NVCC_FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC,-O2",
              "--expt-relaxed-constexpr", "-Xptxas", "-v"]


def _nvcc():
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cpp")))


def _headers():
    return glob.glob(os.path.join(CSRC, "*.h")) + glob.glob(os.path.join(CSRC, "*.cuh")) + \
        glob.glob(os.path.join(INCLUDE, "*.h"))


def _compile(src, obj, extra, verbose_log):
    cmd = [_nvcc()] + ARCH + NVCC_FLAGS + extra + ["-I", INCLUDE, "-I", CSRC,
                                                   "-c", src, "-o", obj]
    r = subprocess.run(cmd, capture_output=True, text=True)
    with open(verbose_log, "w") as f:
        f.write(" ".join(cmd) + "\n" + r.stdout + r.stderr)
    if r.returncode != 0:
        raise RuntimeError("nvcc failed for %s:\n%s" % (src, r.stderr[-6000:]))
    return obj


def build(force=False, jobs=None):
    os.makedirs(BUILD, exist_ok=True)
    extra = os.environ.get("PAGEDKV_NVCC_FLAGS", "").split()
    newest_header = max((os.path.getmtime(h) for h in _headers()), default=0)
    todo, objs = [], []
    for src in _sources():
        obj = os.path.join(BUILD, os.path.basename(src) + ".o")
        objs.append(obj)
        stale = (force or not os.path.exists(obj)
                 or os.path.getmtime(obj) < max(os.path.getmtime(src), newest_header))
        if stale:
            todo.append((src, obj))
    if todo:
        with concurrent.futures.ThreadPoolExecutor(max_workers=jobs or os.cpu_count()) as ex:
            futs = [ex.submit(_compile, s, o, extra, o + ".log") for s, o in todo]
            for f in futs:
                f.result()
    if todo or not os.path.exists(LIB):
        cmd = [_nvcc()] + ARCH + ["-shared", "-Xcompiler", "-fPIC", "-cudart", "static",
                                  "-o", LIB] + objs + ["-lpthread", "-ldl", "-lrt"]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError("link failed:\n" + r.stderr[-4000:])
    return LIB


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    a = ap.parse_args()
    print(build(force=a.force))
    sys.exit(0)
