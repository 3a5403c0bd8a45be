"""Builds libjamba.so (sm_100a) in-tree from csrc/*.cu with nvcc, and with
--checked the checked build libjamba_checked.so (-DJAMBA_CHECKS: device-side
checks of indices read from device data, reported as JAMBA_ERR_BOUNDS).

Usage: python -m mamba_selective_scan_mixer_b200.build [--force] [--verbose] [--checked]
"""
import concurrent.futures as cf
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
BUILD = os.path.join(HERE, "_build")
LIB = os.path.join(HERE, "libjamba.so")
BUILD_CHECKED = os.path.join(HERE, "_build_checked")
LIB_CHECKED = os.path.join(HERE, "libjamba_checked.so")

NVCC = os.environ.get("NVCC", "nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "--expt-relaxed-constexpr",
         "-I" + os.path.join(ROOT, "include")]


def _sources():
    return sorted(f for f in os.listdir(CSRC) if f.endswith(".cu"))


def _deps():
    hdrs = [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".cuh", ".hpp"))]
    hdrs.append(os.path.join(ROOT, "include", "jamba.h"))
    return max(os.path.getmtime(h) for h in hdrs)


def _compile(src, verbose, build_dir, extra):
    obj = os.path.join(build_dir, src[:-3] + ".o")
    cmd = [NVCC] + ARCH + FLAGS + extra + (["-Xptxas", "-v"] if verbose else []) + \
        ["-c", os.path.join(CSRC, src), "-o", obj]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError("nvcc failed for %s:\n%s%s" % (src, r.stdout, r.stderr))
    return obj, r.stderr


def build(force=False, verbose=False, checked=False):
    build_dir, lib = (BUILD_CHECKED, LIB_CHECKED) if checked else (BUILD, LIB)
    extra = ["-DJAMBA_CHECKS"] if checked else []
    os.makedirs(build_dir, exist_ok=True)
    srcs = _sources()
    newest = max([_deps()] + [os.path.getmtime(os.path.join(CSRC, s)) for s in srcs] +
                 [os.path.getmtime(os.path.abspath(__file__))])
    if not force and os.path.exists(lib) and os.path.getmtime(lib) >= newest:
        return lib
    with cf.ThreadPoolExecutor(max_workers=min(8, len(srcs))) as ex:
        results = list(ex.map(lambda s: _compile(s, verbose, build_dir, extra), srcs))
    if verbose:
        for _, log in results:
            sys.stderr.write(log)
    tmp = lib + ".tmp%d" % os.getpid()
    cmd = [NVCC] + ARCH + ["-shared", "-o", tmp] + [o for o, _ in results]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError("link failed:\n" + r.stdout + r.stderr)
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="--verbose" in sys.argv, checked="--checked" in sys.argv))
