"""Build liblrs.so (the CUDA library behind include/lrs.h) in-tree for sm_100a.

Each csrc/*.cu is compiled to an object under _build/ (in parallel), then the
objects are linked into quantized_recurrent_state_decode_b200/liblrs.so with
the CUDA runtime linked statically. Rebuilds only what changed.

    python -m quantized_recurrent_state_decode_b200.build [--force] [-v]
"""
import concurrent.futures as cf
import glob
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD = os.path.join(ROOT, "_build", "liblrs")
LIB = os.path.join(PKG, "liblrs.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
# -fmad=false: no implicit multiply-add contraction; every fused operation in
# the kernels is an explicit __fmaf_rn, so results are bit-reproducible.
NVCC_FLAGS = ["-std=c++17", "-O3", "-lineinfo", "-fmad=false", "-Xcompiler", "-fPIC",
              "-Xcompiler", "-Wall", "--expt-relaxed-constexpr", "-I", INCLUDE, "-I", CSRC]


def nvcc():
    exe = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(exe):
        raise RuntimeError("nvcc not found: the CUDA toolkit is needed to build liblrs")
    return exe


def _headers():
    return glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h")) + \
        glob.glob(os.path.join(INCLUDE, "*.h"))


def _stale(target, deps):
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(d) > t for d in deps)


def _compile(src, obj, verbose):
    cmd = [nvcc(), *ARCH, *NVCC_FLAGS, "-c", src, "-o", obj + ".tmp"]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError("nvcc failed for %s:\n%s%s" % (src, r.stdout, r.stderr))
    os.replace(obj + ".tmp", obj)
    return r.stderr if verbose else ""


def build(force: bool = False, verbose: bool = False) -> str:
    srcs = sorted(glob.glob(os.path.join(CSRC, "*.cu")))
    hdrs = _headers()
    # a library newer than every source and header is current, whether or not
    # its object files are at hand (a copy of the tree may carry only the .so)
    if not force and not verbose and not _stale(LIB, [*srcs, *hdrs]):
        return LIB
    os.makedirs(BUILD, exist_ok=True)
    jobs = []
    objs = []
    for src in srcs:
        obj = os.path.join(BUILD, os.path.basename(src)[:-3] + ".o")
        objs.append(obj)
        if force or _stale(obj, [src, *hdrs]):
            jobs.append((src, obj))
    if jobs:
        workers = max(1, min(len(jobs), os.cpu_count() or 1))
        with cf.ThreadPoolExecutor(workers) as ex:
            for log in ex.map(lambda j: _compile(*j, verbose), jobs):
                if log:
                    sys.stderr.write(log)
    if force or jobs or _stale(LIB, objs):
        tmp = LIB + ".tmp.%d" % os.getpid()
        cmd = [nvcc(), *ARCH, "-shared", "-o", tmp, *objs, "-cudart", "static"]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError("link of liblrs.so failed:\n%s%s" % (r.stdout, r.stderr))
        os.replace(tmp, LIB)
    return LIB


CHECKED_LIB = os.path.join(PKG, "liblrs_checked.so")
CHECKED_BUILD = os.path.join(ROOT, "_build", "liblrs_checked")
# the translation units of the step kernel and its launchers, which carry the
# bounds checks; the rest are linked from the normal build
CHECKED_UNITS = ["step_rtn.cu", "step_sr.cu", "step_bdr.cu", "step_rtn_bf16.cu",
                 "step_sr_bf16.cu", "step_bdr_bf16.cu", "lrs_api.cu", "lrs_static.cu"]


def build_checked(force: bool = False) -> str:
    """liblrs_checked.so: the library with the step kernel's bounds checks
    (LRS_BOUNDS_CHECK): an index outside its buffer records
    LRS_ERR_DEVICE_BOUNDS and the access is skipped. A debug build for tests."""
    hdrs = _headers()
    if not force and not _stale(CHECKED_LIB, [*glob.glob(os.path.join(CSRC, "*.cu")), *hdrs]):
        return CHECKED_LIB
    build(force=force)
    os.makedirs(CHECKED_BUILD, exist_ok=True)
    jobs, objs = [], []
    for src in sorted(glob.glob(os.path.join(CSRC, "*.cu"))):
        name = os.path.basename(src)
        if name in CHECKED_UNITS:
            obj = os.path.join(CHECKED_BUILD, name[:-3] + ".o")
            if force or _stale(obj, [src, *hdrs]):
                jobs.append((src, obj))
        else:
            obj = os.path.join(BUILD, name[:-3] + ".o")
        objs.append(obj)
    if jobs:
        def one(j):
            src, obj = j
            cmd = [nvcc(), *ARCH, *NVCC_FLAGS, "-DLRS_BOUNDS_CHECK", "-c", src, "-o", obj + ".tmp"]
            r = subprocess.run(cmd, capture_output=True, text=True)
            if r.returncode != 0:
                raise RuntimeError("nvcc failed for %s:\n%s%s" % (src, r.stdout, r.stderr))
            os.replace(obj + ".tmp", obj)
        with cf.ThreadPoolExecutor(max(1, min(len(jobs), os.cpu_count() or 1))) as ex:
            list(ex.map(one, jobs))
    if force or jobs or _stale(CHECKED_LIB, objs):
        tmp = CHECKED_LIB + ".tmp.%d" % os.getpid()
        r = subprocess.run([nvcc(), *ARCH, "-shared", "-o", tmp, *objs, "-cudart", "static"],
                           capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError("link of liblrs_checked.so failed:\n%s%s" % (r.stdout, r.stderr))
        os.replace(tmp, CHECKED_LIB)
    return CHECKED_LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
    if "--checked" in sys.argv:
        print(build_checked(force="--force" in sys.argv))
