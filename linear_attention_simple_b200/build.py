"""Build libgla.so in-tree for sm_100a (nvcc; no JIT cache, no pip install).

Each ``csrc/*.cu`` file is compiled separately (in parallel) with
``-gencode arch=compute_100a,code=sm_100a -lineinfo -O3`` and linked, with
the static CUDA runtime, into ``linear_attention_simple_b200/libgla.so``.
The driver library is not linked: ``cuTensorMapEncodeTiled`` is fetched at
run time through ``cudaGetDriverEntryPoint``, so the library loads on hosts
without a GPU.

``build(debug=True)`` makes the checking build ``libgla_debug.so`` from the
same sources with ``-DGLA_DEBUG_BOUNDS`` (objects under ``_build/debug``): the
same ABI, plus input scans and index checks that record an error in the
device status word instead of trapping.  The binding loads it instead of
``libgla.so`` when the environment sets ``GLA_DEBUG_BOUNDS=1``.

Several processes may call build() at once (one per rank under torchrun):
an exclusive lock on ``_build/.lock`` serialises them, and every object and
the library are written under a temporary name and renamed into place.
"""
import concurrent.futures
import fcntl
import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
ROOT = os.path.dirname(HERE)
BUILD = os.path.join(ROOT, "_build")
LIB = os.path.join(HERE, "libgla.so")
LIB_DEBUG = os.path.join(HERE, "libgla_debug.so")
DEBUG_FLAGS = ["-DGLA_DEBUG_BOUNDS"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-Xcompiler", "-Wall",
         "--expt-relaxed-constexpr", "-I" + os.path.join(ROOT, "include"), "-I" + CSRC]


def nvcc():
    exe = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    return exe


def sources():
    return sorted(os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith(".cu"))


def _headers_mtime():
    hs = [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".cuh", ".h"))]
    hs.append(os.path.join(ROOT, "include", "gla.h"))
    return max(os.path.getmtime(h) for h in hs)


def _compile(src, verbose=False, debug=False):
    out_dir = os.path.join(BUILD, "debug") if debug else BUILD
    obj = os.path.join(out_dir, os.path.basename(src) + ".o")
    if (os.path.exists(obj) and os.path.getmtime(obj) >= os.path.getmtime(src)
            and os.path.getmtime(obj) >= _headers_mtime()):
        return obj
    tmp = obj + ".tmp.%d" % os.getpid()
    cmd = [nvcc()] + ARCH + FLAGS + (DEBUG_FLAGS if debug else []) + (["-Xptxas", "-v"] if verbose else []) + \
        ["-c", src, "-o", tmp]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError("nvcc failed for %s:\n%s\n%s" % (src, r.stdout, r.stderr))
    os.replace(tmp, obj)
    if verbose:
        sys.stderr.write(r.stderr)
    return obj


def build(verbose=False, force=False, debug=False):
    os.makedirs(os.path.join(BUILD, "debug"), exist_ok=True)
    with open(os.path.join(BUILD, ".lock"), "w") as lock:
        fcntl.flock(lock, fcntl.LOCK_EX)
        return _build_locked(verbose, force, debug)


def _build_locked(verbose, force, debug):
    out_dir = os.path.join(BUILD, "debug") if debug else BUILD
    lib = LIB_DEBUG if debug else LIB
    if force:
        for f in os.listdir(out_dir):
            if f.endswith(".o"):
                os.remove(os.path.join(out_dir, f))
    srcs = sources()
    with concurrent.futures.ThreadPoolExecutor(max_workers=min(8, len(srcs))) as ex:
        objs = list(ex.map(lambda s: _compile(s, verbose, debug), srcs))
    if os.path.exists(lib) and all(os.path.getmtime(lib) >= os.path.getmtime(o) for o in objs):
        return lib
    tmp = lib + ".tmp.%d" % os.getpid()
    cmd = [nvcc()] + ARCH + ["-shared", "-Xcompiler", "-fPIC", "-cudart", "static", "-o", tmp] + objs
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError("link failed:\n%s\n%s" % (r.stdout, r.stderr))
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    print(build(verbose="-v" in sys.argv, force="--force" in sys.argv, debug="--debug" in sys.argv))
