"""Build libcsla.so (sm_100a) in-tree with nvcc.

    python compressed_sparse_long_append_b200/build.py [--force] [--ptxas-v]
    python compressed_sparse_long_append_b200/build.py --timeline OUT.so

The second form builds a separate library with the device timeline hooks
compiled in (-DCSLA_TIMELINE, csla_timeline_read/clear exported).

The library has no torch dependency: it is plain CUDA C++ behind the C ABI
of include/csla.h.  Kernels are compiled for sm_100a only.
"""
import glob
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
LIB = os.path.join(PKG, "libcsla.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17", "-rdc=true",
    "-Xcompiler", "-fPIC", "-Xcompiler", "-O2",
    "--expt-relaxed-constexpr",
    "-I" + os.path.join(ROOT, "include"),
]


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _stale():
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    deps = sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h")) \
        + [os.path.join(ROOT, "include", "csla.h")]
    return any(os.path.getmtime(p) > t for p in deps)


def build(force=False, verbose=False, extra=()):
    if not force and not _stale():
        return LIB
    tmp = LIB + ".tmp%d" % os.getpid()
    cmd = [NVCC, *FLAGS, *extra, "-shared", "-o", tmp, *sources()]
    if verbose:
        print(" ".join(cmd))
    subprocess.run(cmd, check=True)
    os.replace(tmp, LIB)
    return LIB


def build_timeline(out):
    cmd = [NVCC, *FLAGS, "-DCSLA_TIMELINE", "-shared", "-o", out, *sources()]
    subprocess.run(cmd, check=True)
    return out


if __name__ == "__main__":
    if "--timeline" in sys.argv:
        print(build_timeline(os.path.abspath(sys.argv[sys.argv.index("--timeline") + 1])))
        sys.exit(0)
    extra = ["-Xptxas", "-v"] if "--ptxas-v" in sys.argv else []
    print(build(force="--force" in sys.argv or bool(extra), verbose=True, extra=extra))
