"""Build libep.so (the C-ABI CUDA library) in-tree for sm_100a with nvcc.

    python -m combine_ep_layout_12_b200.build [--force] [--verbose-ptxas]

Also builds libep_checked.so: the same sources with -DEP_CHECKED, in which every
row or offset a kernel computes is tested against its array's extent before the
access (EP_ERRBIT_CHECKED in the error word).  The tests run the GPU parity cases
against it as well; the benchmark uses libep.so.

No fast-math: IEEE division, denormals kept, and every rounding the results
depend on is written with explicit _rn intrinsics in the kernels.  The CUDA
runtime is linked statically, so the library needs only the driver at run time.
"""
import glob
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libep.so")
LIB_CHECKED = os.path.join(PKG, "libep_checked.so")

NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-std=c++17", "-O3", "-lineinfo", "-Xcompiler", "-fPIC,-fvisibility=hidden",
         "-shared", "-cudart", "static", "--expt-relaxed-constexpr"]


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cpp")))


def _deps():
    return sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + [os.path.join(INCLUDE, "ep.h")]


def up_to_date(out=LIB):
    if not os.path.exists(out):
        return False
    t = os.path.getmtime(out)
    return all(os.path.getmtime(p) <= t for p in _deps())


def build(force=False, verbose_ptxas=False, quiet=True, out=LIB, extra=()):
    if not force and up_to_date(out):
        return out
    tmp = out + ".tmp%d" % os.getpid()
    cmd = [NVCC, *ARCH, *FLAGS, "-I", INCLUDE, "-I", CSRC, *extra]
    if verbose_ptxas:
        cmd += ["-Xptxas", "-v"]
    cmd += [*sources(), "-o", tmp]
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError("libep build failed:\n%s\n%s%s" % (" ".join(cmd), res.stdout, res.stderr))
    os.replace(tmp, out)
    if not quiet or verbose_ptxas:
        print(" ".join(cmd))
        if res.stderr:
            print(res.stderr)
    return out


def build_checked(force=False, quiet=True):
    return build(force=force, quiet=quiet, out=LIB_CHECKED, extra=("-DEP_CHECKED",))


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose_ptxas="--verbose-ptxas" in sys.argv, quiet=False)
    build_checked(force="--force" in sys.argv, quiet=False)
