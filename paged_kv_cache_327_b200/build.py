"""Build libpa.so (the C ABI of include/pa.h) for sm_100a with nvcc, in-tree.

The CUDA runtime is linked statically, so the library loads on a machine without a GPU
(for symbol checks); the driver's tensor-map encoder is looked up at run time.

Several processes may build at once (one per GPU rank): they take turns under an exclusive
file lock beside the library, the freshness check is repeated under the lock (so only the
first one compiles), and each compiles into a temporary file of its own that is renamed over
the library in one step.
"""
import fcntl
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
LIB = os.path.join(PKG, "libpa.so")
SOURCES = [os.path.join(CSRC, "pa_api.cu")]
DEPENDS = SOURCES + [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith(".cuh")] + \
    [os.path.join(ROOT, "include", "pa.h")]

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17", "--expt-relaxed-constexpr",
    "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
    "-shared", "-cudart", "static",
]


def nvcc():
    cuda = os.environ.get("CUDA_HOME", "/usr/local/cuda")
    path = os.path.join(cuda, "bin", "nvcc")
    return path if os.path.exists(path) else "nvcc"


def _fresh(lib: str) -> bool:
    if not os.path.exists(lib):
        return False
    mtime = os.path.getmtime(lib)
    return all(os.path.getmtime(f) <= mtime for f in DEPENDS)


def build(force: bool = False, verbose: bool = False, extra=(), lib: str = LIB) -> str:
    """Compile `lib` (default: the in-tree libpa.so) unless it is newer than every source."""
    if not force and _fresh(lib):
        return lib
    with open(lib + ".lock", "w") as lock:
        fcntl.flock(lock, fcntl.LOCK_EX)  # released when the file closes
        if not force and _fresh(lib):      # another process built it while this one waited
            return lib
        tmp = f"{lib}.{os.getpid()}.tmp"
        cmd = [nvcc(), *NVCC_FLAGS, *extra, "-I", os.path.join(ROOT, "include"), "-I", CSRC,
               *SOURCES, "-o", tmp]
        if verbose:
            cmd.insert(1, "-Xptxas=-v")
        try:
            subprocess.run(cmd, check=True)
            os.replace(tmp, lib)
        finally:
            if os.path.exists(tmp):
                os.unlink(tmp)
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
