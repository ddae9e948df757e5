"""Build ``liblard.so`` (the C-ABI library) for sm_100a with nvcc.

The library is built in-tree, next to this file, so that it travels with the
repository.  cudart is linked statically: the library needs only the NVIDIA
driver at run time and carries its own runtime state.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
SRC_DIR = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "liblard.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo", "-O3", "-std=c++17",
         "--expt-relaxed-constexpr", "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
         "-shared", "-cudart", "static"]


def sources():
    return [os.path.join(SRC_DIR, f) for f in sorted(os.listdir(SRC_DIR))
            if f.endswith((".cu", ".cuh"))] + [os.path.join(ROOT, "include", "lard.h")]


def source_digest() -> str:
    """Short hash of the device code (the kernel headers, which also fix the
    kernels' thread counts and shared-memory layouts): identifies the kernels
    that a profile was taken of.  Host-side argument checks and the C ABI
    wrappers in lard.cu do not enter it."""
    import hashlib
    h = hashlib.sha256()
    for path in sources():
        if not path.endswith(".cuh"):
            continue
        with open(path, "rb") as f:
            h.update(os.path.basename(path).encode() + b"\0" + f.read())
    return h.hexdigest()[:16]


def build(force: bool = False, verbose_ptxas: bool = False) -> str:
    if (not force and os.path.exists(LIB)
            and os.path.getmtime(LIB) >= max(os.path.getmtime(s) for s in sources())):
        return LIB
    cmd = [NVCC] + FLAGS + ["-I", os.path.join(ROOT, "include"), "-I", SRC_DIR]
    if verbose_ptxas:
        cmd += ["-Xptxas", "-v"]
    cmd += ["-o", LIB + ".tmp", os.path.join(SRC_DIR, "lard.cu")]
    subprocess.run(cmd, check=True)
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose_ptxas="-v" in sys.argv))
