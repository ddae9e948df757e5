"""Build ``liblard.so`` (the C-ABI library) and ``liblard_probe.so`` for sm_100a with nvcc.

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
PROBE_LIB = os.path.join(HERE, "liblard_probe.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo", "-O3", "-std=c++17",
         "--expt-relaxed-constexpr", "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
         "-shared", "-cudart", "static"]

# (library, main source, header) of each build target
TARGETS = {"lard": (LIB, "lard.cu", "lard.h"), "probe": (PROBE_LIB, "lard_probe.cu", "lard_probe.h")}


def sources(target: str = "lard"):
    """The files a target is built from: its main source, every kernel header and its C header."""
    _, main, header = TARGETS[target]
    return ([os.path.join(SRC_DIR, main)] +
            [os.path.join(SRC_DIR, f) for f in sorted(os.listdir(SRC_DIR)) if f.endswith(".cuh")] +
            [os.path.join(ROOT, "include", header)])


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


def build_target(target: str, force: bool = False, verbose_ptxas: bool = False) -> str:
    lib, main, _ = TARGETS[target]
    srcs = sources(target)
    if not force and os.path.exists(lib) and os.path.getmtime(lib) >= max(os.path.getmtime(s) for s in srcs):
        return lib
    cmd = [NVCC] + FLAGS + ["-I", os.path.join(ROOT, "include"), "-I", SRC_DIR]
    if verbose_ptxas:
        cmd += ["-Xptxas", "-v"]
    cmd += ["-o", lib + ".tmp", os.path.join(SRC_DIR, main)]
    subprocess.run(cmd, check=True)
    os.replace(lib + ".tmp", lib)
    return lib


def build(force: bool = False, verbose_ptxas: bool = False) -> str:
    """Build liblard.so (the C-ABI library) and liblard_probe.so (the exponential-unit
    probe the benchmark uses); returns the path of liblard.so."""
    build_target("probe", force, verbose_ptxas)
    return build_target("lard", force, verbose_ptxas)


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose_ptxas="-v" in sys.argv))
