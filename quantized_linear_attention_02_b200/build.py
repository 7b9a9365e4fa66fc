"""Build step of the CUDA library: compiles csrc/ into libstq.so in this directory
(sm_100a, in-tree, so the built library travels with the source tree)."""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
LIB = os.path.join(HERE, "libstq.so")
SOURCES = ["csrc/stq_abi.cpp", "csrc/stq_kernels.cu", "csrc/stq_absmax.cu", "csrc/stq_calib.cu",
           "csrc/stq_static_staging.cu", "csrc/stq_pipeline.cpp", "csrc/stq_probe.cu"]
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-lineinfo", "-O3", "-std=c++17",
    "--fmad=false",                 # products are rounded before they are added
    "-Xcompiler", "-fPIC,-O2,-Wall,-ffp-contract=off",   # host double sums: no fused multiply-add
    "-shared",
]


LIB_CHECKED = os.path.join(HERE, "libstq_checked.so")


def needs_build(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    deps = [os.path.join(HERE, s) for s in SOURCES]
    deps += [os.path.join(HERE, "csrc", h) for h in ("stq_internal.h", "stq_device.cuh")]
    deps += [os.path.join(ROOT, "include", "stq.h")]
    return any(os.path.getmtime(p) > t for p in deps)


def build(force: bool = False, verbose: bool = False, extra=None, checked: bool = False) -> str:
    """Compile libstq.so; checked=True compiles libstq_checked.so with STQ_CHECKS (device
    checks that record stored codes 0 and non-finite states in the pool's error word)."""
    lib = LIB_CHECKED if checked else LIB
    if not force and not needs_build(lib):
        return lib
    cmd = [NVCC] + FLAGS + (["-DSTQ_CHECKS"] if checked else []) + (extra or [])
    cmd += ["-I", os.path.join(ROOT, "include"), "-I", os.path.join(HERE, "csrc"), "-o", lib + ".tmp"]
    cmd += [os.path.join(HERE, s) for s in SOURCES]
    if verbose:
        print(" ".join(cmd), file=sys.stderr)
    subprocess.run(cmd, check=True)
    os.replace(lib + ".tmp", lib)
    return lib


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose=True, checked="--checked" in sys.argv,
          extra=["-Xptxas", "-v"] if "--ptxas-v" in sys.argv else None)
