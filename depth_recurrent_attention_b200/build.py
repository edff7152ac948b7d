"""Build libdreamer.so (the product), libdreamer_inputs.so (seeded input generator) and
libdreamer_testhooks.so (test infrastructure: the product's sources with the timeout-test hook
and a 20 ms device wait limit) for sm_100a with nvcc, in-tree."""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
ROOT = os.path.dirname(HERE)
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "--expt-relaxed-constexpr", "-Xcompiler", "-fPIC",
         "-shared", "-Xptxas", "-v"] if os.environ.get("DREAMER_PTXAS_VERBOSE") else \
        ["-O3", "-lineinfo", "-std=c++17", "--expt-relaxed-constexpr", "-Xcompiler", "-fPIC",
         "-shared"]


def _newer(target, deps):
    if not os.path.exists(target):
        return False
    t = os.path.getmtime(target)
    return all(os.path.getmtime(d) <= t for d in deps)


def _sources(exts=(".cu", ".cuh", ".h")):
    out = [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith(exts)]
    out.append(os.path.join(ROOT, "include", "dreamer.h"))
    return out


def build(force: bool = False, verbose: bool = False) -> list:
    outs = []
    lib = os.path.join(HERE, "libdreamer.so")
    deps = [p for p in _sources() if not p.endswith("inputs_gen.cu")]
    if force or not _newer(lib, deps):
        cmd = ["nvcc", *ARCH, *FLAGS, "-o", lib, os.path.join(CSRC, "dreamer.cu"),
               os.path.join(CSRC, "route_noalloc.cu")]
        if verbose:
            print(" ".join(cmd))
        subprocess.run(cmd, check=True)
    outs.append(lib)
    hooks = os.path.join(HERE, "libdreamer_testhooks.so")
    if force or not _newer(hooks, deps):
        cmd = ["nvcc", *ARCH, *FLAGS, "-DDREAMER_TEST_HOOKS",
               "-DDREAMER_WAIT_LIMIT_NS=20000000ull", "-o", hooks,
               os.path.join(CSRC, "dreamer.cu"), os.path.join(CSRC, "route_noalloc.cu")]
        if verbose:
            print(" ".join(cmd))
        subprocess.run(cmd, check=True)
    outs.append(hooks)
    gen = os.path.join(HERE, "libdreamer_inputs.so")
    src = os.path.join(CSRC, "inputs_gen.cu")
    if force or not _newer(gen, [src]):
        cmd = ["nvcc", *ARCH, *FLAGS, "-Xcompiler", "-fopenmp", "-o", gen, src, "-lgomp"]
        subprocess.run(cmd, check=True)
    outs.append(gen)
    return outs


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True))
