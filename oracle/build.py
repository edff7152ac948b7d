"""Build the CPU oracle (test infrastructure) into oracle/liboracle.so with gcc."""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SO = os.path.join(HERE, "liboracle.so")


def build(force: bool = False) -> str:
    src = os.path.join(HERE, "dreamer_oracle.c")
    hdr = os.path.join(HERE, "dreamer_oracle.h")
    if (not force and os.path.exists(SO)
            and os.path.getmtime(SO) >= max(os.path.getmtime(src), os.path.getmtime(hdr))):
        return SO
    cmd = ["gcc", "-O3", "-march=x86-64-v3", "-fopenmp", "-Wall", "-shared", "-fPIC",
           "-o", SO, src, "-lm"]
    subprocess.run(cmd, check=True)
    return SO


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
