"""Build the fp64 CPU oracle (test infrastructure) into oracle/liboracle.so with gcc.

Only the test suite, the package smoke check and the benchmark's CPU-baseline leg load
the result.  Flags: no fast-math and no floating-point contraction, so that the fp32
remap of the approximate top-k is evaluated operation by operation in round-to-nearest.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "vx_oracle.c")
LIB = os.path.join(HERE, "liboracle.so")


def build(force: bool = False) -> str:
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= os.path.getmtime(SRC):
        return LIB
    cmd = ["gcc", "-std=c11", "-O2", "-fopenmp", "-fPIC", "-shared", "-ffp-contract=off",
           "-fno-fast-math", "-Wall", "-Wextra", "-o", LIB, SRC, "-lm"]
    subprocess.run(cmd, check=True)
    return LIB



def build_variant(source_text: str, out_dir: str, name: str) -> str:
    """Compile an edited copy of the oracle source (mutation tests) into out_dir."""
    src = os.path.join(out_dir, name + ".c")
    lib = os.path.join(out_dir, name + ".so")
    with open(src, "w") as f:
        f.write(source_text)
    subprocess.run(["gcc", "-std=c11", "-O1", "-fopenmp", "-fPIC", "-shared", "-ffp-contract=off",
                    "-fno-fast-math", "-w", "-o", lib, src, "-lm"], check=True)
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
