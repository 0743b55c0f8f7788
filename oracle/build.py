"""Builds the CPU oracle shared library (test infrastructure only)."""
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
LIB = os.path.join(HERE, "libds4g_oracle.so")


def build(force: bool = False) -> str:
    src = [os.path.join(HERE, "ds4g_oracle.c")]
    hdr = os.path.join(HERE, "ds4g_oracle.h")
    if not force and os.path.exists(LIB):
        newest = max(os.path.getmtime(p) for p in src + [hdr, __file__])
        if os.path.getmtime(LIB) >= newest:
            return LIB
    cmd = ["gcc", "-std=c11", "-O2", "-fPIC", "-shared", "-fopenmp",
           "-ffp-contract=off", "-fexcess-precision=standard", "-fno-fast-math",
           "-o", LIB] + src + ["-lm"]
    subprocess.run(cmd, check=True)
    return LIB


if __name__ == "__main__":
    print(build(force=True))
