"""Builds the host (gcc) and device (nvcc, sm_100a) generator libraries."""
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
HOST_LIB = os.path.join(HERE, "libsynth.so")
CUDA_LIB = os.path.join(HERE, "libsynth_cuda.so")


def _stale(lib, deps):
    if not os.path.exists(lib):
        return True
    return os.path.getmtime(lib) < max(os.path.getmtime(d) for d in deps)


def build(force: bool = False, cuda: bool = True):
    core = os.path.join(HERE, "synth_core.h")
    host_src = os.path.join(HERE, "synth.c")
    if force or _stale(HOST_LIB, [core, host_src, __file__]):
        subprocess.run(["gcc", "-std=c11", "-O2", "-fPIC", "-shared", "-fopenmp",
                        "-ffp-contract=off", "-fno-fast-math", "-o", HOST_LIB, host_src, "-lm"],
                       check=True)
    if cuda:
        cu = os.path.join(HERE, "synth_cuda.cu")
        if force or _stale(CUDA_LIB, [core, cu, __file__]):
            subprocess.run(["nvcc", "-gencode", "arch=compute_100a,code=sm_100a", "-O3",
                            "-lineinfo", "--fmad=false", "-Xcompiler", "-fPIC", "-shared",
                            "-o", CUDA_LIB, cu], check=True)
    return HOST_LIB, CUDA_LIB


if __name__ == "__main__":
    print(build(force=True))
