"""Build the seeded-generator libraries: libsynth.so (CPU, gcc) and libsynth_cuda.so (sm_100a, nvcc)."""
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))


def build(cuda: bool = True) -> None:
    # -ffp-contract=off: the value recipe is one fp32 multiply then one fp32 add, never an FMA.
    subprocess.check_call(["gcc", "-O2", "-fopenmp", "-ffp-contract=off", "-fPIC", "-shared",
                           os.path.join(HERE, "synth.c"), "-o", os.path.join(HERE, "libsynth.so"), "-lm"])
    if cuda:
        subprocess.check_call(["nvcc", "-O3", "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo",
                               "-Xcompiler", "-fPIC", "-shared", os.path.join(HERE, "synth_cuda.cu"),
                               "-o", os.path.join(HERE, "libsynth_cuda.so")])


if __name__ == "__main__":
    build()
