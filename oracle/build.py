"""Build liboracle.so, the float64 GEMV helpers of the CPU oracle (test infrastructure)."""
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))


def build() -> None:
    subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", os.path.join(HERE, "gemv.c"),
                           "-o", os.path.join(HERE, "liboracle.so")])


if __name__ == "__main__":
    build()
