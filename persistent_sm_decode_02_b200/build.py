"""Build libdec.so (sm_100a) in-tree with nvcc."""
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
SOURCES = [os.path.join(HERE, "csrc", "dec_api.cu"), os.path.join(HERE, "csrc", "noalloc.cu")]
FLAGS = ["-O3", "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo", "-Xcompiler", "-fPIC",
         "-shared", "-I", os.path.join(ROOT, "include")]


def build(verbose: bool = False) -> str:
    out = os.path.join(HERE, "libdec.so")
    cmd = ["nvcc"] + FLAGS + (["-Xptxas", "-v"] if verbose else []) + SOURCES + ["-o", out]
    subprocess.check_call(cmd)
    return out


if __name__ == "__main__":
    build(verbose=True)
