"""Builds libfmoe.so (the C-ABI library, sm_100a) in the package directory."""
import glob
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
SO = os.path.join(HERE, "libfmoe.so")
CSRC = os.path.join(HERE, "csrc")
MAIN = os.path.join(CSRC, "fmoe_api.cu")

NVCC_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17",
              "-Xcompiler", "-fPIC", "-shared"]


def _sources():
    return glob.glob(os.path.join(CSRC, "*")) + [os.path.join(ROOT, "include", "fmoe.h")]


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and os.path.exists(SO):
        newest = max(os.path.getmtime(s) for s in _sources())
        if os.path.getmtime(SO) >= newest:
            return SO
    cmd = ["nvcc", *NVCC_FLAGS, MAIN, "-o", SO]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    subprocess.run(cmd, check=True)
    return SO


if __name__ == "__main__":
    print(build(force=True, verbose=True))
