"""Builds the device-side input generator ``fmoe_synth/_synth.so`` (sm_100a)."""
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
SO = os.path.join(HERE, "_synth.so")
SRC = os.path.join(HERE, "csrc", "synth.cu")


def build(force: bool = False) -> str:
    if not force and os.path.exists(SO) and os.path.getmtime(SO) >= os.path.getmtime(SRC):
        return SO
    cmd = ["nvcc", "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo",
           "-fmad=false", "-Xcompiler", "-fPIC,-ffp-contract=off", "-shared", "-std=c++17",
           SRC, "-o", SO]
    subprocess.run(cmd, check=True)
    return SO


if __name__ == "__main__":
    print(build(force=True))
