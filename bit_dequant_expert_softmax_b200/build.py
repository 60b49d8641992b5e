"""Builds libfmoe.so (the C-ABI library, sm_100a) in the package directory."""
import glob
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
SO = os.path.join(HERE, "libfmoe.so")
CSRC = os.path.join(HERE, "csrc")
MAIN = os.path.join(CSRC, "fmoe_api.cu")
TIER = os.path.join(CSRC, "fmoe_tier.cpp")  # host-memory expert tier (host code on the C ABI)

# -ftz=false is explicit: the single-token dot products read 4-/2-bit codes masked in
# place as subnormal floats (code * 2^(s - 149)); flushing subnormals to zero would turn
# every code into 0.  Fast-math flags imply flushing and are refused below.
NVCC_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17",
              "-ftz=false", "-Xcompiler", "-fPIC", "-shared"]
FORBIDDEN_FLAGS = ("-ftz=true", "--use_fast_math", "-use_fast_math", "--ftz=true")


def check_flags(flags) -> None:
    """Raises if the flags would flush subnormals (the kernels rely on them)."""
    bad = [f for f in flags if f in FORBIDDEN_FLAGS]
    if bad:
        raise ValueError(f"libfmoe.so must be built without {bad}: its dequantising dot products "
                         "read codes as subnormal floats")


def _sources():
    return glob.glob(os.path.join(CSRC, "*")) + [os.path.join(ROOT, "include", "fmoe.h")]


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and os.path.exists(SO):
        newest = max(os.path.getmtime(s) for s in _sources())
        if os.path.getmtime(SO) >= newest:
            return SO
    check_flags(NVCC_FLAGS)
    cmd = ["nvcc", *NVCC_FLAGS, MAIN, TIER, "-o", SO]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    subprocess.run(cmd, check=True)
    return SO


if __name__ == "__main__":
    print(build(force=True, verbose=True))
