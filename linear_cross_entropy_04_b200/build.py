"""Build the CUDA library in-tree: linear_cross_entropy_04_b200/libflce.so.

    python -m linear_cross_entropy_04_b200.build [--verbose]

Compiles csrc/flce.cu for sm_100a only (B200) with nvcc. The CUDA runtime is
linked statically and the driver's cuTensorMapEncodeTiled is looked up at run
time, so the library also loads on a host without a GPU or driver (its
argument checks and planning then work; compute calls need a B200).
"""
import glob
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
SRC = os.path.join(PKG, "csrc", "flce.cu")
OUT = os.path.join(PKG, "libflce.so")

def deps():
    """Every source the library is compiled from: all of csrc/ and the public headers."""
    return sorted(glob.glob(os.path.join(PKG, "csrc", "*")) + glob.glob(os.path.join(ROOT, "include", "*.h")))


def nvcc_path():
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def command(verbose=False, out=OUT, defines=()):
    cmd = [nvcc_path(), "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo", "-O3",
           "-std=c++17", "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden", "-shared",
           "-cudart", "static", "-I", os.path.join(ROOT, "include"), "-o", out, SRC]
    cmd[1:1] = [f"-D{d}" for d in defines]
    if verbose:
        cmd[1:1] = ["-Xptxas", "-v"]
    return cmd


def up_to_date():
    if not os.path.exists(OUT):
        return False
    t = os.path.getmtime(OUT)
    return all(os.path.getmtime(d) <= t for d in deps())


def build(force=False, verbose=False, out=None, defines=()):
    """Compile the library; out/defines build a variant (e.g. tuning knobs) elsewhere."""
    if out is None and not force and up_to_date():
        return OUT
    r = subprocess.run(command(verbose, out or OUT, defines), capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError("nvcc failed:\n" + r.stdout + r.stderr)
    if verbose:
        sys.stderr.write(r.stdout + r.stderr)
    return out or OUT


if __name__ == "__main__":
    build(force=True, verbose="--verbose" in sys.argv)
    print(OUT)
