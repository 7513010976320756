"""Builds libadamw4.so in-tree with nvcc for sm_100a.

Flags that matter for the results: -fmad=false (no implicit multiply-add
contraction), IEEE division and square root, denormals kept.  The kernel names
every fused multiply-add it wants explicitly, so the result does not depend on
the compiler's contraction choices.
"""
import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "csrc", "adamw4.cu")
OUT = os.path.join(HERE, "libadamw4.so")
DEPS = [SRC, os.path.join(HERE, "csrc", "adamw4_kernel.cuh"), os.path.join(HERE, "csrc", "nf4_table.h"),
        os.path.join(HERE, "csrc", "exact_math.cuh"),
        os.path.join(os.path.dirname(HERE), "include", "adamw4.h")]
# The GPU verification of exact_math.cuh against the IEEE operations (a test
# library; the step library does not link it).
CHECK_SRC = os.path.join(HERE, "csrc", "exact_math_check.cu")
OUT_EXACT_CHECK = os.path.join(HERE, "libadamw4_exact_check.so")


def nvcc():
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def flags():
    return ["-O3", "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo",
            "-fmad=false", "-prec-div=true", "-prec-sqrt=true", "-ftz=false",
            "-Xcompiler", "-fPIC", "-Xcompiler", "-Wall", "-shared", "-Xptxas", "-v"]


OUT_CHECKED = os.path.join(HERE, "libadamw4_checked.so")


def build(force=False, verbose=False, checked=False, exact_check=False):
    """Builds libadamw4.so, or with checked=True libadamw4_checked.so, the
    same library with device-side range checks (-DADAMW4_CHECKED), or with
    exact_check=True the verification library of the fast division and
    square root, libadamw4_exact_check.so."""
    out = OUT_EXACT_CHECK if exact_check else (OUT_CHECKED if checked else OUT)
    src = CHECK_SRC if exact_check else SRC
    deps = [CHECK_SRC, os.path.join(HERE, "csrc", "exact_math.cuh")] if exact_check else DEPS
    if not force and os.path.exists(out) and all(
            os.path.getmtime(out) >= os.path.getmtime(d) for d in deps):
        return out
    tmp = out + f".tmp{os.getpid()}"
    cmd = [nvcc()] + flags() + (["-DADAMW4_CHECKED"] if checked else []) + [src, "-o", tmp]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError("nvcc failed:\n" + r.stdout + r.stderr)
    if verbose:
        sys.stderr.write(r.stderr)
    os.replace(tmp, out)
    return out


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True, checked="--checked" in sys.argv,
                exact_check="--exact-check" in sys.argv))
