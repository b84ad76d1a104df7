"""Build libwave.so in-tree with nvcc for sm_100a.

Usage: ``python -m block_causal_attention_wave_b200.build [--verbose-ptxas]``.
Compiles every ``csrc/*.cu`` / ``csrc/*.cpp`` into one shared library next to
this file; the CUDA runtime is linked statically so the library needs only the
NVIDIA driver at run time.
"""
from __future__ import annotations

import glob
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
LIB = os.path.join(PKG, "libwave.so")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc() -> str:
    path = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(path):
        raise RuntimeError("nvcc not found")
    return path


def sources():
    csrc = os.path.join(PKG, "csrc")
    return sorted(glob.glob(os.path.join(csrc, "*.cu")) + glob.glob(os.path.join(csrc, "*.cpp")))


def build(verbose_ptxas: bool = False, out: str = LIB, defines=(), replace=None) -> str:
    """Compile every source into ``out``; ``defines`` are extra -D macros;
    ``replace`` maps a source's file name to another file compiled in its place
    (a test build of one kernel; headers still come from ``csrc``)."""
    replace = dict(replace or {})
    objdir = os.path.join(PKG, "_build", os.path.splitext(os.path.basename(out))[0])
    os.makedirs(objdir, exist_ok=True)
    common = ARCH + ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC,-O2,-Wall",
                     "-I", os.path.join(ROOT, "include"), "-I", os.path.join(PKG, "csrc")]
    if verbose_ptxas:
        common += ["-Xptxas", "-v"]
    common += [f"-D{d}" for d in defines]
    objs = []
    for src in sources():
        obj = os.path.join(objdir, os.path.basename(src) + ".o")
        src = replace.pop(os.path.basename(src), src)
        cmd = [nvcc()] + common + ["-c", src, "-o", obj]
        r = subprocess.run(cmd, capture_output=True, text=True, timeout=900)
        if r.returncode != 0 or verbose_ptxas:
            sys.stderr.write(r.stdout + r.stderr)
        if r.returncode != 0:
            raise RuntimeError(f"nvcc failed on {os.path.basename(src)}")
        objs.append(obj)
    if replace:
        raise ValueError(f"no source named {sorted(replace)}")
    tmp = out + ".tmp"
    cmd = [nvcc()] + ARCH + ["-shared", "-cudart", "static", "-o", tmp] + objs
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=300)
    if r.returncode != 0:
        sys.stderr.write(r.stdout + r.stderr)
        raise RuntimeError("link of libwave.so failed")
    os.replace(tmp, out)
    return out


if __name__ == "__main__":
    print(build(verbose_ptxas="--verbose-ptxas" in sys.argv))
