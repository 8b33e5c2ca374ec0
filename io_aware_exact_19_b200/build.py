"""Build libfa.so in-tree with nvcc for sm_100a.

Usage: ``python -m io_aware_exact_19_b200.build`` (or call :func:`build`).
Objects go to ``io_aware_exact_19_b200/_build``; the library is
``io_aware_exact_19_b200/libfa.so``. Rebuilds only what changed.
"""
from __future__ import annotations

import glob
import os
import shutil
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
BUILD = os.path.join(HERE, "_build")
LIB = os.path.join(HERE, "libfa.so")
INCLUDE = os.path.join(os.path.dirname(HERE), "include")
SOURCES = ["fa_api.cu", "fa_fwd.cu", "fa_bwd.cu", "fa_splitkv.cu", "fa_decode.cu", "fa_dropout.cu", "fa_bwd_noalloc.cu"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "--expt-relaxed-constexpr",
         "-Xptxas", "-v"]


def _nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _deps_mtime() -> float:
    files = glob.glob(os.path.join(CSRC, "*")) + glob.glob(os.path.join(INCLUDE, "*.h")) + [__file__]
    return max(os.path.getmtime(f) for f in files)


def _compile(src: str, verbose: bool) -> str:
    obj = os.path.join(BUILD, os.path.splitext(src)[0] + ".o")
    if os.path.exists(obj) and os.path.getmtime(obj) >= _deps_mtime():
        return obj
    cmd = [_nvcc(), *ARCH, *FLAGS, "-I", INCLUDE, "-c", os.path.join(CSRC, src), "-o", obj]
    r = subprocess.run(cmd, capture_output=True, text=True)
    log = os.path.join(BUILD, os.path.splitext(src)[0] + ".log")
    with open(log, "w") as f:
        f.write(" ".join(cmd) + "\n" + r.stdout + r.stderr)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed for {src}:\n{r.stderr[-4000:]}")
    if verbose:
        sys.stdout.write(r.stderr)
    return obj


# Kernels that re-split registers with setmaxnreg: the split assumes this many
# registers per thread at launch. A smaller launch allocation would leave the
# setmaxnreg.inc waiting forever, so the build refuses it.
SETMAXNREG_LAUNCH_REGS = {"fa_fwd_kernel": 168, "fa_bwd_main_kernel": 168}


def _check_launch_registers(src: str) -> None:
    import re
    log = os.path.join(BUILD, os.path.splitext(src)[0] + ".log")
    if not os.path.exists(log):
        return
    text = open(log).read()
    entries = re.findall(r"Compiling entry function '(\S+)'.*?Used (\d+) registers", text, flags=re.S)
    for mangled, regs in entries:
        for name, want in SETMAXNREG_LAUNCH_REGS.items():
            if name in mangled and int(regs) != want:
                raise RuntimeError(f"{mangled}: {regs} registers at launch, the register split needs {want}")


def build(verbose: bool = False) -> str:
    """Compile every CUDA source for sm_100a and link libfa.so; returns its path."""
    os.makedirs(BUILD, exist_ok=True)
    with ThreadPoolExecutor(max_workers=len(SOURCES)) as ex:
        objs = list(ex.map(lambda s: _compile(s, verbose), SOURCES))
    for src in SOURCES:
        _check_launch_registers(src)
    if not os.path.exists(LIB) or os.path.getmtime(LIB) < max(os.path.getmtime(o) for o in objs):
        tmp = LIB + ".tmp"
        cmd = [_nvcc(), *ARCH, "-shared", "-o", tmp, *objs]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"link failed:\n{r.stderr[-4000:]}")
        os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(verbose="-v" in sys.argv))
