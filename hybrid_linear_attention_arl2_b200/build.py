"""Build libarl2.so in-tree with nvcc for sm_100a.

    python -m hybrid_linear_attention_arl2_b200.build [--debug-ptxas] [--debug-bounds]

The library is a plain shared object with a C ABI (include/arl2.h); the CUDA
runtime is linked statically, so loading it needs only the NVIDIA driver at
call time (the CPU tests load it without a GPU).  `--debug-bounds` builds
libarl2_debug.so instead: the same sources with -DARL2_DEBUG_BOUNDS, whose
kernels check the indices they take from their parameters and launch shape and
report a failed check through arl2_last_error (ARL2_ERR_BOUNDS).
"""
from __future__ import annotations

import os
import re
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
ROOT = os.path.dirname(HERE)
LIB = os.path.join(HERE, "libarl2.so")
LIB_DEBUG = os.path.join(HERE, "libarl2_debug.so")
SOURCES = ["arl2_api.cu", "attn_pair.cu", "gemm_bf16.cu", "state_bf16.cu", "f32_path.cu", "util.cu", "block.cu", "token_level.cu"]
HEADERS = ["params.h", "layer.h", "sm100.cuh"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc() -> str:
    for c in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if c and (os.path.isabs(c) and os.path.exists(c) or not os.path.isabs(c)):
            return c
    return "nvcc"


def _stale(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    deps = [os.path.join(CSRC, f) for f in SOURCES + HEADERS] + [os.path.join(ROOT, "include", "arl2.h"),
                                                                 os.path.abspath(__file__)]
    return any(os.path.getmtime(p) > t for p in deps)


def _check_launch_registers(cmd: list, echo: bool = False) -> None:
    """Compile the attention kernel and check that it was allocated exactly
    the registers per thread its warp-role split (setmaxnreg) is sized for:
    with any other count the launch is refused at run time (a larger split
    than the launch holds would never be granted)."""
    if "-v" not in cmd:
        cmd = cmd + ["-Xptxas", "-v"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if echo or r.returncode != 0:
        sys.stderr.write(r.stderr)
    if r.returncode != 0:
        raise subprocess.CalledProcessError(r.returncode, cmd)
    src = open(os.path.join(CSRC, "attn_pair.cu")).read()
    want = int(re.search(r"constexpr int kLaunchRegs = (\d+);", src).group(1))
    m = re.search(r"Compiling entry function '[^']*attn_pair_kernel[^']*'.*?Used (\d+) registers", r.stderr, re.S)
    if not m or int(m.group(1)) != want:
        got = m.group(1) if m else "an unknown number of"
        raise RuntimeError(f"attn_pair_kernel compiled to {got} registers per thread; its register split "
                           f"needs {want}")


def build(force: bool = False, verbose_ptxas: bool = False, debug_bounds: bool = False) -> str:
    """Build libarl2.so (or, with debug_bounds, libarl2_debug.so) when a
    source is newer than it; returns its path."""
    lib = LIB_DEBUG if debug_bounds else LIB
    if not force and not _stale(lib):
        return lib
    objdir = os.path.join(HERE, "_build_debug" if debug_bounds else "_build")
    os.makedirs(objdir, exist_ok=True)
    objs = []
    flags = ARCH + ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC,-O2", "--expt-relaxed-constexpr",
                    "-I" + os.path.join(ROOT, "include")]
    if debug_bounds:
        flags += ["-DARL2_DEBUG_BOUNDS"]
    if verbose_ptxas:
        flags += ["-Xptxas", "-v"]
    for src in SOURCES:
        obj = os.path.join(objdir, src.replace(".cu", ".o"))
        cmd = [nvcc()] + flags + ["-c", os.path.join(CSRC, src), "-o", obj]
        if src == "attn_pair.cu":
            _check_launch_registers(cmd, echo=verbose_ptxas)
        else:
            subprocess.run(cmd, check=True)
        objs.append(obj)
    tmp = lib + ".tmp"
    subprocess.run([nvcc()] + ARCH + ["-shared", "-o", tmp] + objs + ["-lcudart_static", "-ldl", "-lrt", "-lpthread"],
                   check=True)
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    print(build(force=True, verbose_ptxas="--debug-ptxas" in sys.argv, debug_bounds="--debug-bounds" in sys.argv))
