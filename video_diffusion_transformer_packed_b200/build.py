"""Builds the in-tree C-ABI library libwanattn.so for sm_100a with nvcc.

    python -m video_diffusion_transformer_packed_b200.build [--force] [--verbose] [--debug-bounds]

The library is self-contained (static CUDA runtime, driver entry points
resolved at run time), so it loads on a machine without a GPU.
"""
from __future__ import annotations

import argparse
import os
import re
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
SOURCES = ["abi.cu", "qk_norm_rope.cu", "attn_fwd.cu", "host_pipeline.cu", "fp8_quant.cu", "attn_fwd_fp8.cu", "gemm_bf16.cu",
           "attn_merge.cu", "host_static.cu"]
HEADERS = ["sm100.cuh", "wan_kernels.h", "debug_bounds.cuh"]
LIB = os.path.join(PKG, "_lib", "libwanattn.so")
# The debug-bounds build: device-side index checks (debug_bounds.cuh) compiled in.
LIB_DEBUG = os.path.join(PKG, "_lib", "libwanattn_debug.so")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: the CUDA toolkit is required to build libwanattn.so")


def _inputs():
    files = [os.path.join(CSRC, f) for f in SOURCES + HEADERS]
    files.append(os.path.join(ROOT, "include", "wan_attn.h"))
    files.append(os.path.abspath(__file__))
    return files


def stale(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    return any(os.path.getmtime(f) > t for f in _inputs())


# Kernels that split their registers between warpgroups with setmaxnreg: the
# split is only valid when the compiled kernel launches with exactly the
# register count its source names (kLaunchRegs). (source file, kernel name)
SPLIT_REGISTER_KERNELS = [("attn_fwd.cu", "attn_fwd_kernel"), ("attn_fwd_fp8.cu", "attn_fwd_fp8_kernel")]


def check_register_splits(ptxas_log: str) -> None:
    """Fail the build when a split-register kernel did not compile to the
    register count its source assumes (ptxas -v: 'Used N registers' after
    'Compiling entry function <name>')."""
    entries = re.findall(r"Compiling entry function '([^']+)'.*?Used (\d+) registers", ptxas_log, re.S)
    for src, kernel in SPLIT_REGISTER_KERNELS:
        text = open(os.path.join(CSRC, src)).read()
        m = re.search(r"constexpr int kLaunchRegs = (\d+);", text)
        if m is None:
            continue  # this kernel no longer splits its registers
        want = int(m.group(1))
        found = [(name, int(n)) for name, n in entries if kernel in name and src.replace(".", "_") in name]
        if not found:
            raise RuntimeError(f"ptxas reported no entry function {kernel} of {src}")
        bad = [(name, n) for name, n in found if n != want]
        if bad:
            raise RuntimeError(f"{kernel} ({src}) compiled to {bad[0][1]} registers per thread; its per-warpgroup "
                               f"register split (setmaxnreg) assumes kLaunchRegs = {want}. Adjust kLaunchRegs and "
                               f"the split, or build with the toolkit the source was tuned for.")


def build(force: bool = False, verbose: bool = False, extra_flags=(), debug_bounds: bool = False) -> str:
    """Builds libwanattn.so, or with debug_bounds the checked libwanattn_debug.so."""
    lib = LIB_DEBUG if debug_bounds else LIB
    if debug_bounds:
        extra_flags = (*extra_flags, "-DWAN_DEBUG_BOUNDS")
    if not force and not stale(lib):
        return lib
    os.makedirs(os.path.dirname(lib), exist_ok=True)
    tmp = lib + f".{os.getpid()}.tmp"
    cmd = [nvcc(), *ARCH, "-O3", "-lineinfo", "-std=c++17", "-shared", "-Xcompiler", "-fPIC",
           "-Xcompiler", "-fvisibility=hidden", "--expt-relaxed-constexpr",
           "-I", os.path.join(ROOT, "include"), "-Xptxas", "-v", *extra_flags]
    cmd += [os.path.join(CSRC, f) for f in SOURCES] + ["-o", tmp]
    res = subprocess.run(cmd, capture_output=True, text=True)
    if verbose or res.returncode != 0:
        sys.stderr.write(res.stdout + res.stderr)
    if res.returncode != 0:
        raise subprocess.CalledProcessError(res.returncode, cmd, res.stdout, res.stderr)
    try:
        check_register_splits(res.stdout + res.stderr)
    except RuntimeError:
        os.remove(tmp)
        raise
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose", action="store_true")
    ap.add_argument("--debug-bounds", action="store_true", help="build the checked libwanattn_debug.so")
    a = ap.parse_args()
    print(build(force=a.force, verbose=a.verbose, debug_bounds=a.debug_bounds))
    sys.exit(0)
