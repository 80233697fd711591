"""Builds liblosa.so in-tree with nvcc for sm_100a.

    python block_sparse_attention_losa_b200/build.py   (or build())

The library is plain C ABI (include/losa.h) over CUDA kernels; it links the
CUDA runtime statically and resolves the driver's tensor-map encoder at run
time, so it needs no libcuda at link time.
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "liblosa.so")
SOURCES = ["losa_api.cu", "losa_attention.cu", "losa_select.cu"]
HEADERS = ["losa_device.cuh", "losa_attention.cuh", "losa_cut.cuh", "losa_internal.h"]


def nvcc_path() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    deps = [os.path.join(CSRC, f) for f in SOURCES + HEADERS]
    deps.append(os.path.join(ROOT, "include", "losa.h"))
    deps.append(os.path.abspath(__file__))
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and not _stale():
        return LIB
    out_tmp = LIB + ".tmp"
    cmd = [nvcc_path(), "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo", "-O3",
           "-std=c++17", "-Xcompiler", "-fPIC", "-shared", "--expt-relaxed-constexpr",
           "-Xptxas", "-v", "-I", os.path.join(ROOT, "include"), "-o", out_tmp]
    cmd += [os.path.join(CSRC, f) for f in SOURCES]
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError("nvcc failed:\n" + res.stdout + res.stderr)
    if verbose:
        sys.stderr.write(res.stderr)
    check_attention_registers(res.stderr)
    os.replace(out_tmp, LIB)
    return LIB


def check_attention_registers(ptxas_log: str, want: int = 168) -> None:
    """The attention kernels split their launch registers between
    warpgroups with setmaxnreg; the split adds up only if every instance
    launches with exactly `want` registers per thread (else a warpgroup
    would wait for registers that never come). Refuse the build otherwise."""
    current, seen = None, 0
    for line in ptxas_log.splitlines():
        if "Compiling entry function" in line:
            current = "attn_kernel" in line
        elif current and "Used" in line and "registers" in line:
            used = int(line.split("Used")[1].split("registers")[0])
            seen += 1
            if used != want:
                raise RuntimeError(f"attention kernel launches with {used} registers, "
                                   f"the setmaxnreg split assumes {want}")
    if seen == 0:
        raise RuntimeError("no attention kernel found in the ptxas log")


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
