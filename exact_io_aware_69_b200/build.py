"""Build the CUDA library libfa.so in-tree (sm_100a only).

``python -m exact_io_aware_69_b200.build`` or ``build_library()``. The CUDA runtime is
linked statically and the driver entry point for TMA descriptors is fetched at run
time, so the library loads on a machine without a GPU (nothing can be launched
there, but every exported symbol can be checked).
"""

from __future__ import annotations

import json
import os
import re
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libfa.so")
# ptxas's resource report of the last build (registers and spills per kernel)
RESOURCES = os.path.join(PKG, "libfa.resources.json")
SOURCES = [os.path.join(CSRC, "fa_api.cu")]
DEPS = SOURCES + [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith(".cuh")] + [
    os.path.join(INCLUDE, "fa.h")]

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-lineinfo", "-O3", "-std=c++17",
    "-Xcompiler", "-fPIC", "-shared",
    "-cudart", "static",
]


def nvcc() -> str:
    cand = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    return cand if os.path.exists(cand) else "nvcc"


def up_to_date() -> bool:
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    return all(os.path.getmtime(p) <= t for p in DEPS if os.path.exists(p))


def parse_ptxas_report(text: str) -> dict:
    """Registers and spill bytes per kernel from ptxas's -v report: maps each mangled
    kernel name to {"registers", "spill_stores", "spill_loads"}."""
    out, cur = {}, None
    for line in text.splitlines():
        m = re.search(r"Compiling entry function '([^']+)'", line)
        if m:
            cur = m.group(1)
            out[cur] = {"registers": None, "spill_stores": 0, "spill_loads": 0}
            continue
        if cur is None:
            continue
        m = re.search(r"(\d+) bytes spill stores, (\d+) bytes spill loads", line)
        if m:
            out[cur]["spill_stores"], out[cur]["spill_loads"] = int(m.group(1)), int(m.group(2))
        m = re.search(r"Used (\d+) registers", line)
        if m:
            out[cur]["registers"] = int(m.group(1))
    return out


# Kernels that move registers between warpgroups with setmaxnreg: their split adds up
# to exactly this many registers per thread at launch, so the compiled kernel must use
# exactly that many (the library also refuses to launch otherwise).
FIXED_REGISTERS = {"fa_bwd_main_kernel": 128, "fa_fwd_pp_kernel": 168}


def check_resources(report: dict) -> None:
    for name, res in report.items():
        for kernel, regs in FIXED_REGISTERS.items():
            if kernel in name and res["registers"] != regs:
                raise RuntimeError(f"{name}: compiled with {res['registers']} registers per "
                                   f"thread; its register split needs exactly {regs}")


def build_library(force: bool = False, verbose: bool = False) -> str:
    if not force and up_to_date() and os.path.exists(RESOURCES):
        return LIB
    tmp = LIB + f".tmp{os.getpid()}"
    cmd = [nvcc(), *NVCC_FLAGS, "-Xptxas", "-v", "-I", INCLUDE, "-I", CSRC, *SOURCES, "-o", tmp]
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError(f"nvcc failed ({res.returncode}):\n{res.stdout}\n{res.stderr}")
    if verbose:
        sys.stderr.write(res.stderr)
    report = parse_ptxas_report(res.stderr)
    try:
        check_resources(report)
    except RuntimeError:
        os.unlink(tmp)
        raise
    with open(RESOURCES + ".tmp", "w") as fh:
        json.dump(report, fh, indent=1, sort_keys=True)
    os.replace(RESOURCES + ".tmp", RESOURCES)
    os.replace(tmp, LIB)
    return LIB


def resources() -> dict:
    """ptxas's report of the current build (builds first when it is missing)."""
    build_library()
    with open(RESOURCES) as fh:
        return json.load(fh)


if __name__ == "__main__":
    print(build_library(force="--force" in sys.argv, verbose="-v" in sys.argv))
