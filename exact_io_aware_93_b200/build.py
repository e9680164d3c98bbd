"""Build the sm_100a shared library ``libfa_b200.so`` in-tree with nvcc.

    python -m exact_io_aware_93_b200.build [--verbose]

The library statically links the CUDA runtime and reaches the driver's
tensor-map encoder through the runtime's entry-point query, so it loads on a
machine without a GPU (the exported symbols can be inspected there) and needs
only the NVIDIA driver at run time.
"""
from __future__ import annotations

import os
import re
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(PKG, "csrc")
LIB_NAME = "libfa_b200.so"
LIB_PATH = os.path.join(PKG, LIB_NAME)
# the same sources compiled with FA_CHECKS: every kernel bounds-checks its TMA coordinates
# and global indices and reports a violation in the device status word (include/fa.h)
CHECKS_LIB_PATH = os.path.join(PKG, "libfa_b200_checks.so")
SOURCES = ["fa_api.cu"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def _nvcc() -> str:
    cand = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(cand):
        raise RuntimeError("nvcc not found: the CUDA toolkit is required to build libfa_b200.so")
    return cand


def _deps():
    out = []
    for f in sorted(os.listdir(CSRC)):
        if f.endswith((".cu", ".cuh", ".h")):
            out.append(os.path.join(CSRC, f))
    out.append(os.path.join(os.path.dirname(PKG), "include", "fa.h"))
    return out


def up_to_date(path: str = LIB_PATH) -> bool:
    if not os.path.exists(path):
        return False
    t = os.path.getmtime(path)
    return all(os.path.getmtime(p) <= t for p in _deps())


# Kernels whose warpgroups rebalance registers with setmaxnreg: the split assumes that ptxas
# gives every instantiation exactly the launch allocation named by the constant.
REG_CONTRACT = {
    "fa_fwd_kernel": ("fa_fwd_kernel.cuh", "kLaunchRegs"),
    "fa_bwd_main_kernel": ("fa_bwd_kernel.cuh", "kBwdLaunchRegs"),
}


def _constant(header: str, name: str) -> int:
    with open(os.path.join(CSRC, header)) as f:
        m = re.search(r"constexpr\s+uint32_t\s+" + name + r"\s*=\s*(\d+)", f.read())
    if not m:
        raise RuntimeError(f"{name} not found in {header}")
    return int(m.group(1))


def ptxas_registers(log: str):
    """(mangled entry name, registers) for every entry function in a `-Xptxas -v` report."""
    out, current = [], None
    for line in log.splitlines():
        m = re.search(r"Compiling entry function '([^']+)'", line)
        if m:
            current = m.group(1)
            continue
        m = re.search(r"Used (\d+) registers", line)
        if m and current is not None:
            out.append((current, int(m.group(1))))
            current = None
    return out


def check_register_contract(log: str) -> None:
    """Fail when a setmaxnreg kernel was compiled to a register count other than its launch
    allocation: the warpgroups' register split would then not add up."""
    regs = ptxas_registers(log)
    bad = []
    for kernel, (header, const) in REG_CONTRACT.items():
        want = _constant(header, const)
        found = [(name, n) for name, n in regs if kernel in name]
        if not found:
            bad.append(f"{kernel}: no instantiation in the ptxas report")
        bad += [f"{name}: {n} registers, the split assumes {want}" for name, n in found if n != want]
    if bad:
        raise RuntimeError("register contract broken:\n  " + "\n  ".join(bad))


def _build_one(path: str, defines, log_name: str, verbose: bool) -> None:
    tmp = f"{path}.{os.getpid()}.tmp"
    cmd = [_nvcc(), *ARCH, "-O3", "-std=c++17", "-lineinfo", "-shared", "-Xcompiler", "-fPIC",
           "-Xptxas", "-v", "-cudart", "static", *defines,
           *[os.path.join(CSRC, s) for s in SOURCES], "-o", tmp]
    res = subprocess.run(cmd, capture_output=True, text=True)
    log = os.path.join(PKG, log_name)
    with open(log, "w") as f:
        f.write(" ".join(cmd) + "\n" + res.stdout + res.stderr)
    if res.returncode != 0:
        raise RuntimeError(f"nvcc failed (see {log}):\n{res.stderr[-4000:]}")
    try:
        check_register_contract(res.stdout + res.stderr)
    except RuntimeError:
        os.unlink(tmp)
        raise
    os.replace(tmp, path)
    if verbose:
        print(res.stderr)


def build(force: bool = False, verbose: bool = False, checks: bool = True) -> str:
    """Build the release library and (checks=True) the checking build; returns the release
    library's path."""
    if force or not up_to_date(LIB_PATH):
        _build_one(LIB_PATH, [], "build.log", verbose)
    if checks and (force or not up_to_date(CHECKS_LIB_PATH)):
        _build_one(CHECKS_LIB_PATH, ["-DFA_CHECKS"], "build_checks.log", verbose)
    return LIB_PATH


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose="--verbose" in sys.argv)
    print(LIB_PATH)
