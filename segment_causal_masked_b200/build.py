"""Build libsca.so in place with nvcc for sm_100a.

    python -m segment_causal_masked_b200.build [--verbose]

The library is a plain C-ABI shared object (include/sca.h); the CUDA runtime
is linked statically and the driver's tensor-map encoder is looked up at run
time, so the .so loads on a machine without a GPU.
"""
from __future__ import annotations

import os
import re
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libsca.so")
SOURCES = ["sca_host.cpp", "sca_kernels.cu", "sca_bwd.cu", "sca_static_ws.cu", "sca_camera.cu"]
HEADERS = ["sca_internal.h", "sca_ptx.cuh", "sca_camera.h"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
# Registers per thread that each warp-specialised kernel must be launched
# with: its setmaxnreg split (static_asserts beside the kernels) adds up to
# exactly threads x this. A kernel launched with fewer would have its
# growing warpgroups wait for registers that never come free, so the build
# refuses such a library. Keys are fragments of the mangled entry names.
LAUNCH_REGISTERS = {
    "attn_fwd_kernelILb0E": 168,   # bf16 cache: 384 threads, 224 / 224 / 56
    "attn_fwd_kernelILb1E": 128,   # INT8 cache: 512 threads, 216 / 216 / 40 / 40
    "bwd_dq_kernel": 168,          # 384 threads, 224 / 224 / 56
    "bwd_dkdv_kernel": 168,
}


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _newer(target: str, deps) -> bool:
    if not os.path.exists(target):
        return False
    t = os.path.getmtime(target)
    return all(os.path.getmtime(d) <= t for d in deps)


def kernel_registers(ptxas_log: str) -> dict:
    """{mangled entry name: registers per thread} from `-Xptxas -v` output."""
    regs, entry = {}, None
    for line in ptxas_log.splitlines():
        m = re.search(r"Compiling entry function '([^']+)'", line)
        if m:
            entry = m.group(1)
            continue
        m = re.search(r"Used (\d+) registers", line)
        if m and entry is not None:
            regs[entry] = int(m.group(1))
            entry = None
    return regs


def check_launch_registers(ptxas_log: str) -> None:
    """Raise unless every warp-specialised kernel was given exactly the
    registers its setmaxnreg split is built for."""
    regs = kernel_registers(ptxas_log)
    for frag, want in LAUNCH_REGISTERS.items():
        got = [r for name, r in regs.items() if frag in name]
        if not got:
            raise RuntimeError(f"no kernel matching {frag} in the ptxas report")
        if any(r != want for r in got):
            raise RuntimeError(f"{frag}: ptxas assigned {got} registers per thread, the "
                               f"setmaxnreg split needs {want}")


def build(verbose: bool = False, force: bool = False) -> str:
    deps = [os.path.join(CSRC, s) for s in SOURCES]
    deps += [os.path.join(CSRC, h) for h in HEADERS] + [os.path.join(INCLUDE, "sca.h")]
    if not force and _newer(LIB, deps):
        return LIB
    cmd = [nvcc(), *ARCH, "-O3", "-lineinfo", "-std=c++17", "-shared", "-Xcompiler", "-fPIC",
           "-Xcompiler", "-fvisibility=hidden", "-I", INCLUDE, "-I", CSRC,
           "-DSCA_BUILD", "-Xptxas", "-v", "-o", LIB + ".tmp"]
    cmd += [os.path.join(CSRC, s) for s in SOURCES]
    proc = subprocess.run(cmd, capture_output=True, text=True)
    if verbose or proc.returncode != 0:
        sys.stderr.write(proc.stdout + proc.stderr)
    if proc.returncode != 0:
        raise RuntimeError("nvcc failed building libsca.so")
    try:
        check_launch_registers(proc.stdout + proc.stderr)
    except RuntimeError:
        os.remove(LIB + ".tmp")
        raise
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    build(verbose="--verbose" in sys.argv, force=True)
    print(LIB)
