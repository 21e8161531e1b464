"""Builds the CUDA library libvlaq.so in-tree (sm_100a only).

    python vlaq_quantize_act_b200/build.py [--force]

nvcc compiles every .cu under csrc/ with -gencode arch=compute_100a,code=sm_100a
and links them into vlaq_quantize_act_b200/libvlaq.so with the CUDA runtime
linked statically (the driver API is reached through cudaGetDriverEntryPoint),
so the library loads on a machine without a GPU.
"""
from __future__ import annotations

import glob
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
OUT = os.path.join(HERE, "libvlaq.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17",
         "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden", "--expt-relaxed-constexpr"]


# Kernels that re-split registers between warpgroups with setmaxnreg: the
# per-warpgroup budgets they request add up to exactly this entry register
# count times the block size, so ptxas must allocate exactly this many at
# entry (fewer would make setmaxnreg.inc wait for registers that never free).
ENTRY_REGISTERS = {"gemm_fp4_sfw_kernel": 128, "gemm_fp4_pair_kernel": 128}


def _check_entry_registers(ptxas_log: str) -> None:
    current = None
    for line in ptxas_log.splitlines():
        if "Compiling entry function" in line:
            current = line
        elif current and "Used" in line and "registers" in line:
            for name, regs in ENTRY_REGISTERS.items():
                if name in current:
                    used = int(line.split("Used")[1].split("registers")[0])
                    if used != regs:
                        raise RuntimeError(f"{name}: ptxas allocated {used} registers at entry, "
                                           f"the setmaxnreg split needs exactly {regs}")
            current = None


def _sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _deps():
    return _sources() + sorted(glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h"))
                               + [os.path.join(HERE, "..", "include", "vlaq.h")])


def up_to_date() -> bool:
    if not os.path.exists(OUT):
        return False
    t = os.path.getmtime(OUT)
    return all(os.path.getmtime(d) <= t for d in _deps())


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and up_to_date():
        return OUT
    objdir = os.path.join(HERE, "_build")
    os.makedirs(objdir, exist_ok=True)
    objs = []
    for src in _sources():
        obj = os.path.join(objdir, os.path.basename(src) + ".o")
        cmd = [NVCC, *FLAGS, "-Xptxas=-v", "-c", src, "-o", obj]
        res = subprocess.run(cmd, capture_output=True, text=True)
        if verbose or res.returncode != 0:
            sys.stderr.write(res.stdout + res.stderr)
        if res.returncode != 0:
            raise subprocess.CalledProcessError(res.returncode, cmd)
        _check_entry_registers(res.stderr)
        objs.append(obj)
    tmp = OUT + ".tmp"
    subprocess.run([NVCC, "-shared", "-gencode", "arch=compute_100a,code=sm_100a", *objs, "-o", tmp,
                    "-cudart", "static"], check=True)
    os.replace(tmp, OUT)
    return OUT


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
