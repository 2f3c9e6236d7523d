"""Build the sm_100a CUDA library in-tree (``libexact_attn_b200.so`` beside this file).

csrc/attn_api.cu (which includes every kernel) and csrc/attn_noalloc.cu,
compiled with nvcc for sm_100a only. No GPU is needed to build.
"""
from __future__ import annotations

import os
import re
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libexact_attn_b200.so")
# The debug build: the same sources with -DATTN_DEBUG, whose kernels check the
# global-memory indices they compute (see dcheck in csrc/ptx_sm100.cuh).
LIB_DEBUG = os.path.join(HERE, "libexact_attn_b200_debug.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "--expt-relaxed-constexpr",
    "-Xcompiler", "-fPIC", "-shared",
    "-Xptxas", "-v",
]


def sources():
    return [os.path.join(CSRC, f) for f in sorted(os.listdir(CSRC))
            if f.endswith((".cu", ".cuh"))] + [os.path.join(ROOT, "include", "exact_attn.h")]


def up_to_date(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return False
    t = os.path.getmtime(lib)
    return all(os.path.getmtime(s) <= t for s in sources())


def build(force: bool = False, verbose: bool = False, debug: bool = False) -> str:
    lib = LIB_DEBUG if debug else LIB
    if not force and up_to_date(lib):
        return lib
    cmd = [NVCC, *FLAGS, *(["-DATTN_DEBUG"] if debug else []), "-I", os.path.join(ROOT, "include"),
           "-I", CSRC, os.path.join(CSRC, "attn_api.cu"), os.path.join(CSRC, "attn_noalloc.cu"),
           "-o", lib]
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        sys.stderr.write(res.stdout + res.stderr)
        raise RuntimeError("nvcc failed building the attention library")
    if verbose:
        sys.stderr.write(res.stderr)
    check_register_budget(res.stdout + res.stderr, lib)
    return lib


# The prefill kernel redistributes registers with setmaxnreg assuming each of
# its 384 threads received exactly this many at launch (FwdTraits::kLaunchRegs).
# Fewer at launch would make the softmax warpgroups' increase wait forever, so
# the build refuses to produce such a library.
FWD_LAUNCH_REGS = 168
# The backward kernel launches 20 warps with this many registers each and
# redistributes them with setmaxnreg (BwdTraits::kLaunchRegs); with fewer at
# launch the P/dS warpgroups' increase would wait forever, and more would not
# fit five warps per SM scheduler, so the build requires exactly this count.
BWD_LAUNCH_REGS = 96


def check_register_budget(ptxas_log: str, lib: str = LIB) -> None:
    current = None
    seen = 0
    seen_bwd = 0
    for line in ptxas_log.splitlines():
        m = re.search(r"Compiling entry function '([^']+)'", line)
        if m:
            current = m.group(1)
            continue
        m = re.search(r"Used (\d+) registers", line)
        if m and current and "attn_bwd_sm100_kernel" in current:
            seen_bwd += 1
            if int(m.group(1)) != BWD_LAUNCH_REGS:
                os.remove(lib)
                raise RuntimeError(f"{current} uses {m.group(1)} registers, expected "
                                   f"{BWD_LAUNCH_REGS}: the setmaxnreg split would not fit")
        if m and current and "attn_fwd_sm100_kernel" in current:
            seen += 1
            if int(m.group(1)) != FWD_LAUNCH_REGS:
                os.remove(lib)
                raise RuntimeError(f"{current} uses {m.group(1)} registers, expected "
                                   f"{FWD_LAUNCH_REGS}: the setmaxnreg split would not fit")
    if seen == 0 or seen_bwd == 0:
        os.remove(lib)
        raise RuntimeError("ptxas register report for the prefill or backward kernel not found")


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True, debug="--debug" in sys.argv))
