"""In-tree build of libdcattn.so (nvcc, sm_100a only)."""
from __future__ import annotations

import glob
import os
import re
import subprocess

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libdcattn.so")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++20",
    "-Xcompiler", "-fPIC", "-shared",
    "--expt-relaxed-constexpr",
]


def _sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cuh")) +
                  [os.path.join(INCLUDE, "dcattn.h")])


# Every tcgen05 kernel splits its registers between warpgroups with setmaxnreg
# on the assumption that it launches with exactly this many per thread.
TC_LAUNCH_REGS = 128


def check_register_split(ptxas_log: str) -> None:
    """Fail unless every tcgen05 kernel (namespace dc::tc) uses exactly TC_LAUNCH_REGS."""
    current = None
    seen = 0
    for line in ptxas_log.splitlines():
        m = re.search(r"Function properties for (\S+)", line)
        if m:
            current = m.group(1)
            continue
        m = re.search(r"Used (\d+) registers", line)
        if m and current and "_ZN2dc2tc" in current and "_kernel" in current:
            seen += 1
            if int(m.group(1)) != TC_LAUNCH_REGS:
                raise RuntimeError(f"{current} uses {m.group(1)} registers, the register split needs "
                                   f"{TC_LAUNCH_REGS}")
    if seen == 0:
        raise RuntimeError("no tcgen05 kernel found in the ptxas report")


def build(force: bool = False, verbose: bool = False) -> str:
    """Compile csrc/dcattn.cu (which includes every kernel) into libdcattn.so."""
    newest = max(os.path.getmtime(p) for p in _sources())
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= newest:
        return LIB
    nvcc = os.environ.get("NVCC", "nvcc")
    tmp = LIB + f".tmp{os.getpid()}"
    cmd = [nvcc, *NVCC_FLAGS, "-Xptxas=-v", "-I", INCLUDE, "-I", CSRC, "-o", tmp, os.path.join(CSRC, "dcattn.cu")]
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError(f"nvcc failed:\n{res.stdout}\n{res.stderr}")
    if verbose:
        print(res.stderr)
    try:
        check_register_split(res.stderr)
    except RuntimeError:
        os.remove(tmp)
        raise
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    import sys
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
