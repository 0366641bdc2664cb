"""Build the in-tree CUDA library ``libwf_b200.so`` for sm_100a (nvcc cross-compiles; no GPU needed).

    python -m block_causal_streaming_b200.build [-v]

The library is two translation units linked against the static CUDA runtime, so it only needs
the driver at run time:
- ``csrc/wf_api.cu`` includes the kernels;
- ``csrc/wf_window.cpp`` is the host-only rolling-window planner.
"""
from __future__ import annotations

import os
import re
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libwf_b200.so")
SOURCES = [os.path.join(CSRC, "wf_api.cu"), os.path.join(CSRC, "wf_window.cpp")]
DEPENDS = SOURCES + [os.path.join(CSRC, f) for f in ("sm100.cuh", "attn_kernel.cuh",
                                                      "append_kernel.cuh", "combine_kernel.cuh",
                                                      "fp8_kernel.cuh",
                                                      "publish_kernel.cuh")] + \
    [os.path.join(ROOT, "include", "wf.h")]

NVCC_FLAGS = [
    "-O3", "-std=c++17", "-lineinfo",
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-shared", "-Xcompiler", "-fPIC", "-cudart", "static",
    "-I" + os.path.join(ROOT, "include"),
]


def nvcc() -> str:
    cand = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    return cand if os.path.exists(cand) else "nvcc"


def needs_build(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    return any(os.path.getmtime(f) > t for f in DEPENDS if os.path.exists(f))


# The attention kernel splits its register file with setmaxnreg assuming it is launched with
# 168 registers per thread (384 threads); a different count would make the split wait forever.
ATTN_LAUNCH_REGS = 168


def check_register_counts(ptxas_log: str) -> None:
    """Fail the build unless every attention kernel was compiled for ATTN_LAUNCH_REGS."""
    entry = None
    found = 0
    for line in ptxas_log.splitlines():
        m = re.search(r"Compiling entry function '([^']+)'", line)
        if m:
            entry = m.group(1)
            continue
        m = re.search(r"Used (\d+) registers", line)
        if m and entry and "wf_attn_fwd_kernel" in entry:
            found += 1
            if int(m.group(1)) != ATTN_LAUNCH_REGS:
                raise RuntimeError(f"{entry}: {m.group(1)} registers, expected {ATTN_LAUNCH_REGS}"
                                   " (the setmaxnreg split in attn_kernel.cuh depends on it)")
            entry = None
    if found == 0:
        raise RuntimeError("ptxas reported no attention kernel")


def build(verbose: bool = False, force: bool = False, out: str = LIB) -> str:
    if not force and not needs_build(out):
        return out
    cmd = [nvcc()] + NVCC_FLAGS + ["-Xptxas", "-v"] + SOURCES + ["-o", out]
    res = subprocess.run(cmd, capture_output=True, text=True)
    if verbose or res.returncode != 0:
        sys.stderr.write(res.stdout + res.stderr)
    if res.returncode != 0:
        raise RuntimeError(f"nvcc failed ({res.returncode}): {' '.join(cmd)}")
    try:
        check_register_counts(res.stdout + res.stderr)
    except RuntimeError:
        os.remove(out)
        raise
    return out


if __name__ == "__main__":
    print(build(verbose="-v" in sys.argv, force=True))
