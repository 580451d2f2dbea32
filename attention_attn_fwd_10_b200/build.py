"""Compile libattn.so (the C-ABI library of include/attn.h) for sm_100a, in-tree.

    python -m attention_attn_fwd_10_b200.build          # or build() from Python
    python -m attention_attn_fwd_10_b200.build --timeline

The second form builds libattn_timeline.so: the same sources with -DATTN_TIMELINE,
whose kernels record a per-block clock64 timeline of one chosen CTA
(include/attn_timeline.h; read by attention_attn_fwd_10_b200.timeline).  It is a
measurement aid, never loaded by the package unless asked for.

nvcc cross-compiles without a GPU.  The library links the CUDA runtime
statically and reaches the driver only through cudaGetDriverEntryPoint, so it
needs no libcuda at link time.
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
LIB = os.path.join(HERE, "libattn.so")
LIB_TIMELINE = os.path.join(HERE, "libattn_timeline.so")
SOURCES = [os.path.join(HERE, "csrc", "attn_api.cu")]
DEPS = SOURCES + [
    os.path.join(HERE, "csrc", f)
    for f in sorted(os.listdir(os.path.join(HERE, "csrc")))
    if f.endswith((".cuh", ".h"))
] + [os.path.join(ROOT, "include", "attn.h"), os.path.join(ROOT, "include", "attn_timeline.h")]

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-lineinfo", "-O3", "-std=c++17",
    "-shared", "-Xcompiler", "-fPIC",
    "-Xptxas", "-v",
]


def nvcc_path() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: the CUDA toolkit is required to build libattn.so")


def up_to_date(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return False
    t = os.path.getmtime(lib)
    return all(os.path.getmtime(d) <= t for d in DEPS)


def build(force: bool = False, verbose: bool = False, timeline: bool = False) -> str:
    lib = LIB_TIMELINE if timeline else LIB
    if not force and up_to_date(lib):
        return lib
    cmd = [nvcc_path(), *NVCC_FLAGS, *(["-DATTN_TIMELINE"] if timeline else []), "-o", lib + ".tmp", *SOURCES]
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError("nvcc failed:\n" + res.stdout + res.stderr)
    os.replace(lib + ".tmp", lib)
    if verbose:
        for line in (res.stdout + res.stderr).splitlines():
            if "registers" in line or "spill" in line or "Compiling entry" in line:
                print(line)
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True, timeline="--timeline" in sys.argv))
