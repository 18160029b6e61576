"""Build libjetlong.so in-tree with nvcc for sm_100a (B200).

``python -m rope_context_extension_sm_b200.build`` compiles the single
translation unit ``csrc/jetlong.cu`` (which includes the kernel headers) into
``rope_context_extension_sm_b200/libjetlong.so``.  nvcc cross-compiles, so this
also works on a machine without a GPU.
"""
from __future__ import annotations

import glob
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libjetlong.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

FLAGS = [
    "-O3", "-std=c++17", "-lineinfo",
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-Xcompiler", "-fPIC,-O2,-Wall",
    "--expt-relaxed-constexpr",
    "-shared",
]


def sources() -> list[str]:
    return sorted(glob.glob(os.path.join(CSRC, "*")) + [os.path.join(ROOT, "include", "jetlong.h")])


# The debug-bounds build: the same library with device-side index checks compiled in
# (-DJL_DEBUG_BOUNDS; each failed check is recorded in the status word, see jl_device.cuh).
BOUNDS_LIB = os.path.join(HERE, "libjetlong_bounds.so")


def build(force: bool = False, verbose: bool = False, extra: list[str] | None = None, out: str | None = None) -> str:
    out = out or LIB
    newest = max(os.path.getmtime(p) for p in sources())
    if not force and os.path.exists(out) and os.path.getmtime(out) >= newest and (not extra or out != LIB):
        return out
    cmd = [NVCC, *FLAGS, *(extra or []), "-I", os.path.join(ROOT, "include"), "-I", CSRC,
           "-o", out, os.path.join(CSRC, "jetlong.cu")]
    if verbose:
        print(" ".join(cmd), file=sys.stderr)
    subprocess.run(cmd, check=True)
    return out


def build_bounds(force: bool = False) -> str:
    """Build libjetlong_bounds.so (the debug-bounds variant) in-tree."""
    return build(force=force, extra=["-DJL_DEBUG_BOUNDS"], out=BOUNDS_LIB)


# The single-launch decode build: the last split CTA of each (entry, KV head) merges
# the partials instead of a second kernel (-DJL_DECODE_LAST_CTA_MERGE=1).
LAST_CTA_LIB = os.path.join(HERE, "libjetlong_lastcta.so")


def build_last_cta(force: bool = False) -> str:
    """Build libjetlong_lastcta.so (the single-launch decode variant) in-tree."""
    return build(force=force, extra=["-DJL_DECODE_LAST_CTA_MERGE=1"], out=LAST_CTA_LIB)


if __name__ == "__main__":
    build(force=True, verbose=True, extra=sys.argv[1:])
    print(LIB)
