"""Build libpagedattn.so in-tree with nvcc for sm_100a (B200).

    python -m paged_kv_cache_416_b200.build [--force] [--verbose]

nvcc cross-compiles without a GPU, so this runs on any machine with the CUDA
toolkit.  The library lands next to this file, where the binding loads it.
"""

from __future__ import annotations

import argparse
import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
HEADER = os.path.join(ROOT, "include", "pagedattn.h")
LIB = os.path.join(HERE, "libpagedattn.so")
MAIN_SRC = os.path.join(CSRC, "pagedattn.cu")

ARCH_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a"]
CXX_FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC,-O2", "-shared"]


def nvcc_path() -> str:
    p = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(p):
        raise RuntimeError("nvcc not found: the CUDA toolkit is needed to build libpagedattn.so")
    return p


def sources():
    out = [HEADER]
    for f in sorted(os.listdir(CSRC)):
        if f.endswith((".cu", ".cuh", ".h")):
            out.append(os.path.join(CSRC, f))
    return out


def up_to_date() -> bool:
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    return all(os.path.getmtime(s) <= t for s in sources())


def build(force: bool = False, verbose: bool = False, extra_flags=None, out=None) -> str:
    """Compile the library unless it is newer than every source; returns its
    path.  With `out` (a test build with its own `extra_flags`, e.g. -D
    defines), always compile, to that path instead of the package's library."""
    target = LIB if out is None else str(out)
    if out is None and not force and up_to_date():
        return LIB
    cmd = [nvcc_path(), *ARCH_FLAGS, *CXX_FLAGS, *(extra_flags or []), "-o", target + ".tmp", MAIN_SRC]
    if verbose:
        print(" ".join(cmd), flush=True)
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed ({r.returncode}):\n{r.stdout}\n{r.stderr}")
    if verbose and (r.stdout or r.stderr):
        print(r.stdout, r.stderr, file=sys.stderr)
    os.replace(target + ".tmp", target)
    return target


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__)
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose", action="store_true")
    a = ap.parse_args(argv)
    print(build(force=a.force, verbose=a.verbose))


if __name__ == "__main__":
    main()
