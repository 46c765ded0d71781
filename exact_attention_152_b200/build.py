"""Build the in-tree CUDA libraries for sm_100a with nvcc.

    python -m exact_attention_152_b200.build [--force]

Produces, next to this file:
  libattn.so         the product: attn_fwd and friends (include/attn.h)
  libattn_blocks.so  building-block checks used by the tests (include/attn_blocks.h)
The CUDA runtime is linked statically, so the libraries only need the driver.
ptxas resource reports (registers, spills, shared memory) go to _build/*.ptxas.txt.
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
INCLUDE = os.path.join(ROOT, "include")
BUILD = os.path.join(HERE, "_build")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
TARGETS = {
    "libattn.so": ["attn_fwd.cu", "attn_bwd.cu"],
    "libattn_blocks.so": ["blocks.cu"],
}


def nvcc() -> str:
    path = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(path):
        raise RuntimeError("nvcc not found")
    return path


def _deps():
    out = []
    for d in (CSRC, INCLUDE):
        for f in os.listdir(d):
            if f.endswith((".cu", ".cuh", ".h")):
                out.append(os.path.join(d, f))
    return out


def _stale(target: str, sources) -> bool:
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(s) > t for s in list(sources) + _deps())


def build(force: bool = False, verbose: bool = False) -> list[str]:
    os.makedirs(BUILD, exist_ok=True)
    procs = []
    for lib, srcs in TARGETS.items():
        target = os.path.join(HERE, lib)
        sources = [os.path.join(CSRC, s) for s in srcs]
        if not force and not _stale(target, sources):
            continue
        tmp = os.path.join(BUILD, lib + f".tmp{os.getpid()}")
        cmd = [nvcc(), *ARCH, "-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-shared",
               "-cudart", "static", "-Xptxas", "-v", "-I", INCLUDE, "-I", CSRC,
               "-o", tmp, *sources]
        log = open(os.path.join(BUILD, lib + ".ptxas.txt"), "w")
        procs.append((lib, target, tmp, cmd, subprocess.Popen(cmd, stdout=log, stderr=subprocess.STDOUT), log))
    built = []
    errors = []
    for lib, target, tmp, cmd, p, log in procs:
        rc = p.wait()
        log.close()
        if rc != 0:
            errors.append(f"{lib}: nvcc exited {rc}; see {log.name}\n" + open(log.name).read()[-4000:])
            continue
        os.replace(tmp, target)
        built.append(target)
        if verbose:
            print(f"built {target}")
    if errors:
        raise RuntimeError("\n".join(errors))
    return built


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    a = ap.parse_args(argv)
    build(force=a.force, verbose=True)


if __name__ == "__main__":
    sys.exit(main())
