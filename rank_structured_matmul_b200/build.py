"""Build the DyRA CUDA library in-tree: rank_structured_matmul_b200/libdyra.so.

    python -m rank_structured_matmul_b200.build [--force] [-v] [--debug]

--debug builds the bounds-checked variant libdyra_debug.so instead (the same
sources compiled with DYRA_DEBUG: every direct global access of the kernels
is checked against its buffer, and one outside raises DYRA_STATUS_BOUNDS and
is skipped). The binding loads it when DYRA_DEBUG_LIB=1.

Compiles every .cu under csrc/ for sm_100a with nvcc (objects in _build/ at
the repository root) and links one shared library with the CUDA runtime
linked statically, so the library loads without a GPU present.
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
BUILD_DIR = os.path.join(ROOT, "_build")
LIB_PATH = os.path.join(HERE, "libdyra.so")
DEBUG_LIB_PATH = os.path.join(HERE, "libdyra_debug.so")

SOURCES = ["dyra_api.cu", "kernels_umma.cu", "kernels_simt.cu"]
ARCH_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ARCH_FLAGS + ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC",
                           "-Xptxas", "-warn-spills", "-I", INCLUDE, "-I", CSRC]


def nvcc() -> str:
    path = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(path):
        raise RuntimeError("nvcc not found")
    return path


def _headers():
    out = [os.path.join(INCLUDE, f) for f in os.listdir(INCLUDE) if f.endswith(".h")]
    out += [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".h", ".cuh"))]
    return out


def _stale(target: str, deps) -> bool:
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, verbose: bool = False, extra_flags=(), debug: bool = False) -> str:
    build_dir = os.path.join(BUILD_DIR, "debug") if debug else BUILD_DIR
    lib_path = DEBUG_LIB_PATH if debug else LIB_PATH
    extra_flags = list(extra_flags) + (["-DDYRA_DEBUG"] if debug else [])
    os.makedirs(build_dir, exist_ok=True)
    headers = _headers()
    objs, procs = [], []
    for src in SOURCES:
        s = os.path.join(CSRC, src)
        o = os.path.join(build_dir, src.replace(".cu", ".o"))
        objs.append(o)
        if force or _stale(o, [s] + headers):
            cmd = [nvcc()] + NVCC_FLAGS + list(extra_flags) + ["-c", s, "-o", o]
            if verbose:
                print(" ".join(cmd), flush=True)
            procs.append((src, subprocess.Popen(cmd, stdout=subprocess.PIPE,
                                                stderr=subprocess.STDOUT, text=True)))
    failed = []
    for src, p in procs:
        out, _ = p.communicate()
        if verbose or p.returncode != 0:
            sys.stdout.write(out)
        if p.returncode != 0:
            failed.append(src)
    if failed:
        raise RuntimeError("nvcc failed for " + ", ".join(failed))
    if force or procs or _stale(lib_path, objs):
        cmd = [nvcc()] + ARCH_FLAGS + ["-shared", "-cudart", "static", "-o", lib_path] + objs
        if verbose:
            print(" ".join(cmd), flush=True)
        subprocess.run(cmd, check=True)
    return lib_path


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("-v", "--verbose", action="store_true")
    ap.add_argument("--debug", action="store_true", help="the bounds-checked libdyra_debug.so")
    a = ap.parse_args(argv)
    print(build(force=a.force, verbose=a.verbose, debug=a.debug))


if __name__ == "__main__":
    main()
