"""Build ``libflashprefill.so`` in-tree with nvcc for sm_100a (B200).

Usage: python -m block_sparse_long_blocks_b200.build [--verbose-ptxas]

Compiles each ``csrc/*.cu`` to an object (in parallel) and links one shared
library with the CUDA runtime linked statically, so the library depends only on
the driver. The build is skipped when the library is newer than every source.

``build_variant(name, defines)`` builds the same sources with extra
preprocessor definitions into ``libflashprefill_<name>.so`` (objects in
``_build_<name>/``); the tests use one with a microsecond pipeline-wait limit
(``short_wait``) to drive the kernels' abort path.
"""
from __future__ import annotations

import argparse
import concurrent.futures as cf
import glob
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD = os.path.join(PKG, "_build")
LIB = os.path.join(PKG, "libflashprefill.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=default",
         "--expt-relaxed-constexpr", "-I", INCLUDE, "-I", CSRC]


def nvcc() -> str:
    path = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(path):
        raise RuntimeError("nvcc not found")
    return path


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def deps():
    return sources() + sorted(glob.glob(os.path.join(CSRC, "*.cuh"))) + [os.path.join(INCLUDE, "flashprefill.h")]


# Variants built by __graft_entry__.build() next to the library: name -> defines.
VARIANTS = {"short_wait": {"FP_WAIT_LIMIT_NS": "500ull"}}


def variant_path(name: str) -> str:
    return os.path.join(PKG, f"libflashprefill_{name}.so")


def up_to_date(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return False
    t = os.path.getmtime(lib)
    return all(os.path.getmtime(p) <= t for p in deps() + [os.path.abspath(__file__)])


def _compile(src: str, verbose_ptxas: bool, build_dir: str = BUILD, defines=None) -> tuple:
    obj = os.path.join(build_dir, os.path.basename(src).replace(".cu", ".o"))
    cmd = [nvcc(), *ARCH, *FLAGS, *[f"-D{k}={v}" for k, v in (defines or {}).items()], "-c", src, "-o", obj]
    if verbose_ptxas:
        cmd += ["-Xptxas", "-v"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    return obj, r.returncode, r.stdout + r.stderr


def build_variant(name: str, defines=None, force: bool = False, quiet: bool = True) -> str:
    """The library built with extra preprocessor definitions (default: VARIANTS[name])."""
    defines = VARIANTS[name] if defines is None else defines
    return build(force=force, quiet=quiet, lib=variant_path(name), build_dir=os.path.join(PKG, f"_build_{name}"),
                 defines=defines)


def build(force: bool = False, verbose_ptxas: bool = False, quiet: bool = False, lib: str = LIB,
          build_dir: str = BUILD, defines=None) -> str:
    if not force and up_to_date(lib):
        return lib
    os.makedirs(build_dir, exist_ok=True)
    srcs = sources()
    with cf.ThreadPoolExecutor(max_workers=min(8, len(srcs))) as ex:
        results = list(ex.map(lambda s: _compile(s, verbose_ptxas, build_dir, defines), srcs))
    for obj, rc, out in results:
        if rc != 0:
            raise RuntimeError(f"nvcc failed for {obj}:\n{out}")
        if out.strip() and (verbose_ptxas or not quiet):
            print(out, file=sys.stderr)
    tmp = lib + ".tmp"
    cmd = [nvcc(), *ARCH, "-shared", "-o", tmp, *[o for o, _, _ in results], "-ldl"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"link failed:\n{r.stdout}{r.stderr}")
    os.replace(tmp, lib)
    return lib


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose-ptxas", action="store_true")
    a = ap.parse_args()
    print(build(force=a.force, verbose_ptxas=a.verbose_ptxas))


if __name__ == "__main__":
    main()
