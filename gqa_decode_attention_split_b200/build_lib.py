"""Build libfadecode.so (sm_100a) in-tree with nvcc.

Every .cu file under csrc/ is compiled in parallel with
``-gencode arch=compute_100a,code=sm_100a -O3 -lineinfo`` and linked into
gqa_decode_attention_split_b200/lib/libfadecode.so (CUDA runtime linked
statically; the driver API is reached through cudaGetDriverEntryPoint, so the
library loads on hosts without a GPU driver and fails only when used).

Usage: python -m gqa_decode_attention_split_b200.build_lib [--force] [-v]
"""
from __future__ import annotations

import argparse
import glob
import os
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
BUILD = os.path.join(PKG, "_build")
LIB = os.path.join(PKG, "lib", "libfadecode.so")

NVCC_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17",
              "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
              "-I" + os.path.join(ROOT, "include")]


def _nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if cand and (os.path.isabs(cand) and os.path.exists(cand) or not os.path.isabs(cand)):
            return cand
    return "nvcc"


def _sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _deps():
    return (sorted(glob.glob(os.path.join(CSRC, "*.cu*"))) + sorted(glob.glob(os.path.join(CSRC, "*.h")))
            + [os.path.join(ROOT, "include", "fadecode.h"), os.path.abspath(__file__)])


def up_to_date() -> bool:
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    return all(os.path.getmtime(p) <= t for p in _deps())


def build(force: bool = False, verbose: bool = False, ptxas_info: bool = False,
          checks: bool = False, out: str = None, defines=()) -> str:
    """Compile and link.  checks=True builds the self-checking variant
    (-DFA_CHECKS: range/alignment checks on every shared-memory read, bulk
    copy destination and global write, reported through the status word)."""
    lib = out or LIB
    if not force and out is None and not checks and not defines and up_to_date():
        return LIB
    tag = ("_checks" if checks else "") + "".join("_" + d.replace("=", "") for d in defines)
    build_dir = BUILD + tag
    os.makedirs(build_dir, exist_ok=True)
    os.makedirs(os.path.dirname(lib), exist_ok=True)
    nvcc = _nvcc()
    extra = (["-DFA_CHECKS"] if checks else []) + ["-D" + d for d in defines]

    def compile_one(src):
        obj = os.path.join(build_dir, os.path.basename(src) + ".o")
        cmd = [nvcc, *NVCC_FLAGS, *extra, "-c", src, "-o", obj]
        if ptxas_info:
            cmd += ["-Xptxas", "-v"]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"nvcc failed for {src}:\n{r.stdout}\n{r.stderr}")
        if verbose or ptxas_info:
            sys.stderr.write(r.stderr)
        return obj

    srcs = _sources()
    with ThreadPoolExecutor(max_workers=min(len(srcs), os.cpu_count() or 4)) as ex:
        objs = list(ex.map(compile_one, srcs))
    tmp = lib + f".tmp{os.getpid()}"
    cmd = [nvcc, "-shared", "-gencode", "arch=compute_100a,code=sm_100a", "-o", tmp, *objs,
           "-Xcompiler", "-fPIC"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
    os.replace(tmp, lib)
    return lib


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("-v", "--verbose", action="store_true")
    ap.add_argument("--ptxas-info", action="store_true")
    ap.add_argument("--checks", action="store_true", help="self-checking build (-DFA_CHECKS)")
    ap.add_argument("--out", default=None, help="output path (default: lib/libfadecode.so)")
    ap.add_argument("-D", dest="defines", action="append", default=[],
                    help="extra preprocessor definition, e.g. -D FA_TILE_BYTES=8192")
    args = ap.parse_args()
    print(build(force=args.force, verbose=args.verbose, ptxas_info=args.ptxas_info,
                checks=args.checks, out=args.out, defines=tuple(args.defines)))


if __name__ == "__main__":
    main()
