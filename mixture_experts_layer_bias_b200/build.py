"""Build the MoE layer library (libmoe_b200.so) in-tree with nvcc for sm_100a.

    python -m mixture_experts_layer_bias_b200.build [--force] [-j N]

Objects go to ``_build/`` at the repository root; the shared library lands
next to this file so it ships with the package.  Only sources newer than their
object are recompiled.

A second library, libmoe_b200_testhooks.so, is linked from the same objects
except the GEMM launch file, which is compiled with MOE_B200_TEST_HOOKS: it
adds the failure-detection test hook (moe_test_stall_gemms) that the product
library does not contain.  Only the failure-detection test loads it.

A third, libmoe_b200_debug.so, is the guard build: the permutation and
combine files are compiled with MOE_DEBUG, which adds a check kernel after
every permutation (counts, offsets, row_of_slot and token_of_row agree) and a
range check of every row the combine reads; a violation sets
MOE_STATUS_DEBUG_CHECK in the status block.  Its results are otherwise those
of the product library.
"""
from __future__ import annotations

import argparse
import concurrent.futures as cf
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD = os.path.join(ROOT, "_build")
LIB = os.path.join(PKG, "libmoe_b200.so")
TEST_HOOKS_LIB = os.path.join(PKG, "libmoe_b200_testhooks.so")
TEST_HOOKS_SOURCE = "gemm_dispatch.cu"
DEBUG_LIB = os.path.join(PKG, "libmoe_b200_debug.so")
DEBUG_SOURCES = ("permute.cu", "combine.cu")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ARCH + ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC,-O2", "--expt-relaxed-constexpr",
                     "-I", INCLUDE, "-I", CSRC]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def sources():
    return sorted(os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith(".cu"))


def headers():
    hs = [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".cuh", ".h"))]
    hs.append(os.path.join(INCLUDE, "moe.h"))
    return hs


def _compile(src: str, force: bool, extra, build_dir: str = BUILD) -> str:
    obj = os.path.join(build_dir, os.path.basename(src) + ".o")
    newest_dep = max(os.path.getmtime(p) for p in [src] + headers())
    if not force and os.path.exists(obj) and os.path.getmtime(obj) >= newest_dep:
        return obj
    cmd = [nvcc()] + NVCC_FLAGS + list(extra) + ["-c", src, "-o", obj]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed for {src}:\n{r.stdout}\n{r.stderr}")
    return obj


def _link(objs, out: str, force: bool) -> str:
    if force or not os.path.exists(out) or os.path.getmtime(out) < max(os.path.getmtime(o) for o in objs):
        tmp = out + ".tmp"
        cmd = [nvcc()] + ARCH + ["-shared", "-o", tmp] + objs
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
        os.replace(tmp, out)
    return out


def build(force: bool = False, jobs: int = 8, extra=(), out: str = LIB, build_dir: str = BUILD,
          test_hooks: bool = True) -> str:
    """Compile every source (extra nvcc flags, e.g. -D tuning macros, go to
    all of them) into build_dir and link `out`; with test_hooks also link the
    test-hook and guard (MOE_DEBUG) libraries next to the product one."""
    os.makedirs(build_dir, exist_ok=True)
    srcs = sources()
    with cf.ThreadPoolExecutor(max_workers=jobs) as ex:
        objs = list(ex.map(lambda s: _compile(s, force, extra, build_dir), srcs))
    _link(objs, out, force)
    if test_hooks and out == LIB:
        hook_dir = os.path.join(build_dir, "testhooks")
        os.makedirs(hook_dir, exist_ok=True)
        hook_src = os.path.join(CSRC, TEST_HOOKS_SOURCE)
        hook_obj = _compile(hook_src, force, list(extra) + ["-DMOE_B200_TEST_HOOKS"], hook_dir)
        objs_h = [hook_obj if os.path.basename(o) == TEST_HOOKS_SOURCE + ".o" else o for o in objs]
        _link(objs_h, TEST_HOOKS_LIB, force)
        debug_dir = os.path.join(build_dir, "debug")
        os.makedirs(debug_dir, exist_ok=True)
        dbg = {src: _compile(os.path.join(CSRC, src), force, list(extra) + ["-DMOE_DEBUG"], debug_dir)
               for src in DEBUG_SOURCES}
        objs_d = [dbg.get(os.path.basename(o)[:-2], o) for o in objs]
        _link(objs_d, DEBUG_LIB, force)
    return out


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("-j", type=int, default=8)
    ap.add_argument("--ptxas-verbose", action="store_true")
    ap.add_argument("-D", dest="defines", action="append", default=[], help="extra -D macro for every source")
    ap.add_argument("--out", default=LIB, help="library path (variants go elsewhere)")
    ap.add_argument("--build-dir", default=BUILD)
    a = ap.parse_args(argv)
    extra = ["-Xptxas", "-v"] if a.ptxas_verbose else []
    extra += ["-D" + d for d in a.defines]
    print(build(force=a.force or a.ptxas_verbose or bool(a.defines), jobs=a.j, extra=extra, out=a.out,
                build_dir=a.build_dir))


if __name__ == "__main__":
    sys.exit(main())
