"""Build libkda.so in-tree with nvcc for sm_100a.

    python -m chunked_kda_prefill_b200.build [--force] [--define NAME=VALUE ...]

Compiles every ``csrc/*.cu`` and ``csrc/*.cpp`` to objects under ``_build/`` (in parallel)
and links ``chunked_kda_prefill_b200/libkda.so`` with the CUDA runtime linked statically, so
the library loads on a machine without a GPU (its host entry points work there).

``--define`` builds a variant instead (for example ``KDA_STATE_LO=0``, the state operand without
its bf16 remainder, or ``KDA_PHASE_TIMING=1``, per-phase clock stamps for
``kda_forward_debug``): objects under ``_build_<tag>/`` and ``libkda_<tag>.so``, where
``<tag>`` joins the definitions; load it with ``KDA_LIB=<path>``.
"""
from __future__ import annotations

import glob
import os
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

PKG = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(PKG, "csrc")
BUILD = os.path.join(PKG, "_build")
LIB = os.path.join(PKG, "libkda.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
COMMON = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC,-fvisibility=hidden",
          "-I", os.path.join(PKG, "..", "include")]


def _sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cpp")))


def _headers():
    return (glob.glob(os.path.join(CSRC, "*.h")) + glob.glob(os.path.join(CSRC, "*.cuh"))
            + glob.glob(os.path.join(PKG, "..", "include", "*.h")))


def _stale(target, deps):
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(d) > t for d in deps)


def _compile(src, verbose, build_dir=BUILD, defines=()):
    obj = os.path.join(build_dir, os.path.basename(src) + ".o")
    if not _stale(obj, [src] + _headers()):
        return obj
    cmd = [NVCC] + ARCH + COMMON + [f"-D{d}" for d in defines] + ["-c", src, "-o", obj + ".tmp"]
    if src.endswith(".cu") and verbose:
        cmd += ["-Xptxas", "-v"]
    if src.endswith(".cpp"):
        cmd += ["-x", "cu"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed for {src}:\n{r.stdout}\n{r.stderr}")
    if verbose and r.stderr:
        sys.stderr.write(r.stderr)
    os.replace(obj + ".tmp", obj)
    return obj


def variant_tag(defines) -> str:
    return "_".join(d.replace("=", "").lower() for d in sorted(defines))


def build(force: bool = False, verbose: bool = False, defines=()) -> str:
    defines = tuple(defines)
    build_dir = BUILD if not defines else BUILD + "_" + variant_tag(defines)
    lib = LIB if not defines else os.path.join(PKG, f"libkda_{variant_tag(defines)}.so")
    os.makedirs(build_dir, exist_ok=True)
    srcs = _sources()
    if force:
        for f in glob.glob(os.path.join(build_dir, "*.o")):
            os.remove(f)
    with ThreadPoolExecutor(max_workers=min(8, len(srcs))) as ex:
        objs = list(ex.map(lambda s: _compile(s, verbose, build_dir, defines), srcs))
    if force or _stale(lib, objs):
        tmp = lib + f".tmp{os.getpid()}"
        # no -lcuda: driver entry points are resolved at run time through the runtime, so
        # the library also loads on a host without the driver
        cmd = [NVCC] + ARCH + ["-shared", "-cudart", "static", "-o", tmp] + objs
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
        os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    import argparse

    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose", action="store_true")
    ap.add_argument("--define", action="append", default=[])
    a = ap.parse_args()
    print(build(force=a.force, verbose=a.verbose, defines=a.define))
