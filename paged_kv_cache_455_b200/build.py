"""Builds libpa.so (sm_100a) in-tree with nvcc.

    python -m paged_kv_cache_455_b200.build [--force] [--verbose]

The library links the CUDA runtime statically, so it loads on a machine
without a GPU driver (nothing CUDA runs until a kernel is launched).
"""
from __future__ import annotations

import argparse
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libpa.so")
SOURCES = [os.path.join(CSRC, f) for f in
           ("pa.cu", "pa_inst_f32.cu", "pa_inst_bf16.cu", "pa_inst_bf16_simt.cu",
            "pa_inst_fp8.cu", "pa_inst_prefill.cu")]
DEPS = SOURCES + [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith(".cuh")] + \
    [os.path.join(INCLUDE, f) for f in os.listdir(INCLUDE) if f.endswith(".h")]
OBJ_DIR = os.path.join(PKG, "_build")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
COMPILE_FLAGS = ARCH + ["-lineinfo", "-O3", "-std=c++17", "-Xcompiler", "-fPIC",
                        "--expt-relaxed-constexpr"]
LINK_FLAGS = ARCH + ["-shared", "-cudart", "static"]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if cand and (os.path.sep not in cand or os.path.exists(cand)):
            return cand
    return "nvcc"


def up_to_date() -> bool:
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    return all(os.path.getmtime(d) <= t for d in DEPS)


def build(force: bool = False, verbose: bool = False, extra=(), out: str = LIB) -> str:
    """Compiles every translation unit in parallel, then links libpa.so."""
    if not force and out == LIB and up_to_date():
        return out
    os.makedirs(OBJ_DIR, exist_ok=True)
    tag = "%d" % os.getpid()
    objs, procs = [], []
    for src in SOURCES:
        obj = os.path.join(OBJ_DIR, os.path.basename(src) + "." + tag + ".o")
        cmd = [nvcc(), *COMPILE_FLAGS, *extra, "-I", INCLUDE, "-c", "-o", obj, src]
        if verbose:
            cmd.insert(1, "-Xptxas=-v")
            print(" ".join(cmd), file=sys.stderr)
        procs.append(subprocess.Popen(cmd))
        objs.append(obj)
    failed = [p.args[-1] for p in procs if p.wait() != 0]
    if failed:
        raise RuntimeError("nvcc failed on " + ", ".join(failed))
    tmp = out + ".tmp" + tag
    subprocess.check_call([nvcc(), *LINK_FLAGS, "-o", tmp, *objs])
    os.replace(tmp, out)
    for o in objs:
        os.remove(o)
    return out


def main(argv=None) -> None:
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose", action="store_true", help="print ptxas register/smem use")
    a = ap.parse_args(argv)
    print(build(force=a.force, verbose=a.verbose))


if __name__ == "__main__":
    main()
