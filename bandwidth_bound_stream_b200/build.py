"""In-tree build of the native libraries (run by ``__graft_entry__.build()``).

* ``libkie.so``  : the decode engine, CUDA for sm_100a only (nvcc cross-compiles without a GPU).
* ``libsynth.so``: the seeded input generator (plain C, OpenMP).
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
ROOT = os.path.dirname(HERE)
INCLUDE = os.path.join(ROOT, "include")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]

KIE_SOURCES = ["kie_engine.cu", "kie_b1.cu", "kie_mr.cu", "kie_attn.cu", "kie_fp8.cu"]
# build variants of the engine library: the product ("") and two diagnostic builds, each its own
# file (selected at import by KIE_VARIANT): "debug" checks the index of every kernel write to
# global memory (recording an error instead of writing) and keeps guard words around every
# engine buffer, which the host checks after each command; "profile" times the GEMV consumer
# warps per chunk
VARIANTS = {"": [], "debug": ["-DKIE_CHECK_BOUNDS"], "profile": ["-DKIE_PROFILE_GEMV"]}
KIE_HEADERS = ["kie_device.cuh", "kie_internal.h", "kie_attn.cuh", "kie_sample.cuh"]


def _run(cmd):
    res = subprocess.run(cmd, stdout=subprocess.PIPE, stderr=subprocess.STDOUT, text=True)
    if res.returncode != 0:
        sys.stderr.write(res.stdout)
        raise RuntimeError("build failed: " + " ".join(cmd))
    return res.stdout


def _stale(target, deps):
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(d) > t for d in deps if os.path.exists(d))


def build_synth(force: bool = False) -> str:
    src = os.path.join(CSRC, "synth.c")
    out = os.path.join(HERE, "libsynth.so")
    if force or _stale(out, [src]):
        _run(["gcc", "-O2", "-fPIC", "-shared", "-fopenmp", "-o", out, src, "-lm"])
    return out


def lib_name(variant: str = "") -> str:
    if variant not in VARIANTS:
        raise ValueError(f"unknown build variant {variant!r} (one of {sorted(VARIANTS)})")
    return "libkie.so" if not variant else f"libkie_{variant}.so"


def build_kie(force: bool = False, verbose_ptxas: bool = False, variant: str = "") -> str:
    out = os.path.join(HERE, lib_name(variant))
    srcs = [os.path.join(CSRC, s) for s in KIE_SOURCES]
    deps = srcs + [os.path.join(CSRC, h) for h in KIE_HEADERS] + [os.path.join(INCLUDE, "kie.h")]
    if not (force or verbose_ptxas or _stale(out, deps)):
        return out
    objdir = os.path.join(HERE, "_build" + (f"_{variant}" if variant else ""))
    os.makedirs(objdir, exist_ok=True)
    objs, procs = [], []
    for s in srcs:
        o = os.path.join(objdir, os.path.basename(s) + ".o")
        cmd = [NVCC, *ARCH, "-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-rdc=false",
               "-I", INCLUDE, "-I", CSRC, *VARIANTS[variant], "-c", s, "-o", o]
        if verbose_ptxas:
            cmd.insert(1, "-Xptxas=-v")
        procs.append((cmd, subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.STDOUT, text=True)))
        objs.append(o)
    failed = False
    for cmd, pr in procs:
        log, _ = pr.communicate()
        if pr.returncode != 0:
            sys.stderr.write(log)
            failed = True
        elif verbose_ptxas:
            sys.stdout.write(log)
    if failed:
        raise RuntimeError("nvcc failed")
    _run([NVCC, *ARCH, "-shared", "-o", out, *objs])  # the CUDA runtime only (no driver library at link time)
    return out


def build_all(force: bool = False) -> None:
    build_synth(force)
    build_kie(force)


if __name__ == "__main__":
    build_all(force="--force" in sys.argv)
    if "--ptxas" in sys.argv:
        build_kie(verbose_ptxas=True)
    if "--variant" in sys.argv:  # e.g. --variant profile
        build_kie(force="--force" in sys.argv, variant=sys.argv[sys.argv.index("--variant") + 1])
