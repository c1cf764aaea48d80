"""Builds libkdverify.so in-tree for sm_100a with nvcc (no JIT cache).

    python -m tree_speculative_decoding_kd_b200.build           # the library
    python -m tree_speculative_decoding_kd_b200.build --trace   # + libkdverify_trace.so

The trace build compiles the attention with -DKD_TRACE: the same kernel recording a
per-CTA timeline and wait counters of each launch (read by trace.py), plus the L2
delivery probes of csrc/kd_probe.cu.
"""
from __future__ import annotations

import concurrent.futures
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
OBJ = os.path.join(ROOT, "_build")
LIB = os.path.join(PKG, "libkdverify.so")
TRACE_LIB = os.path.join(PKG, "libkdverify_trace.so")

SOURCES = ["kd_tree.cu", "kd_attn_simt.cu", "kd_attn_tc.cu", "kd_argmax.cu", "kd_tree_build.cu"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "--expt-relaxed-constexpr",
         "-I" + INCLUDE, "-I" + CSRC]


def nvcc() -> str:
    for c in [os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"]:
        if c and os.path.exists(c):
            return c
    raise RuntimeError("nvcc not found")


def _compile(src: str, verbose: bool, extra=(), suffix: str = "") -> str:
    obj = os.path.join(OBJ, os.path.splitext(src)[0] + suffix + ".o")
    cmd = [nvcc(), *ARCH, *FLAGS, *extra, "-c", os.path.join(CSRC, src), "-o", obj]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed for {src}:\n{r.stdout}\n{r.stderr}")
    if verbose:
        sys.stderr.write(r.stderr)
    return obj


def build(verbose: bool = False, force: bool = False) -> str:
    """Compile every source (in parallel) and link libkdverify.so; returns its path."""
    os.makedirs(OBJ, exist_ok=True)
    deps = [os.path.join(CSRC, f) for f in os.listdir(CSRC)] + \
           [os.path.join(INCLUDE, f) for f in os.listdir(INCLUDE)] + [os.path.abspath(__file__)]
    if (not force and os.path.exists(LIB)
            and os.path.getmtime(LIB) >= max(os.path.getmtime(d) for d in deps)):
        return LIB
    with concurrent.futures.ThreadPoolExecutor(len(SOURCES)) as ex:
        objs = list(ex.map(lambda s: _compile(s, verbose), SOURCES))
    tmp = LIB + ".tmp"
    cmd = [nvcc(), *ARCH, "-shared", "-o", tmp, *objs, "-cudart", "static"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
    os.replace(tmp, LIB)
    return LIB


def build_trace(verbose: bool = False, force: bool = False) -> str:
    """libkdverify_trace.so: the library with the attention compiled with -DKD_TRACE."""
    lib = build(verbose)
    if not force and os.path.exists(TRACE_LIB) and os.path.getmtime(TRACE_LIB) >= os.path.getmtime(lib):
        return TRACE_LIB
    objs = [os.path.join(OBJ, os.path.splitext(s)[0] + ".o") for s in SOURCES if s != "kd_attn_tc.cu"]
    objs.append(_compile("kd_attn_tc.cu", verbose, ["-DKD_TRACE"], "_trace"))
    objs.append(_compile("kd_probe.cu", verbose, ["-DKD_TRACE"], "_trace"))     # delivery probes
    tmp = TRACE_LIB + ".tmp"
    r = subprocess.run([nvcc(), *ARCH, "-shared", "-o", tmp, *objs, "-cudart", "static"], capture_output=True,
                       text=True)
    if r.returncode != 0:
        raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
    os.replace(tmp, TRACE_LIB)
    return TRACE_LIB


if __name__ == "__main__":
    print(build(verbose="-v" in sys.argv, force=True))
    if "--trace" in sys.argv:
        print(build_trace(verbose="-v" in sys.argv, force=True))
