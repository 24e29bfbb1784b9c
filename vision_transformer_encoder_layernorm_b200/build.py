"""Builds libvit.so in-tree for sm_100a with nvcc (no GPU needed).

    python vision_transformer_encoder_layernorm_b200/build.py [--force]

The shared library is written next to this file; the CUDA runtime is linked
statically, the driver API (cuTensorMapEncodeTiled) is resolved at run time
through cudaGetDriverEntryPoint, so libvit.so depends on libcuda only.
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libvit.so")
INCLUDE = os.path.join(os.path.dirname(HERE), "include")

SOURCES = ["vit_api.cu", "k_rows.cu", "k_simt.cu", "k_gemm_tc.cu", "k_attn_tc.cu", "k_embed.cu", "k_mx8.cu"]
FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-lineinfo", "-O3", "-std=c++17",
    "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
    "--expt-relaxed-constexpr",
]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    deps = [os.path.join(CSRC, f) for f in os.listdir(CSRC)]
    deps += [os.path.join(INCLUDE, f) for f in os.listdir(INCLUDE)]
    deps.append(os.path.abspath(__file__))
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, verbose: bool = False, extra=()) -> str:
    """Compiles every CUDA source into libvit.so (skipped when up to date)."""
    if not force and not _stale():
        return LIB
    tmp_dir = os.path.join(HERE, "_build")
    os.makedirs(tmp_dir, exist_ok=True)
    objs, cmds = [], []
    for src in SOURCES:
        obj = os.path.join(tmp_dir, src.replace(".cu", ".o"))
        cmds.append([nvcc(), *FLAGS, *extra, "-I", INCLUDE, "-c", os.path.join(CSRC, src),
                     "-o", obj])
        objs.append(obj)
    procs = []
    for cmd in cmds:
        if verbose:
            print(" ".join(cmd), flush=True)
        procs.append(subprocess.Popen(cmd))
    failed = [c for c, p in zip(cmds, procs) if p.wait() != 0]
    if failed:
        raise RuntimeError("nvcc failed: " + " ".join(failed[0]))
    out_tmp = LIB + ".tmp"
    cmd = [nvcc(), "-gencode", "arch=compute_100a,code=sm_100a", "-shared", "-o", out_tmp, *objs,
           "-Xcompiler", "-fPIC"]
    if verbose:
        print(" ".join(cmd), flush=True)
    subprocess.run(cmd, check=True)
    os.replace(out_tmp, LIB)
    return LIB


if __name__ == "__main__":
    args = sys.argv[1:]
    extra = []
    if "--ptxas-v" in args:
        extra = ["-Xptxas", "-v"]
    print(build(force="--force" in args or bool(extra), verbose=True, extra=extra))
