"""Build the TACT-KV CUDA library in-tree: csrc/*.cu -> dct_transform_coding_b200/libtactkv.so.

Runs the two generators (pencil DCT code, Lloyd-Max codebooks), compiles the translation units
in parallel with nvcc for sm_100a only, and links the shared library.  No GPU is needed.
"""
from __future__ import annotations

import concurrent.futures as cf
import os
import subprocess
import sys
import time

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
ROOT = os.path.dirname(HERE)
LIB = os.path.join(HERE, "libtactkv.so")
OBJ = os.path.join(ROOT, "_build")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17",
         "-Xcompiler", "-fPIC", "-I", os.path.join(ROOT, "include"), "-I", CSRC]

# (object name, source, extra defines)
UNITS = [
    ("axis_s_16", "axis_s.cu", ["-DTACTKV_CLASS=16"]),
    ("axis_s_32", "axis_s.cu", ["-DTACTKV_CLASS=32"]),
    ("axis_s_64", "axis_s.cu", ["-DTACTKV_CLASS=64"]),
    ("axis_hw_16_16", "axis_hw.cu", ["-DTACTKV_HCLASS=16", "-DTACTKV_WCLASS=16"]),
    ("axis_hw_16_32", "axis_hw.cu", ["-DTACTKV_HCLASS=16", "-DTACTKV_WCLASS=32"]),
    ("axis_hw_32_16", "axis_hw.cu", ["-DTACTKV_HCLASS=32", "-DTACTKV_WCLASS=16"]),
    ("axis_hw_32_32", "axis_hw.cu", ["-DTACTKV_HCLASS=32", "-DTACTKV_WCLASS=32"]),
    ("fused_8", "fused.cu", ["-DTACTKV_FUSED_S=8"]),
    ("fused_16", "fused.cu", ["-DTACTKV_FUSED_S=16"]),
    ("fused_32", "fused.cu", ["-DTACTKV_FUSED_S=32"]),
    ("fused_64", "fused.cu", ["-DTACTKV_FUSED_S=64"]),
    ("fused_inv_16", "fused_inv.cu", ["-DTACTKV_FUSED_S=16"]),
    ("fused_inv_32", "fused_inv.cu", ["-DTACTKV_FUSED_S=32"]),
    ("fused_inv_64", "fused_inv.cu", ["-DTACTKV_FUSED_S=64"]),
    ("allocate", "allocate.cu", []),
    ("attention", "attention.cu", []),
    ("pack", "pack.cu", []),
    ("tactkv", "tactkv.cu", []),
]


def _compile(name, src, defs, ptxas_info):
    out = os.path.join(OBJ, name + ".o")
    cmd = [NVCC, *FLAGS, *defs, "-c", os.path.join(CSRC, src), "-o", out]
    if ptxas_info:
        cmd[1:1] = ["-Xptxas", "-v"]
    t = time.time()
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError(f"nvcc failed for {name}:\n{res.stdout}{res.stderr}")
    return out, time.time() - t, res.stdout + res.stderr


def build(verbose: bool = False, ptxas_info: bool = False, jobs: int = 0) -> str:
    for gen in ("gen_dct.py", "gen_tables.py", "gen_mma_tables.py"):
        subprocess.run([sys.executable, os.path.join(CSRC, gen)], check=True,
                       stdout=None if verbose else subprocess.DEVNULL)
    os.makedirs(OBJ, exist_ok=True)
    jobs = jobs or min(len(UNITS), os.cpu_count() or 1)
    with cf.ThreadPoolExecutor(jobs) as ex:
        results = list(ex.map(lambda u: _compile(*u, ptxas_info), UNITS))
    for (name, _, _), (_, dt, log) in zip(UNITS, results):
        if verbose:
            print(f"[build] {name}: {dt:.1f}s")
        if ptxas_info and log:
            sys.stdout.write(log)
    tmp = LIB + ".tmp"
    res = subprocess.run([NVCC, "-gencode", "arch=compute_100a,code=sm_100a", "-shared",
                          *[r[0] for r in results], "-o", tmp], capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError("link failed:\n" + res.stdout + res.stderr)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    build(verbose=True, ptxas_info="-v" in sys.argv)
    print("built", LIB)
