"""Build libarc_attn.so in-tree with nvcc for sm_100a (no -rdc, whole-program).

Separable compilation (-rdc) is left off on purpose: the FlashMLA build on the
TensorRT-LLM page ("FlashMLA without -rdc", ptxas table) showed -rdc adding
spill stores to the sm100 sparse kernels and doubling their time.  The build
also records ptxas's register / spill report next to the library, so a spill
in a hot kernel is visible without reading any compiled code.

Usage: python -m exact_attention_131_b200.build [--force]
"""
from __future__ import annotations

import os
import re
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libarc_attn.so")
PTXAS_LOG = os.path.join(HERE, "_ptxas_report.txt")
SOURCES = ["api.cu", "simple_kernels.cu", "attn_tc.cu", "attn_pair.cu", "sparse_tc.cu", "decode.cu", "merge.cu",
           "attn_bwd.cu"]
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17",
         "-Xcompiler", "-fPIC", "-Xptxas", "-v", "--expt-relaxed-constexpr"]


def _sources():
    return [os.path.join(CSRC, s) for s in SOURCES if os.path.exists(os.path.join(CSRC, s))]


def _stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    deps = _sources() + [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".cuh", ".h"))]
    deps.append(os.path.join(os.path.dirname(HERE), "include", "arc_attn.h"))
    return any(os.path.getmtime(d) > t for d in deps if os.path.exists(d))


def spill_report(text: str) -> list[str]:
    """Kernels whose ptxas report shows spill stores (the build gate)."""
    bad, cur = [], None
    for line in text.splitlines():
        m = re.search(r"Compiling entry function '([^']+)'", line)
        if m:
            cur = m.group(1)
        m = re.search(r"(\d+) bytes spill stores", line)
        if m and int(m.group(1)) > 0 and cur:
            bad.append(f"{cur}: {m.group(1)} bytes spill stores")
    return bad


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and not _stale():
        return LIB
    objs, log = [], []
    bdir = os.path.join(HERE, "_build")
    os.makedirs(bdir, exist_ok=True)
    for src in _sources():
        obj = os.path.join(bdir, os.path.basename(src) + ".o")
        cmd = [NVCC, *FLAGS, "-c", src, "-o", obj]
        r = subprocess.run(cmd, capture_output=True, text=True)
        log.append(r.stdout + r.stderr)
        if r.returncode != 0:
            sys.stderr.write(r.stdout + r.stderr)
            raise RuntimeError(f"nvcc failed on {os.path.basename(src)}")
        objs.append(obj)
    tmp = LIB + f".tmp{os.getpid()}"
    r = subprocess.run([NVCC, "-gencode", "arch=compute_100a,code=sm_100a", "-shared", "-Xcompiler", "-fPIC",
                        *objs, "-o", tmp], capture_output=True, text=True)
    if r.returncode != 0:
        sys.stderr.write(r.stdout + r.stderr)
        raise RuntimeError("nvcc link failed")
    os.replace(tmp, LIB)
    text = "\n".join(log)
    with open(PTXAS_LOG, "w") as f:
        f.write(text)
    bad = spill_report(text)
    if bad:
        raise RuntimeError("spill stores in hot kernels:\n" + "\n".join(bad))
    if verbose:
        print(text)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
