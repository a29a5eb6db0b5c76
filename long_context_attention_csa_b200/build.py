"""Builds libcsa.so in-tree from csrc/*.cu for sm_100a with nvcc.

Usage: python -m long_context_attention_csa_b200.build [--force]
"""
from __future__ import annotations

import glob
import os
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
BUILD = os.path.join(PKG, "_build")
LIB = os.path.join(PKG, "libcsa.so")

NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "-Xcompiler", "-Wall",
         "--expt-relaxed-constexpr", "-Xptxas", "-v", "-I", os.path.join(ROOT, "include")]


def _sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _deps():
    return (glob.glob(os.path.join(CSRC, "*")) + glob.glob(os.path.join(ROOT, "include", "*.h"))
            + [os.path.abspath(__file__)])


def _stale(target, deps):
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(d) > t for d in deps)


def _compile(src, log):
    obj = os.path.join(BUILD, os.path.basename(src)[:-3] + ".o")
    cmd = [NVCC, *ARCH, *FLAGS, "-c", src, "-o", obj]
    r = subprocess.run(cmd, capture_output=True, text=True)
    log.append((src, r.returncode, r.stdout + r.stderr))
    return obj, r.returncode


def build(force: bool = False, verbose: bool = False) -> str:
    """Compile every kernel source and link libcsa.so; returns its path."""
    deps = _deps()
    if not force and not _stale(LIB, deps):
        return LIB
    os.makedirs(BUILD, exist_ok=True)
    log: list = []
    with ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as ex:
        results = list(ex.map(lambda s: _compile(s, log), _sources()))
    failed = [(s, rc, out) for s, rc, out in log if rc != 0]
    if verbose or failed:
        for s, rc, out in log:
            if verbose or rc != 0:
                sys.stderr.write(f"== {os.path.basename(s)} (rc={rc})\n{out}\n")
    if failed:
        raise RuntimeError("nvcc failed: " + ", ".join(os.path.basename(s) for s, _, _ in failed))
    tmp = LIB + f".tmp{os.getpid()}"
    subprocess.check_call([NVCC, *ARCH, "-shared", "-o", tmp, *[o for o, _ in results],
                           "-lcudart"])
    os.replace(tmp, LIB)
    with open(os.path.join(BUILD, "ptxas.log"), "w") as fh:
        for s, rc, out in log:
            fh.write(f"== {os.path.basename(s)}\n{out}\n")
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
