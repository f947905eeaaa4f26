"""Build libwkv7.so in-tree with nvcc for sm_100a (no JIT cache, no torch types).

``python -m linear_attention_rnn_wkv7_b200.build`` or ``build()`` from Python.
Prints a one-line JSON manifest (library path, nvcc version, flags).
"""
from __future__ import annotations

import glob
import json
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libwkv7.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo", "-O3", "-std=c++17",
         "-Xcompiler", "-fPIC", "-shared", "--expt-relaxed-constexpr", "-Xptxas", "-v"]


def sources():
    return [os.path.join(CSRC, "wkv7_api.cu")]


def _stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    deps = glob.glob(os.path.join(CSRC, "*")) + glob.glob(os.path.join(INCLUDE, "*.h"))
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, verbose: bool = False) -> str:
    if force or _stale():
        tmp = LIB + f".tmp{os.getpid()}"
        cmd = [NVCC, *FLAGS, "-I", INCLUDE, "-I", CSRC, "-o", tmp, *sources()]
        res = subprocess.run(cmd, capture_output=True, text=True)
        if res.returncode != 0:
            raise RuntimeError("nvcc failed:\n" + res.stdout + res.stderr)
        if verbose:
            sys.stderr.write(res.stderr)
        os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    path = build(force="--force" in sys.argv, verbose=True)
    ver = subprocess.run([NVCC, "--version"], capture_output=True, text=True).stdout.strip()
    print(json.dumps({"status": "ok", "library": path, "target": "sm_100a",
                      "nvcc": ver.splitlines()[-1] if ver else None}))
