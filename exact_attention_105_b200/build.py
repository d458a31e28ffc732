"""Build the sm_100a shared library in-tree with nvcc.

``python -m exact_attention_105_b200.build`` (or ``build()``) compiles
``csrc/attn_api.cu``, the single translation unit that holds every kernel, into
``libattn_sm100.so`` next to this file, and ``csrc/pycall.c`` (the CPython
argument marshalling for the per-step calls) into ``_pycall`` with the host C
compiler. Each rebuilds only when its sources are newer than its output.
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys
import sysconfig

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(os.path.dirname(HERE), "include")
LIB_NAME = "libattn_sm100.so"
LIB_PATH = os.path.join(HERE, LIB_NAME)
PYCALL_SRC = os.path.join(CSRC, "pycall.c")
PYCALL_PATH = os.path.join(HERE, "_pycall" + (sysconfig.get_config_var("EXT_SUFFIX") or ".so"))

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-shared", "-Xcompiler", "-fPIC",
    "-Xptxas", "-v",
]


def _sources():
    out = [os.path.join(INCLUDE, "attn.h")]
    for name in sorted(os.listdir(CSRC)):
        if name.endswith((".cu", ".cuh", ".h")):
            out.append(os.path.join(CSRC, name))
    return out


def _nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found (set NVCC or put /usr/local/cuda/bin on PATH)")


def is_stale() -> bool:
    if not os.path.exists(LIB_PATH):
        return True
    lib_m = os.path.getmtime(LIB_PATH)
    return any(os.path.getmtime(s) > lib_m for s in _sources())


def build_pycall(force: bool = False) -> str:
    """Compile the CPython marshalling module if needed; return its path."""
    if (not force and os.path.exists(PYCALL_PATH)
            and os.path.getmtime(PYCALL_PATH) >= os.path.getmtime(PYCALL_SRC)):
        return PYCALL_PATH
    cc = os.environ.get("CC") or shutil.which("gcc") or shutil.which("cc")
    if not cc:
        raise RuntimeError("no host C compiler (gcc/cc) for " + PYCALL_SRC)
    tmp = PYCALL_PATH + ".tmp"
    cmd = [cc, "-O2", "-shared", "-fPIC", "-I", sysconfig.get_paths()["include"], "-o", tmp,
           PYCALL_SRC]
    proc = subprocess.run(cmd, capture_output=True, text=True)
    if proc.returncode != 0:
        raise RuntimeError(f"{cc} failed ({proc.returncode}):\n{' '.join(cmd)}\n"
                           f"{proc.stdout}{proc.stderr}")
    os.replace(tmp, PYCALL_PATH)
    return PYCALL_PATH


def build(force: bool = False, verbose: bool = False) -> str:
    """Compile the library and the marshalling module if needed; return the
    library's path. Raises on failure."""
    if force or is_stale():
        _build_library(verbose)
    build_pycall(force)
    return LIB_PATH


def _build_library(verbose: bool) -> None:
    tmp = LIB_PATH + ".tmp"
    cmd = [_nvcc(), *NVCC_FLAGS, "-o", tmp, os.path.join(CSRC, "attn_api.cu")]
    proc = subprocess.run(cmd, cwd=CSRC, capture_output=True, text=True)
    log = proc.stdout + proc.stderr
    if proc.returncode != 0:
        raise RuntimeError(f"nvcc failed ({proc.returncode}):\n{' '.join(cmd)}\n{log}")
    if verbose:
        sys.stdout.write(log)
    os.replace(tmp, LIB_PATH)
    with open(os.path.join(HERE, "ptxas_info.txt"), "w") as f:
        f.write(log)


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True))
