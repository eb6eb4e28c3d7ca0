"""Builds libragged.so (the CUDA kernels and their C ABI) for sm_100a with nvcc.

    python -m ragged_variable_length_b200.build [--force] [--verbose-ptxas]

The library is built in-tree, next to this file, and statically links the
CUDA runtime so that it does not depend on which libcudart the process loads.
"""
from __future__ import annotations

import glob
import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(HERE, "libragged.so")
# The same sources with RAGGED_TEST_HOOKS: failure-path switches for the tests.
HOOKS_LIB = os.path.join(HERE, "libragged_testhooks.so")
MAIN = os.path.join(CSRC, "ragged_api.cu")

ARCH_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def sources() -> list:
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cuh")) +
                  glob.glob(os.path.join(INCLUDE, "*.h")))


def stale(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    return any(os.path.getmtime(s) > t for s in sources())


def command(out: str, ptxas_verbose: bool = False, test_hooks: bool = False) -> list:
    cmd = [nvcc(), *ARCH_FLAGS, "-O3", "-lineinfo", "-std=c++17", "-shared", "-Xcompiler", "-fPIC",
           "-Xcompiler", "-fvisibility=hidden", "--expt-relaxed-constexpr", "-cudart", "static",
           f"-I{INCLUDE}", f"-I{CSRC}", "-DRAGGED_BUILD", MAIN, "-o", out]
    if test_hooks:
        cmd.insert(-3, "-DRAGGED_TEST_HOOKS")
    if ptxas_verbose:
        cmd[1:1] = ["-Xptxas", "-v"]
    return cmd


FASTCALL_SRC = os.path.join(CSRC, "fastcall.c")


def fastcall_path() -> str:
    import sysconfig
    return os.path.join(HERE, "_fastcall" + sysconfig.get_config_var("EXT_SUFFIX"))


def build_fastcall(force: bool = False) -> str:
    """CPython extension that forwards a pre-marshalled ragged_pipeline call."""
    import sysconfig
    out = fastcall_path()
    if not force and os.path.exists(out) and os.path.getmtime(out) >= os.path.getmtime(FASTCALL_SRC):
        return out
    tmp = f"{out}.{os.getpid()}.tmp"
    subprocess.run(["gcc", "-O2", "-Wall", "-shared", "-fPIC", f"-I{sysconfig.get_paths()['include']}",
                    FASTCALL_SRC, "-o", tmp], check=True)
    os.replace(tmp, out)
    return out


def _compile(lib: str, force: bool, ptxas_verbose: bool, test_hooks: bool) -> str:
    if not force and not stale(lib):
        return lib
    tmp = f"{lib}.{os.getpid()}.tmp"
    proc = subprocess.run(command(tmp, ptxas_verbose, test_hooks), capture_output=True, text=True)
    if proc.returncode != 0:
        sys.stderr.write(proc.stdout + proc.stderr)
        raise RuntimeError(f"nvcc failed building {os.path.basename(lib)}")
    if ptxas_verbose:
        sys.stderr.write(proc.stdout + proc.stderr)
    os.replace(tmp, lib)
    return lib


def build(force: bool = False, ptxas_verbose: bool = False) -> str:
    build_fastcall(force)
    return _compile(LIB, force, ptxas_verbose, False)


def build_test_hooks(force: bool = False) -> str:
    """libragged_testhooks.so: the library with the failure-path test switches."""
    return _compile(HOOKS_LIB, force, False, True)


if __name__ == "__main__":
    build(force="--force" in sys.argv, ptxas_verbose="--verbose-ptxas" in sys.argv)
    print(LIB)
    if "--test-hooks" in sys.argv:
        print(build_test_hooks(force="--force" in sys.argv))
