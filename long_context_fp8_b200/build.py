"""Build the DSA CUDA library in-tree: ``long_context_fp8_b200/libdsa_b200.so``.

nvcc compiles every ``csrc/*.cu`` for sm_100a only (``-gencode
arch=compute_100a,code=sm_100a``) and links one shared library with the CUDA
runtime linked statically, so the library depends on nothing but the driver.
Usable as ``python -m long_context_fp8_b200.build``.
"""
from __future__ import annotations

import concurrent.futures as cf
import glob
import os
import re
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libdsa_b200.so")
BUILD_DIR = os.path.join(ROOT, "_build")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "--expt-relaxed-constexpr",
              "-I", INCLUDE, "-I", CSRC]


# Kernels whose warpgroups re-split their registers with setmaxnreg: the split
# adds up to the launch's register file only when ptxas gives them exactly this
# many registers per thread, so any other count fails the build (instead of a
# launch that would wait forever in setmaxnreg, or a silent slower path).
SETMAXNREG_KERNELS = {"index_tc_kernel": 168, "sparse_attn_tc_kernel": 168}


def kernel_name(mangled: str) -> str:
    """The unqualified function name of an Itanium-mangled nested name
    (_ZN <len><component> ... E|I ...); the input itself if it is not one."""
    if not mangled.startswith("_ZN"):
        return mangled
    i = 3
    while i < len(mangled) and mangled[i].isdigit():
        j = i
        while mangled[j].isdigit():
            j += 1
        n = int(mangled[i:j])
        comp = mangled[j:j + n]
        i = j + n
        if i >= len(mangled) or mangled[i] in "EI":
            return comp
    return mangled


def check_registers(ptxas_log: str, src: str) -> list:
    """Checks the ptxas -v report of one source file against
    SETMAXNREG_KERNELS; returns (mangled name, registers, spill-store bytes)
    per entry function."""
    found, cur, spill = [], None, 0
    for line in ptxas_log.splitlines():
        m = re.search(r"Compiling entry function '([^']+)'", line)
        if m:
            cur, spill = m.group(1), 0
            continue
        m = re.search(r"(\d+) bytes spill stores", line)
        if m and cur is not None:
            spill = int(m.group(1))
            continue
        m = re.search(r"Used (\d+) registers", line)
        if m and cur is not None:
            found.append((cur, int(m.group(1)), spill))
            cur = None
    for name, regs, _ in found:
        want = SETMAXNREG_KERNELS.get(kernel_name(name))
        if want is not None and regs != want:
            raise RuntimeError(f"{os.path.basename(src)}: {kernel_name(name)} built with {regs} registers "
                               f"per thread, its setmaxnreg split needs exactly {want}")
    return found


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _deps():
    return _sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h")) + \
        glob.glob(os.path.join(INCLUDE, "*.h"))


def up_to_date() -> bool:
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    return all(os.path.getmtime(p) <= t for p in _deps())


def build(force: bool = False, verbose: bool = False, extra_flags=()) -> str:
    if not force and up_to_date():
        return LIB
    os.makedirs(BUILD_DIR, exist_ok=True)
    cc = nvcc()
    objs = []

    def compile_one(src):
        obj = os.path.join(BUILD_DIR, os.path.basename(src) + ".o")
        cmd = [cc, *ARCH, *NVCC_FLAGS, *extra_flags, "-Xptxas", "-v", "-c", src, "-o", obj]
        if verbose:
            print(" ".join(cmd), flush=True)
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"nvcc failed for {src}:\n{r.stdout}\n{r.stderr}")
        check_registers(r.stdout + r.stderr, src)
        if verbose and (r.stdout or r.stderr):
            print(r.stdout, r.stderr, flush=True)
        return obj

    with cf.ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as ex:
        objs = list(ex.map(compile_one, _sources()))
    tmp = LIB + ".tmp"
    cmd = [cc, *ARCH, "-shared", "-o", tmp, *objs, "-cudart", "static"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
