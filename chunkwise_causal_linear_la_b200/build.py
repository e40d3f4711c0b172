"""Build the CUDA library libla_b200.so in-tree for sm_100a.

Each ``csrc/*.cu`` file is compiled by nvcc into an object (in parallel) with
``-gencode arch=compute_100a,code=sm_100a -lineinfo -O3`` and the objects are
linked into ``chunkwise_causal_linear_la_b200/libla_b200.so``.  The CUDA
runtime is linked statically; the driver API entry point used for TMA
descriptors is fetched at run time, so the library loads on a machine without
a GPU driver (symbols can be inspected; compute calls need a device).
"""
from __future__ import annotations

import glob
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(os.path.dirname(PKG), "include")
LIB = os.path.join(PKG, "libla_b200.so")
BUILD_DIR = os.path.join(os.path.dirname(PKG), "_build")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ARCH + ["-lineinfo", "-O3", "-std=c++17", "-Xcompiler", "-fPIC,-O2,-fvisibility=hidden",
                     "--expt-relaxed-constexpr", "-I" + INCLUDE]


def nvcc() -> str:
    cand = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(cand):
        raise RuntimeError("nvcc not found; the CUDA toolkit is required to build libla_b200.so")
    return cand


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    deps = sources() + glob.glob(os.path.join(CSRC, "*.h")) + glob.glob(os.path.join(CSRC, "*.cuh"))
    deps += glob.glob(os.path.join(INCLUDE, "*.h"))
    return any(os.path.getmtime(p) > t for p in deps)


# The warp-specialised tensor-core kernels re-split their registers between
# warpgroups with setmaxnreg (.dec to 104, .inc to 232), which is only valid if
# the kernel launches with exactly this many registers per thread.
TC_LAUNCH_REGS = 168
# source file -> kernel whose launch register count is checked
TC_KERNELS = {"la_tc.cu": "chunk_tc_kernel", "la_gdn.cu": "gdn_tc_kernel"}


def _check_tc_registers(ptxas_log: str, kernel: str, src: str) -> None:
    regs, entry = [], None
    for line in ptxas_log.splitlines():
        if "Compiling entry function" in line:
            entry = line
        elif "Used" in line and "registers" in line and entry and kernel in entry:
            regs.append(int(line.split("Used")[1].split("registers")[0]))
            entry = None
    if not regs or any(r != TC_LAUNCH_REGS for r in regs):
        raise RuntimeError("%s launch registers %s != %d: the setmaxnreg split in %s must be revised"
                           % (kernel, regs, TC_LAUNCH_REGS, src))


def build(force: bool = False, verbose: bool = False, extra_flags=()) -> str:
    """Compile and link libla_b200.so if any source is newer; returns its path."""
    if not force and not _stale():
        return LIB
    os.makedirs(BUILD_DIR, exist_ok=True)
    nv = nvcc()
    procs = []
    objs = []
    for src in sources():
        obj = os.path.join(BUILD_DIR, os.path.basename(src) + ".o")
        objs.append(obj)
        cmd = [nv, *NVCC_FLAGS, *extra_flags, "-c", src, "-o", obj]
        if os.path.basename(src) in TC_KERNELS:
            cmd += ["-Xptxas", "-v"]
        if verbose:
            print(" ".join(cmd), file=sys.stderr)
        procs.append((src, subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.STDOUT)))
    failed = []
    for src, p in procs:
        out, _ = p.communicate()
        text = out.decode(errors="replace")
        if verbose or p.returncode:
            sys.stderr.write(text)
        if p.returncode:
            failed.append(os.path.basename(src))
        elif os.path.basename(src) in TC_KERNELS:
            _check_tc_registers(text, TC_KERNELS[os.path.basename(src)], os.path.basename(src))
    if failed:
        raise RuntimeError("nvcc failed for: " + ", ".join(failed))
    tmp = LIB + ".tmp.%d" % os.getpid()
    link = [nv, *ARCH, "-shared", "-Xcompiler", "-fPIC", *objs, "-o", tmp, "-cudart", "static", "-ldl", "-lpthread"]
    if verbose:
        print(" ".join(link), file=sys.stderr)
    subprocess.check_call(link)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
