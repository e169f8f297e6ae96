"""Builds the C-ABI library ``libquest_b200.so`` in-tree with nvcc for sm_100a, and
the benchmark's tensor-core rate probes as a separate ``libquest_probe.so``.

Usage: ``python -m bit_quantization_aware_blockwise_b200.build [--force]``.
The CUDA runtime is linked statically so the library does not depend on the
runtime version that PyTorch bundles; the driver API is reached through
``cudaGetDriverEntryPoint`` (no libcuda link).
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(HERE, "libquest_b200.so")
PROBE_LIB = os.path.join(HERE, "libquest_probe.so")
SOURCES = ["quest_api.cu", "quantize_fwd.cu", "quantize_hs.cu", "quantize_tc.cu", "trust_bwd.cu", "trust_tc.cu",
           "w4a4_gemm.cu", "w4a4_grouped.cu", "trust_linear.cu", "fp4_gemm.cu", "tc_host.cu", "transpose.cu",
           "quantize_sparse.cu", "w4a4_sparse.cu"]
PROBE_SOURCES = ["bench_probe/probe_mma.cu"]
HEADERS = ["quest_device.cuh", "quest_internal.h", "quest_emit.cuh", "quest_tc.cuh", "tc_common.cuh"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    return "nvcc"


def _inputs():
    files = [os.path.join(CSRC, f) for f in SOURCES + HEADERS]
    files += [os.path.join(CSRC, f) for f in PROBE_SOURCES]
    files += [os.path.join(INCLUDE, h) for h in ("quest.h", "quest_debug.h", "quest_probe.h")]
    files.append(os.path.abspath(__file__))
    return files


def stale() -> bool:
    if not os.path.exists(LIB) or not os.path.exists(PROBE_LIB):
        return True
    t = min(os.path.getmtime(LIB), os.path.getmtime(PROBE_LIB))
    return any(os.path.getmtime(f) > t for f in _inputs())


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and not stale():
        return LIB
    out_dir = os.path.join(HERE, "_build")
    os.makedirs(out_dir, exist_ok=True)
    objs = []
    procs = []
    common = [nvcc(), *ARCH, "-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC",
              "-I", INCLUDE, "-I", CSRC, "--expt-relaxed-constexpr"]
    if verbose:
        common += ["-Xptxas", "-v"]
    for src in SOURCES + PROBE_SOURCES:
        obj = os.path.join(out_dir, os.path.basename(src) + ".o")
        objs.append(obj)
        cmd = common + ["-c", os.path.join(CSRC, src), "-o", obj]
        procs.append((cmd, subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.STDOUT)))
    failed = False
    for cmd, p in procs:
        out, _ = p.communicate()
        if out:
            sys.stdout.write(out.decode(errors="replace"))
        if p.returncode != 0:
            failed = True
            sys.stderr.write("nvcc failed: " + " ".join(cmd) + "\n")
    if failed:
        raise RuntimeError("building libquest_b200.so failed")
    n = len(SOURCES)
    for lib, lib_objs in ((LIB, objs[:n]), (PROBE_LIB, objs[n:])):
        tmp = lib + f".{os.getpid()}.tmp"
        subprocess.run([nvcc(), *ARCH, "-shared", "-cudart", "static", "-o", tmp, *lib_objs], check=True)
        os.replace(tmp, lib)
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose="-v" in sys.argv)
    print(LIB)
