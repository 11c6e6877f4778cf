"""Builds the sm_100a attention library ``libfa_sm100.so`` in-tree with nvcc.

Each translation unit under ``csrc/`` compiles in parallel to an object file
(``-gencode arch=compute_100a,code=sm_100a -lineinfo -O3``), then one link
step produces the shared library next to this file.  Run
``python -m exact_io_aware_49_b200.build`` (``-v`` prints ptxas register and
shared-memory usage).
"""

import os
import shutil
import subprocess
import sys
import tempfile

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(os.path.dirname(HERE), "include")
LIB_NAME = "libfa_sm100.so"
LIB_PATH = os.path.join(HERE, LIB_NAME)
SOURCES = ["fa_api.cu", "fa_fwd.cu", "fa_fwd_wide.cu", "fa_bwd.cu", "fa_bwd_wide.cu", "fa_decode.cu", "fa_mask.cu",
           "fa_noalloc.cu"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def _nvcc():
    cand = os.environ.get("NVCC") or shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(cand) and not shutil.which(cand):
        raise RuntimeError("nvcc not found: the CUDA toolkit is required to build " + LIB_NAME)
    return cand


def build(verbose=False, force=False):
    """Compile every CUDA source and link the shared library; returns its path."""
    srcs = [os.path.join(CSRC, s) for s in SOURCES]
    deps = srcs + [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".cuh", ".h"))]
    deps.append(os.path.join(INCLUDE, "fa.h"))
    if not force and os.path.exists(LIB_PATH):
        lib_t = os.path.getmtime(LIB_PATH)
        if all(os.path.getmtime(d) <= lib_t for d in deps) and os.path.getmtime(__file__) <= lib_t:
            return LIB_PATH
    nvcc = _nvcc()
    flags = ARCH + ["-lineinfo", "-O3", "-std=c++17", "-Xcompiler", "-fPIC", "--expt-relaxed-constexpr",
                    "-I", INCLUDE, "-I", CSRC]
    if verbose:
        flags += ["-Xptxas", "-v"]
    tmp = tempfile.mkdtemp(prefix="fa_build_")
    try:
        procs = []
        objs = []
        for s in srcs:
            o = os.path.join(tmp, os.path.basename(s) + ".o")
            objs.append(o)
            procs.append((s, subprocess.Popen([nvcc, "-c", s, "-o", o] + flags, stdout=subprocess.PIPE,
                                              stderr=subprocess.STDOUT, text=True)))
        failed = []
        for s, p in procs:
            out, _ = p.communicate()
            if verbose or p.returncode != 0:
                sys.stdout.write(out)
            if p.returncode != 0:
                failed.append(s)
        if failed:
            raise RuntimeError("nvcc failed for: " + ", ".join(failed))
        tmp_lib = os.path.join(tmp, LIB_NAME)
        subprocess.run([nvcc, "-shared", "-o", tmp_lib] + ARCH + objs, check=True)
        os.replace(tmp_lib, LIB_PATH)
    finally:
        shutil.rmtree(tmp, ignore_errors=True)
    return LIB_PATH


if __name__ == "__main__":
    print(build(verbose="-v" in sys.argv, force=True))
