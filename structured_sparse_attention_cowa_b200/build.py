"""Build libcowa.so in-tree for sm_100a with nvcc (no GPU needed to build).

    python -m structured_sparse_attention_cowa_b200.build [--debug] [-v]

Compiles every csrc/*.cu to an object in _build/ and links them into
structured_sparse_attention_cowa_b200/libcowa.so (static CUDA runtime; the
driver API is reached through cudaGetDriverEntryPoint, so no -lcuda).
Objects are rebuilt only when a source or header is newer.

--debug builds libcowa_debug.so with COWA_DEBUG=1: the kernels check every planned tile and
cache row against the call's tensors before loading it, and a failed check is reported as
COWA_ERR_CHECK through the workspace status (the binding loads this library when the
environment has COWA_DEBUG=1).
"""

from __future__ import annotations

import argparse
import glob
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
BUILD = os.path.join(ROOT, "_build")
LIB = os.path.join(PKG, "libcowa.so")
LIB_DEBUG = os.path.join(PKG, "libcowa_debug.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
CFLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC,-O3", "--expt-relaxed-constexpr",
          "-I" + os.path.join(ROOT, "include"), "-I" + CSRC]


def _nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if cand and (os.path.isabs(cand) and os.path.exists(cand) or not os.path.isabs(cand)):
            return cand
    return "nvcc"


def _newest_header() -> float:
    hdrs = glob.glob(os.path.join(CSRC, "*.h")) + glob.glob(os.path.join(CSRC, "*.cuh")) + \
        glob.glob(os.path.join(ROOT, "include", "*.h"))
    return max((os.path.getmtime(h) for h in hdrs), default=0.0)


def build(debug: bool = False, verbose: bool = False, ptxas_info: bool = False) -> str:
    os.makedirs(BUILD, exist_ok=True)
    nvcc = _nvcc()
    flags = list(CFLAGS)
    if debug:
        flags.append("-DCOWA_DEBUG=1")
    if ptxas_info:
        flags += ["-Xptxas", "-v"]
    hdr_t = _newest_header()
    objs, jobs = [], []
    for src in sorted(glob.glob(os.path.join(CSRC, "*.cu"))):
        obj = os.path.join(BUILD, os.path.basename(src)[:-3] + (".dbg.o" if debug else ".o"))
        objs.append(obj)
        if (not ptxas_info and os.path.exists(obj) and os.path.getmtime(obj) >= os.path.getmtime(src)
                and os.path.getmtime(obj) >= hdr_t):
            continue
        jobs.append((src, [nvcc, *ARCH, *flags, "-c", src, "-o", obj]))

    def compile_one(job):
        src, cmd = job
        if verbose:
            print(" ".join(cmd), flush=True)
        r = subprocess.run(cmd, capture_output=True, text=True)
        return src, r

    # the translation units are independent: compile them side by side
    from concurrent.futures import ThreadPoolExecutor

    with ThreadPoolExecutor(max_workers=max(1, min(len(jobs), os.cpu_count() or 1))) as ex:
        results = list(ex.map(compile_one, jobs))
    for src, r in results:
        if r.returncode != 0 or verbose or ptxas_info:
            sys.stderr.write(r.stdout + r.stderr)
        if r.returncode != 0:
            raise RuntimeError(f"nvcc failed on {os.path.basename(src)}")
    out = LIB_DEBUG if debug else LIB
    lib_t = os.path.getmtime(out) if os.path.exists(out) else -1
    if lib_t < max(os.path.getmtime(o) for o in objs):
        cmd = [nvcc, *ARCH, "-shared", "-Xcompiler", "-fPIC", "-o", out, *objs]
        if verbose:
            print(" ".join(cmd), flush=True)
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            sys.stderr.write(r.stdout + r.stderr)
            raise RuntimeError(f"link of {os.path.basename(out)} failed")
    return out


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--debug", action="store_true")
    ap.add_argument("-v", "--verbose", action="store_true")
    ap.add_argument("--ptxas-info", action="store_true")
    args = ap.parse_args()
    print(build(debug=args.debug, verbose=args.verbose, ptxas_info=args.ptxas_info))
