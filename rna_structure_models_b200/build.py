"""Build the sm_100a C-ABI library (and the test-only probe library) in tree
with nvcc.  `python -m rna_structure_models_b200.build` or build_all()."""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libflashipa_b200.so")
PROBE_SRC = os.path.join(ROOT, "tests", "csrc", "umma_probe.cu")
PROBE_LIB = os.path.join(ROOT, "tests", "libflashipa_probe.so")
CHECKED_LIB = os.path.join(PKG, "libflashipa_b200_checked.so")
BOUNDS_PROBE_SRC = os.path.join(ROOT, "tests", "csrc", "bounds_probe.cu")
BOUNDS_PROBE_LIB = os.path.join(ROOT, "tests", "libflashipa_bounds_probe.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-shared",
         "--expt-relaxed-constexpr", "-Xcompiler", "-fvisibility=hidden"]
SOURCES = ["api.cu", "ipa_prologue.cu", "ipa_attention.cu", "ipa_attention_pair.cu", "geo_kernels.cu",
           "geo_static.cu", "meet.cu", "frames.cu", "geo_backward.cu", "linear.cu",
           "ipa_backward.cu", "distogram.cu"]


def nvcc() -> str:
    exe = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(exe):
        raise RuntimeError("nvcc not found")
    return exe


def _run(cmd, verbose):
    if verbose:
        print(" ".join(cmd), flush=True)
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed ({r.returncode}):\n{r.stdout}\n{r.stderr}")
    return r.stdout + r.stderr


def build_lib(verbose: bool = False, ptxas_info: bool = False) -> str:
    srcs = [os.path.join(CSRC, s) for s in SOURCES]
    cmd = [nvcc(), *ARCH, *FLAGS, f"-I{INCLUDE}", f"-I{CSRC}", "-Xcompiler",
           "-DFLASHIPA_EXPORTS", *srcs, "-o", LIB]
    if ptxas_info:
        cmd.insert(1, "-Xptxas=-v")
    out = _run(cmd, verbose)
    if ptxas_info:
        print(out)
    return LIB


def build_traced(out_path: str, verbose: bool = False) -> str:
    """Same library with per-tile event tracing compiled in (IPA_TRACE)."""
    srcs = [os.path.join(CSRC, s) for s in SOURCES]
    cmd = [nvcc(), *ARCH, *FLAGS, "-DIPA_TRACE", f"-I{INCLUDE}", f"-I{CSRC}", *srcs, "-o", out_path]
    _run(cmd, verbose)
    return out_path


def build_checked(out_path: str = CHECKED_LIB, verbose: bool = False) -> str:
    """Same library with every global store of the kernels bounds-checked
    (IPA_BOUNDS_CHECK): an index outside its buffer is reported in the error
    word as IPA_ERR_BOUNDS and the store redirected; the stand-in for a
    memory checker."""
    srcs = [os.path.join(CSRC, s) for s in SOURCES]
    cmd = [nvcc(), *ARCH, *FLAGS, "-DIPA_BOUNDS_CHECK", f"-I{INCLUDE}", f"-I{CSRC}", "-Xcompiler",
           "-DFLASHIPA_EXPORTS", *srcs, "-o", out_path]
    _run(cmd, verbose)
    return out_path


def build_probe(verbose: bool = False) -> str:
    cmd = [nvcc(), *ARCH, *FLAGS, f"-I{INCLUDE}", f"-I{CSRC}", PROBE_SRC, "-o", PROBE_LIB]
    _run(cmd, verbose)
    return PROBE_LIB


def build_bounds_probe(verbose: bool = False) -> str:
    cmd = [nvcc(), *ARCH, *FLAGS, "-DIPA_BOUNDS_CHECK", f"-I{CSRC}", BOUNDS_PROBE_SRC, "-o", BOUNDS_PROBE_LIB]
    _run(cmd, verbose)
    return BOUNDS_PROBE_LIB


def checked_is_stale(path: str = CHECKED_LIB) -> bool:
    """True when the bounds-checked library is missing or older than a source."""
    if not os.path.exists(path):
        return True
    t = os.path.getmtime(path)
    srcs = [os.path.join(CSRC, f) for f in os.listdir(CSRC)] + [os.path.join(INCLUDE, f) for f in os.listdir(INCLUDE)]
    return any(os.path.getmtime(s) > t for s in srcs)


def build_all(verbose: bool = False) -> None:
    """Product library, bounds-checked library and the test probes (the two
    libraries compile concurrently)."""
    from concurrent.futures import ThreadPoolExecutor
    jobs = [build_lib, build_checked]
    if os.path.exists(PROBE_SRC):
        jobs.append(build_probe)
    if os.path.exists(BOUNDS_PROBE_SRC):
        jobs.append(build_bounds_probe)
    with ThreadPoolExecutor(len(jobs)) as ex:
        for f in [ex.submit(j, verbose=verbose) for j in jobs]:
            f.result()


if __name__ == "__main__":
    build_all(verbose=True)
    if "--ptxas" in sys.argv:
        build_lib(ptxas_info=True)
