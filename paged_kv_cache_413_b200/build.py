"""Build libpa.so in-tree with nvcc for sm_100a (B200).

``python -m paged_kv_cache_413_b200.build`` or :func:`build`.  The library is
placed next to this file so that it travels with the source tree; object files
go to ``_build/`` (not part of the source).
"""

from __future__ import annotations

import glob
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD_DIR = os.path.join(ROOT, "_build")
LIB = os.path.join(PKG, "libpa.so")

NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC,-O3", "-I", INCLUDE, "-I", CSRC,
         "--expt-relaxed-constexpr", "-Xptxas", "-warn-spills"]


def _sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cpp")))


def _deps():
    return _sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(
        os.path.join(CSRC, "*.h")) + glob.glob(os.path.join(INCLUDE, "*.h")) + [__file__]


# The failure-detection test build: the same sources with pipeline waits that give
# up after 2 ms instead of ~1 s, and a decode producer that never announces or
# copies the 4th 16-token tile of a CTA (tile index 3), so the waits on that stage
# must time out and report PA_DEVERR_PIPE_TIMEOUT.  Only the tests load it.
TIMEOUT_TEST_LIB = os.path.join(PKG, "libpa_timeout_test.so")
TIMEOUT_TEST_FLAGS = ["-DPA_WAIT_LIMIT_NS=2000000ull", "-DPA_TEST_STALL_TILE=3"]


def up_to_date(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return False
    t = os.path.getmtime(lib)
    return all(os.path.getmtime(d) <= t for d in _deps())


def build(force: bool = False, verbose: bool = False, extra_flags: list[str] | None = None,
          lib: str = LIB, build_dir: str = BUILD_DIR) -> str:
    """Compile every CUDA/C++ source and link `lib` (libpa.so); returns its path."""
    if not force and up_to_date(lib):
        return lib
    os.makedirs(build_dir, exist_ok=True)
    procs = []
    objs = []
    for src in _sources():
        obj = os.path.join(build_dir, os.path.basename(src) + ".o")
        objs.append(obj)
        cmd = [NVCC, *ARCH, *FLAGS, *(extra_flags or []), "-c", src, "-o", obj]
        if verbose:
            print(" ".join(cmd), file=sys.stderr)
        procs.append((src, subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.STDOUT,
                                            text=True)))
    failed = []
    for src, p in procs:
        out, _ = p.communicate()
        if out and (verbose or p.returncode):
            print(out, file=sys.stderr)
        if p.returncode:
            failed.append(src)
    if failed:
        raise RuntimeError("nvcc failed for: " + ", ".join(failed))
    tmp = lib + ".tmp.%d" % os.getpid()
    cmd = [NVCC, *ARCH, "-shared", "-o", tmp, *objs]
    subprocess.run(cmd, check=True)
    os.replace(tmp, lib)
    return lib


def build_timeout_test(force: bool = False, verbose: bool = False) -> str:
    """Build the failure-detection test library (see TIMEOUT_TEST_FLAGS)."""
    return build(force, verbose, extra_flags=TIMEOUT_TEST_FLAGS, lib=TIMEOUT_TEST_LIB,
                 build_dir=os.path.join(BUILD_DIR, "timeout_test"))


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
    print(build_timeout_test(force="--force" in sys.argv, verbose="-v" in sys.argv))
