"""Build the in-tree shared library ``libkvq.so`` for sm_100a with nvcc.

Run as ``python -m quantized_paged_kv_tile_b200.build``.  The library is
rebuilt when any source under ``csrc/`` or ``include/kvq.h`` is newer than it.
"""

from __future__ import annotations

import glob
import os
import shutil
import subprocess
import sys

PKG_DIR = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG_DIR)
CSRC = os.path.join(PKG_DIR, "csrc")
LIB_PATH = os.path.join(PKG_DIR, "libkvq.so")
HEADER = os.path.join(ROOT, "include", "kvq.h")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-shared", "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
    "--expt-relaxed-constexpr",
]


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _stale() -> bool:
    if not os.path.exists(LIB_PATH):
        return True
    deps = sources() + glob.glob(os.path.join(CSRC, "*.h")) + glob.glob(os.path.join(CSRC, "*.cuh")) + [HEADER]
    lib_time = os.path.getmtime(LIB_PATH)
    return any(os.path.getmtime(p) > lib_time for p in deps)


def nvcc_path() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _run(cmd, verbose):
    if verbose:
        print(" ".join(cmd), file=sys.stderr)
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError(f"nvcc failed ({res.returncode}):\n{res.stdout}\n{res.stderr}")


def build(force: bool = False, verbose: bool = False) -> str:
    """Compile csrc/*.cu into libkvq.so (sm_100a) unless it is up to date.

    Each translation unit compiles in its own nvcc process (they share no
    device code), in parallel, then one nvcc call links the shared library."""
    if not force and not _stale():
        return LIB_PATH
    import concurrent.futures
    import tempfile
    nvcc = nvcc_path()
    compile_flags = [f for f in NVCC_FLAGS if f != "-shared"]
    with tempfile.TemporaryDirectory(prefix="kvq_build_") as tmpdir:
        objs = [os.path.join(tmpdir, os.path.basename(src) + ".o") for src in sources()]
        jobs = [[nvcc, *compile_flags, "-c", "-o", obj, src] for src, obj in zip(sources(), objs)]
        workers = max(1, min(len(jobs), os.cpu_count() or 1))
        with concurrent.futures.ThreadPoolExecutor(workers) as pool:
            for fut in [pool.submit(_run, cmd, verbose) for cmd in jobs]:
                fut.result()
        tmp = LIB_PATH + ".tmp"
        _run([nvcc, "-gencode", "arch=compute_100a,code=sm_100a", "-shared", "-o", tmp, *objs], verbose)
    os.replace(tmp, LIB_PATH)
    return LIB_PATH


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True))
