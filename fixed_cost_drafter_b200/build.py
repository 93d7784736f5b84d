"""Builds the in-tree shared libraries for sm_100a with nvcc.

* ``fixed_cost_drafter_b200/liblongspark.so`` — the C-ABI library (csrc/*.cu).
* ``synth/libls_synth.so`` — the device twin of the seeded input generator.

Each library is rebuilt only when one of its sources (or a header) is newer than it.
Load this file by path (``load_builder()`` in the repository's entry points does), not as
``fixed_cost_drafter_b200.build``: importing the package loads the library it builds.
The CUDA runtime is linked statically, so loading a library needs no GPU driver.
"""

from __future__ import annotations

import concurrent.futures as cf
import glob
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
LIB = os.path.join(PKG, "liblongspark.so")
SYNTH_SRC = os.path.join(ROOT, "synth", "synth.cu")
SYNTH_LIB = os.path.join(ROOT, "synth", "libls_synth.so")
BUILD_DIR = os.path.join(ROOT, "_build")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
         "--expt-relaxed-constexpr"]


def _nvcc():
    cand = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    return cand if os.path.exists(cand) else "nvcc"


def _stale(target, deps):
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(d) > t for d in deps)


def _run(cmd):
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        sys.stderr.write(r.stdout + r.stderr)
        raise RuntimeError("nvcc failed: " + " ".join(cmd))
    return r.stdout + r.stderr


def build(verbose: bool = False, force: bool = False, extra: list | None = None) -> None:
    nvcc = _nvcc()
    os.makedirs(BUILD_DIR, exist_ok=True)
    extra = list(extra or [])
    headers = glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h")) + \
        [os.path.join(ROOT, "include", "longspark.h")]
    sources = sorted(glob.glob(os.path.join(CSRC, "*.cu")))
    if force or _stale(LIB, sources + headers + [__file__]):
        objs = [os.path.join(BUILD_DIR, os.path.basename(s) + ".o") for s in sources]
        jobs = []
        for s, o in zip(sources, objs):
            if force or _stale(o, [s] + headers + [__file__]):
                jobs.append([nvcc, *ARCH, *FLAGS, *extra, "-I", os.path.join(ROOT, "include"), "-c", s, "-o", o])
        with cf.ThreadPoolExecutor(max_workers=min(8, max(1, len(jobs)))) as ex:
            for out in ex.map(_run, jobs):
                if verbose and out.strip():
                    print(out)
        _run([nvcc, *ARCH, "-shared", "-o", LIB, *objs])
    if force or _stale(SYNTH_LIB, [SYNTH_SRC, __file__]):
        _run([nvcc, *ARCH, *FLAGS, "-shared", "-o", SYNTH_LIB, SYNTH_SRC])


if __name__ == "__main__":
    build(verbose=True, force="--force" in sys.argv,
          extra=["-Xptxas", "-v"] if "--ptxas" in sys.argv else None)
    print("built", LIB, SYNTH_LIB)
