"""Build libfp8q.so in-tree with nvcc for sm_100a (B200).

    python fp8_quantized_linear_rms_b200/build.py [--force]

Objects go to ``_build/`` at the repository root; the shared library to
``fp8_quantized_linear_rms_b200/libfp8q.so``.  Only stale objects are rebuilt.
"""
from __future__ import annotations

import concurrent.futures as cf
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD = os.path.join(ROOT, "_build")
LIB = os.path.join(PKG, "libfp8q.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ARCH + ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "-Xcompiler",
                     "-fvisibility=hidden", f"-I{INCLUDE}", "-Xptxas", "-v"]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _sources():
    return sorted(os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith(".cu"))


def _headers():
    hs = [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".cuh", ".h", ".inc"))]
    hs += [os.path.join(INCLUDE, f) for f in os.listdir(INCLUDE) if f.endswith(".h")]
    return hs


def _compile(src: str, obj: str, log: str) -> None:
    cmd = [nvcc(), *NVCC_FLAGS, "-c", src, "-o", obj]
    r = subprocess.run(cmd, capture_output=True, text=True)
    with open(log, "w") as f:
        f.write(" ".join(cmd) + "\n" + r.stdout + r.stderr)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed for {src}:\n{r.stderr[-4000:]}")


def build(force: bool = False, verbose: bool = False) -> str:
    os.makedirs(BUILD, exist_ok=True)
    srcs = _sources()
    newest_header = max(os.path.getmtime(h) for h in _headers())
    jobs = []
    objs = []
    for src in srcs:
        stem = os.path.splitext(os.path.basename(src))[0]
        obj = os.path.join(BUILD, stem + ".o")
        objs.append(obj)
        stale = (force or not os.path.exists(obj) or os.path.getmtime(obj) < os.path.getmtime(src)
                 or os.path.getmtime(obj) < newest_header)
        if stale:
            jobs.append((src, obj, os.path.join(BUILD, stem + ".ptxas.log")))
    if jobs:
        with cf.ThreadPoolExecutor(max_workers=min(len(jobs), os.cpu_count() or 4)) as ex:
            list(ex.map(lambda j: _compile(*j), jobs))
    if jobs or force or not os.path.exists(LIB) or any(
            os.path.getmtime(LIB) < os.path.getmtime(o) for o in objs):
        tmp = LIB + ".tmp"
        cmd = [nvcc(), *ARCH, "-shared", "-Xcompiler", "-fPIC", *objs, "-o", tmp]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"link failed:\n{r.stderr[-4000:]}")
        os.replace(tmp, LIB)
    if verbose:
        print(LIB)
    return LIB


def build_variant(out_dir: str, defines: list[str]) -> str:
    """Build a separate copy of the library with extra preprocessor defines
    (test-only builds, e.g. a shortened device wait limit) into out_dir; the
    shipped libfp8q.so is not touched."""
    os.makedirs(out_dir, exist_ok=True)
    lib = os.path.join(out_dir, "libfp8q.so")
    objs, jobs = [], []
    for src in _sources():
        obj = os.path.join(out_dir, os.path.splitext(os.path.basename(src))[0] + ".o")
        objs.append(obj)
        jobs.append([nvcc(), *NVCC_FLAGS, *[f"-D{d}" for d in defines], "-c", src, "-o", obj])
    with cf.ThreadPoolExecutor(max_workers=min(len(jobs), os.cpu_count() or 4)) as ex:
        results = list(ex.map(lambda c: subprocess.run(c, capture_output=True, text=True), jobs))
    for c, r in zip(jobs, results):
        if r.returncode != 0:
            raise RuntimeError(f"nvcc failed: {' '.join(c)}\n{r.stderr[-4000:]}")
    r = subprocess.run([nvcc(), *ARCH, "-shared", "-Xcompiler", "-fPIC", *objs, "-o", lib],
                       capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"link failed:\n{r.stderr[-4000:]}")
    return lib


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose=True)
