"""Build the CUDA library ``libhla.so`` in-tree with nvcc for sm_100a.

Every ``csrc/*.cu`` file is compiled to an object under ``_build/`` (in
parallel), then linked into ``higher_order_linear_chunked_b200/libhla.so``.
The CUDA runtime is linked statically; the driver entry point used for TMA
tensor maps is resolved at run time, so the library loads on hosts without a GPU.

What to rebuild is decided by content, not by file times: each object has a
stamp holding the sha256 of its source, of every header, of the compiler's
version line and of the command line.  An object whose stamp does not match
(or that has none) is compiled again, and the library is linked again whenever
any object was, or when its own stamp (the hash of all object stamps) differs.
Objects and a library copied from another machine are therefore rebuilt unless
they were built from exactly these sources with exactly these flags.
"""
from __future__ import annotations

import concurrent.futures as cf
import glob
import hashlib
import os
import shutil
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
BUILD = os.path.join(ROOT, "_build")
LIB = os.path.join(HERE, "libhla.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "--expt-relaxed-constexpr",
         "-I", os.path.join(ROOT, "include")]


def _nvcc() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _nvcc_version(nvcc: str) -> str:
    r = subprocess.run([nvcc, "--version"], capture_output=True, text=True)
    return r.stdout.strip().splitlines()[-1] if r.stdout.strip() else ""


def _sha(paths, extra: str) -> str:
    h = hashlib.sha256()
    for p in sorted(paths):
        h.update(os.path.basename(p).encode())
        with open(p, "rb") as f:
            h.update(hashlib.sha256(f.read()).digest())
    h.update(extra.encode())
    return h.hexdigest()


def _stamp_ok(target: str, digest: str) -> bool:
    stamp = target + ".sha256"
    if not (os.path.exists(target) and os.path.exists(stamp)):
        return False
    with open(stamp) as f:
        return f.read().strip() == digest


def _write_stamp(target: str, digest: str) -> None:
    with open(target + ".sha256", "w") as f:
        f.write(digest + "\n")


def build(force: bool = False, verbose: bool = False, extra=None) -> str:
    nvcc = _nvcc()
    version = _nvcc_version(nvcc)
    os.makedirs(BUILD, exist_ok=True)
    sources = sorted(glob.glob(os.path.join(CSRC, "*.cu")))
    headers = glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h")) + \
        glob.glob(os.path.join(ROOT, "include", "*.h"))
    objs, digests, jobs = [], [], []
    for src in sources:
        obj = os.path.join(BUILD, os.path.basename(src)[:-3] + ".o")
        cmd = [nvcc] + ARCH + FLAGS + list(extra or []) + ["-c", src, "-o", obj]
        digest = _sha([src] + headers, version + "\n" + " ".join(cmd))
        objs.append(obj)
        digests.append(digest)
        if force or not _stamp_ok(obj, digest):
            jobs.append((cmd, obj, digest))

    def run(cmd):
        if verbose:
            print(" ".join(cmd), flush=True)
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"nvcc failed:\n{' '.join(cmd)}\n{r.stdout}\n{r.stderr}")
        if verbose and (r.stdout or r.stderr):
            print(r.stdout + r.stderr, flush=True)

    def compile_one(job):
        cmd, obj, digest = job
        if os.path.exists(obj + ".sha256"):
            os.unlink(obj + ".sha256")
        run(cmd)
        _write_stamp(obj, digest)

    with cf.ThreadPoolExecutor(max_workers=max(1, min(len(jobs), os.cpu_count() or 1))) as ex:
        list(ex.map(compile_one, jobs))
    link = [nvcc] + ARCH + ["-shared", "-o", LIB] + objs
    lib_digest = hashlib.sha256(("\n".join(digests) + "\n" + " ".join(link)).encode()).hexdigest()
    if force or jobs or not _stamp_ok(LIB, lib_digest):
        if os.path.exists(LIB + ".sha256"):
            os.unlink(LIB + ".sha256")
        run(link)
        _write_stamp(LIB, lib_digest)
    return LIB


if __name__ == "__main__":
    import sys
    build(force="--force" in sys.argv, verbose=True)
