"""Build libkvq.so (the C-ABI library of include/kvq.h) in-tree for sm_100a.

Compiles every translation unit of ``csrc/`` with nvcc for
``-gencode arch=compute_100a,code=sm_100a`` in parallel (the quantize kernels
once per (d, b) pair from ``quantize_inst.cu``), recompiling only objects
whose source, shared headers or flags changed, and links them into
``calibration_free_rotated_token_b200/libkvq.so`` with the CUDA runtime
linked statically.  Object files go to ``_build/`` at the repository root.

Usage: ``python -m calibration_free_rotated_token_b200.build [--force] [-j N]``.
"""
from __future__ import annotations

import argparse
import concurrent.futures as cf
import hashlib
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
OUT = os.path.join(PKG, "libkvq.so")
BUILD = os.path.join(ROOT, "_build")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC,-O2", "--expt-relaxed-constexpr",
         "-diag-suppress", "177", f"-I{os.path.join(ROOT, 'include')}"]
DIMS = (64, 128, 256)
BITS = (1, 2, 3, 4)


def _nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _sources():
    """(object name, source, extra flags) of every compile job."""
    jobs = [("api.o", "api.cu", []), ("decode.o", "decode.cu", []), ("decode_mma.o", "decode_mma.cu", [])]
    for d in DIMS:
        for b in BITS:
            jobs.append((f"quantize_d{d}_b{b}.o", "quantize_inst.cu", [f"-DKVQ_D={d}", f"-DKVQ_B={b}"]))
    return jobs


def _headers_digest() -> bytes:
    h = hashlib.sha256()
    for name in sorted(os.listdir(CSRC)):
        if name.endswith((".h", ".cuh")):
            with open(os.path.join(CSRC, name), "rb") as f:
                h.update(name.encode() + f.read())
    with open(os.path.join(ROOT, "include", "kvq.h"), "rb") as f:
        h.update(f.read())
    h.update(" ".join(ARCH + FLAGS).encode())
    return h.digest()


def _object_key(src: str, extra) -> str:
    h = hashlib.sha256(_headers_digest())
    with open(os.path.join(CSRC, src), "rb") as f:
        h.update(f.read())
    h.update(" ".join(extra).encode())
    return h.hexdigest()


def _fingerprint() -> str:
    h = hashlib.sha256()
    for obj, src, extra in _sources():
        h.update(_object_key(src, extra).encode())
    return h.hexdigest()


def build(force: bool = False, jobs: int | None = None, verbose: bool = False) -> str:
    """Compile and link libkvq.so if any source changed; returns its path."""
    os.makedirs(BUILD, exist_ok=True)
    stamp = os.path.join(BUILD, "libkvq.fingerprint")
    fp = _fingerprint()
    if not force and os.path.exists(OUT) and os.path.exists(stamp) and open(stamp).read() == fp:
        return OUT
    nvcc = _nvcc()
    objs = []

    def compile_one(job):
        obj, src, extra = job
        out = os.path.join(BUILD, obj)
        key = _object_key(src, extra)
        keyfile = out + ".key"
        if not force and os.path.exists(out) and os.path.exists(keyfile) and open(keyfile).read() == key:
            return out
        cmd = [nvcc, *ARCH, *FLAGS, *extra, "-c", os.path.join(CSRC, src), "-o", out]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"nvcc failed for {src} {' '.join(extra)}:\n{r.stderr}")
        if verbose and r.stderr.strip():
            print(r.stderr, file=sys.stderr)
        with open(keyfile, "w") as f:
            f.write(key)
        return out

    n = jobs or max(1, min(len(_sources()), os.cpu_count() or 4))
    with cf.ThreadPoolExecutor(max_workers=n) as ex:
        objs = list(ex.map(compile_one, _sources()))
    tmp = OUT + f".tmp{os.getpid()}"
    cmd = [nvcc, *ARCH, "-shared", "-cudart", "static", "-o", tmp, *objs]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"link failed:\n{r.stderr}")
    os.replace(tmp, OUT)
    with open(stamp, "w") as f:
        f.write(fp)
    return OUT


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("-j", type=int, default=None)
    ap.add_argument("-v", action="store_true")
    args = ap.parse_args()
    print(build(force=args.force, jobs=args.j, verbose=args.v))
