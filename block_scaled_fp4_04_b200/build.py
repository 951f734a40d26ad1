"""Build libfp4.so in-tree with nvcc for sm_100a (B200).

``python -m block_scaled_fp4_04_b200.build`` compiles every ``csrc/*.cu`` translation
unit in parallel into ``_build/`` and links ``block_scaled_fp4_04_b200/libfp4.so``.
nvcc cross-compiles, so this works on a machine without a GPU.
"""
from __future__ import annotations

import concurrent.futures as cf
import hashlib
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
OUT = os.path.join(PKG, "libfp4.so")
BUILD = os.path.join(ROOT, "_build")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-Xcompiler", "-O2",
         f"-I{os.path.join(ROOT, 'include')}"]


def _nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if cand and (os.path.isabs(cand) and os.path.exists(cand) or not os.path.isabs(cand)):
            return cand
    return "nvcc"


def _sources():
    return sorted(os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith(".cu"))


def _flags_id(extra=()) -> str:
    """The build flags as text, without the checkout's location: the same tree builds
    the same library wherever it sits (a GPU machine runs it from a scratch path)."""
    inc = f"-I{os.path.join(ROOT, 'include')}"
    return " ".join("-I<repo>/include" if f == inc else f for f in ARCH + FLAGS + list(extra))


def _fingerprint(extra=()) -> str:
    h = hashlib.sha256()
    for d in (CSRC, os.path.join(ROOT, "include")):
        for f in sorted(os.listdir(d)):
            with open(os.path.join(d, f), "rb") as fh:
                h.update(f.encode() + fh.read())
    h.update(_flags_id(extra).encode())
    return h.hexdigest()


def sources_fingerprint(rel_paths, extra=()) -> str:
    """Fingerprint of one kernel's translation unit: the named files (paths relative to
    the package directory, e.g. "csrc/fp4_decode.cu") and the build flags.  Profiler
    counters recorded for that kernel stay valid while it is unchanged."""
    h = hashlib.sha256()
    for rel in sorted(rel_paths):
        with open(os.path.join(PKG, rel), "rb") as fh:
            h.update(rel.encode() + fh.read())
    h.update(_flags_id(extra).encode())
    return h.hexdigest()


def build(force: bool = False, verbose: bool = False, extra=()) -> str:
    """Compile and link libfp4.so unless it is up to date with the sources."""
    stamp = OUT + ".sha256"
    fp = _fingerprint(extra)
    if not force and os.path.exists(OUT) and os.path.exists(stamp):
        with open(stamp) as f:
            if f.read().strip() == fp:
                return OUT
    os.makedirs(BUILD, exist_ok=True)
    nvcc = _nvcc()

    def compile_one(src):
        obj = os.path.join(BUILD, os.path.basename(src)[:-3] + ".o")
        cmd = [nvcc, *ARCH, *FLAGS, *extra, "-c", src, "-o", obj]
        if verbose:
            cmd.insert(1, "-Xptxas=-v")
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"nvcc failed for {src}:\n{r.stderr}")
        if verbose:
            sys.stderr.write(r.stderr)
        return obj

    with cf.ThreadPoolExecutor(max_workers=os.cpu_count() or 4) as ex:
        objs = list(ex.map(compile_one, _sources()))
    tmp = OUT + f".tmp{os.getpid()}"
    r = subprocess.run([nvcc, *ARCH, "-shared", "-o", tmp, *objs], capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"link failed:\n{r.stderr}")
    os.replace(tmp, OUT)
    with open(stamp, "w") as f:
        f.write(fp)
    return OUT


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
