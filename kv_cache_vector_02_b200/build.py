"""Build libtq.so (CUDA sm_100a + host C++) in-tree with nvcc.

    python -m kv_cache_vector_02_b200.build [--force] [--verbose]
    TQ_DEBUG=1 python -m kv_cache_vector_02_b200.build --force   # with device invariant checks

Every .cu / .cpp under csrc/ is compiled to an object under _build/ (in
parallel) and linked into kv_cache_vector_02_b200/libtq.so with a static CUDA
runtime.  Objects are rebuilt when their source or any header is newer.
"""
from __future__ import annotations

import argparse
import concurrent.futures as cf
import os
import subprocess
import sys
from pathlib import Path

PKG = Path(__file__).resolve().parent
CSRC = PKG / "csrc"
OBJ = PKG / "_build"
LIB = PKG / "libtq.so"
INCLUDE = PKG.parent / "include"

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
COMMON = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC,-fvisibility=hidden", "-I", str(INCLUDE)]
# TQ_DEBUG=1 in the environment: device-side invariant checks (index bounds of slots,
# rows and pages), each setting TQ_DEVERR_INTERNAL instead of touching memory out of
# range.  Build with --force when switching.
if os.environ.get("TQ_DEBUG", "") not in ("", "0"):
    COMMON += ["-DTQ_DEBUG"]


def _nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if cand and (os.path.isabs(cand) and os.path.exists(cand) or not os.path.isabs(cand)):
            return cand
    return "nvcc"


def _headers():
    return list(CSRC.glob("*.h")) + list(CSRC.glob("*.cuh")) + list(INCLUDE.glob("*.h"))


def _compile(src: Path, verbose: bool) -> Path:
    obj = OBJ / (src.name + ".o")
    cmd = [_nvcc(), *ARCH, *COMMON, "-c", str(src), "-o", str(obj)]
    if src.suffix == ".cu":
        cmd += ["--expt-relaxed-constexpr"]
        if verbose:
            cmd += ["-Xptxas", "-v"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError("nvcc failed for %s:\n%s\n%s" % (src.name, r.stdout, r.stderr))
    if verbose and r.stderr:
        sys.stderr.write(r.stderr)
    return obj


def build(force: bool = False, verbose: bool = False) -> Path:
    OBJ.mkdir(exist_ok=True)
    sources = sorted(CSRC.glob("*.cu")) + sorted(CSRC.glob("*.cpp"))
    newest_header = max((h.stat().st_mtime for h in _headers()), default=0.0)
    todo = []
    for s in sources:
        o = OBJ / (s.name + ".o")
        if force or not o.exists() or o.stat().st_mtime < max(s.stat().st_mtime, newest_header):
            todo.append(s)
    if todo:
        with cf.ThreadPoolExecutor(max_workers=min(8, len(todo))) as ex:
            list(ex.map(lambda s: _compile(s, verbose), todo))
    objs = [OBJ / (s.name + ".o") for s in sources]
    if force or todo or not LIB.exists() or LIB.stat().st_mtime < max(o.stat().st_mtime for o in objs):
        tmp = LIB.with_name("libtq.so.tmp%d" % os.getpid())
        cmd = [_nvcc(), *ARCH, "-shared", "--cudart", "static", "-o", str(tmp), *map(str, objs)]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError("link failed:\n%s\n%s" % (r.stdout, r.stderr))
        os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose", action="store_true", help="print ptxas register / spill reports")
    args = ap.parse_args()
    print(build(force=args.force, verbose=args.verbose))
