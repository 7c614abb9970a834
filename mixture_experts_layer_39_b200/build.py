"""Builds libmoe.so in-tree from csrc/*.cu for sm_100a.

    python -m mixture_experts_layer_39_b200.build [--jobs N] [--force]

Each translation unit is compiled to an object under <repo>/_build/ (only
when its sources changed) and the objects are linked into
mixture_experts_layer_39_b200/libmoe.so next to this file.  The CUDA runtime
is linked statically, so the library needs only the driver at run time.
"""
from __future__ import annotations

import argparse
import concurrent.futures as cf
import glob
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
BUILD = os.path.join(ROOT, "_build")
LIB = os.path.join(HERE, "libmoe.so")

NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
    "-I", os.path.join(ROOT, "include"),
]


def _headers():
    return glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(ROOT, "include", "*.h"))


STAMP = os.path.join(BUILD, "flags.txt")


def _flags_stamp():
    """The compiler and flags the objects are built with: objects built with
    another compiler or other flags are stale whatever their times."""
    try:
        ver = subprocess.run([NVCC, "--version"], capture_output=True, text=True).stdout.strip()
    except OSError:
        ver = "nvcc not found"
    return "\n".join([NVCC, ver, *FLAGS]) + "\n"


def _stale(obj, src, headers):
    if not os.path.exists(obj):
        return True
    t = os.path.getmtime(obj)
    return any(os.path.getmtime(p) > t for p in [src, *headers])


def _compile(src, obj):
    cmd = [NVCC, *FLAGS, "-c", src, "-o", obj]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed on {os.path.basename(src)}:\n{r.stdout}\n{r.stderr}")
    return obj


def build(jobs: int = 8, force: bool = False, verbose: bool = False) -> str:
    os.makedirs(BUILD, exist_ok=True)
    headers = _headers()
    sources = sorted(glob.glob(os.path.join(CSRC, "*.cu")))
    objs = [os.path.join(BUILD, os.path.basename(s)[:-3] + ".o") for s in sources]
    stamp = _flags_stamp()
    if not os.path.exists(STAMP) or open(STAMP).read() != stamp:
        force = True
    todo = [(s, o) for s, o in zip(sources, objs) if force or _stale(o, s, headers)]
    if todo:
        with cf.ThreadPoolExecutor(max_workers=jobs) as ex:
            for o in ex.map(lambda so: _compile(*so), todo):
                if verbose:
                    print("compiled", os.path.relpath(o, ROOT))
    if force or todo or not os.path.exists(LIB) or any(
            os.path.getmtime(o) > os.path.getmtime(LIB) for o in objs):
        cmd = [NVCC, "-gencode", "arch=compute_100a,code=sm_100a", "-shared", "-o", LIB, *objs,
               "-Xcompiler", "-fPIC"]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
        if verbose:
            print("linked", os.path.relpath(LIB, ROOT))
    with open(STAMP, "w") as fh:
        fh.write(stamp)
    return LIB


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--jobs", type=int, default=os.cpu_count() or 4)
    ap.add_argument("--force", action="store_true")
    a = ap.parse_args(argv)
    print(build(a.jobs, a.force, verbose=True))


if __name__ == "__main__":
    sys.exit(main())
