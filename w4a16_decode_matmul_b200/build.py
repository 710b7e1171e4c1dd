"""Build the CUDA library ``libwq.so`` in-tree for sm_100a.

    python w4a16_decode_matmul_b200/build.py [--force] [--verbose] [--jobs N]

(run as a script: importing the package loads the library it builds)

Each ``csrc/*.cu`` file (the C ABI in ``wq.cu`` and one translation unit per
kernel family) is compiled to a relocatable object in parallel, and the
objects are device-linked into one shared library.  An object is rebuilt
only when its source or a header it includes has changed.
"""
from __future__ import annotations

import argparse
import concurrent.futures
import glob
import os
import re
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIBRARY = os.path.join(HERE, "libwq.so")
OBJ_DIR = os.path.join(ROOT, "_build", "obj")
LOG = os.path.join(HERE, "ptxas.log")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
COMPILE_FLAGS = [*ARCH, "-O3", "-lineinfo", "-std=c++17", "-rdc=true",
                 "-Xcompiler", "-fPIC", "-Xptxas", "-v"]
LINK_FLAGS = [*ARCH, "-rdc=true", "-shared", "-Xcompiler", "-fPIC"]

_INCLUDE_RE = re.compile(r'^\s*#\s*include\s+"([^"]+)"', re.M)


def _nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if cand and (os.path.sep not in cand or os.path.exists(cand)):
            return cand
    raise RuntimeError("nvcc not found")


def units() -> list[str]:
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def sources() -> list[str]:
    return sorted(units() + glob.glob(os.path.join(CSRC, "*.cuh"))
                  + glob.glob(os.path.join(CSRC, "*.h")) + glob.glob(os.path.join(INCLUDE, "*.h")))


def dependencies(path: str, seen: set | None = None) -> set:
    """The file and every local header it includes, transitively."""
    seen = set() if seen is None else seen
    if path in seen or not os.path.exists(path):
        return seen
    seen.add(path)
    text = open(path, encoding="utf-8").read()
    for name in _INCLUDE_RE.findall(text):
        for d in (os.path.dirname(path), CSRC, INCLUDE):
            cand = os.path.join(d, name)
            if os.path.exists(cand):
                dependencies(cand, seen)
                break
    return seen


def _obj(unit: str) -> str:
    return os.path.join(OBJ_DIR, os.path.basename(unit)[:-3] + ".o")


def _stale(unit: str) -> bool:
    obj = _obj(unit)
    if not os.path.exists(obj):
        return True
    t = os.path.getmtime(obj)
    return any(os.path.getmtime(d) > t for d in dependencies(unit))


def up_to_date() -> bool:
    if not os.path.exists(LIBRARY):
        return False
    t = os.path.getmtime(LIBRARY)
    return (all(os.path.getmtime(s) <= t for s in sources())
            and not any(_stale(u) for u in units()))


def _compile(unit: str) -> tuple[str, int, str]:
    obj = _obj(unit)
    tmp = obj + f".tmp{os.getpid()}"
    cmd = [_nvcc(), *COMPILE_FLAGS, "-I", INCLUDE, "-I", CSRC, "-c", unit, "-o", tmp]
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode == 0:
        os.replace(tmp, obj)
    return unit, res.returncode, res.stdout + res.stderr


def build(force: bool = False, verbose: bool = False, jobs: int | None = None) -> str:
    if not force and up_to_date():
        return LIBRARY
    os.makedirs(OBJ_DIR, exist_ok=True)
    todo = [u for u in units() if force or _stale(u)]
    jobs = jobs or min(len(todo) or 1, os.cpu_count() or 4)
    logs, failed = [], []
    with concurrent.futures.ThreadPoolExecutor(max_workers=jobs) as ex:
        for unit, rc, log in ex.map(_compile, todo):
            logs.append(f"==== {os.path.basename(unit)}\n{log}")
            if rc != 0:
                failed.append(unit)
    if todo:
        with open(LOG, "w") as f:
            f.write("\n".join(logs))
    if failed:
        sys.stderr.write("\n".join(logs))
        raise RuntimeError("nvcc failed on " + ", ".join(os.path.basename(u) for u in failed))
    tmp = LIBRARY + f".tmp{os.getpid()}"
    cmd = [_nvcc(), *LINK_FLAGS, *[_obj(u) for u in units()], "-o", tmp]
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        sys.stderr.write(res.stdout + res.stderr)
        raise RuntimeError("nvcc failed linking libwq.so")
    if verbose:
        sys.stdout.write("\n".join(logs))
    os.replace(tmp, LIBRARY)
    return LIBRARY


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose", action="store_true")
    ap.add_argument("--jobs", type=int, default=None)
    a = ap.parse_args()
    print(build(force=a.force, verbose=a.verbose, jobs=a.jobs))
