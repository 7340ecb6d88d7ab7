"""Build libbcq.so (the sm_100a kernels behind the C ABI of include/bcq.h)
in-tree, next to this file, with nvcc.

Each translation unit of csrc/ is compiled to an object under _build/ (in
parallel; an object is rebuilt only when its source or a header it includes
changed), then the objects are linked.  The CUDA runtime is linked
statically and its symbols are kept private to the library, so the
process's other CUDA users (torch) are not affected.
"""
from __future__ import annotations

import glob
import os
import re
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
OBJ = os.path.join(ROOT, "_build", "libbcq")
LIB = os.path.join(HERE, "libbcq.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
CFLAGS = ["-O3", "-std=c++17", "-lineinfo", "--expt-relaxed-constexpr",
          "-Xcompiler", "-fPIC", "-Xcompiler", "-Wall"]
LFLAGS = ["-Xlinker", "--exclude-libs,ALL", "-Xlinker", "-Bsymbolic"]


def sources() -> list[str]:
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _includes(path: str, seen: set) -> set:
    """Local headers (csrc/, include/) that `path` includes, transitively."""
    try:
        text = open(path).read()
    except OSError:
        return seen
    for name in re.findall(r'#include\s+"([^"]+)"', text):
        for d in (CSRC, INCLUDE):
            h = os.path.join(d, name)
            if os.path.exists(h) and h not in seen:
                seen.add(h)
                _includes(h, seen)
                break
    return seen


def _obj_of(src: str) -> str:
    return os.path.join(OBJ, os.path.basename(src)[:-3] + ".o")


def _stale(target: str, deps) -> bool:
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(d) > t for d in deps)


def _compile(nvcc: str, src: str, verbose: bool) -> str:
    obj = _obj_of(src)
    tmp = obj + f".tmp{os.getpid()}"
    cmd = [nvcc, *ARCH, *CFLAGS, "-I", INCLUDE, "-I", CSRC, "-c", src, "-o", tmp]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
        print(" ".join(cmd), flush=True)
    subprocess.run(cmd, check=True)
    os.replace(tmp, obj)
    return obj


def build(force: bool = False, verbose: bool = False) -> str:
    nvcc = os.environ.get("NVCC", "nvcc")
    os.makedirs(OBJ, exist_ok=True)
    srcs = sources()
    todo = [s for s in srcs if force or _stale(_obj_of(s), [s, *_includes(s, set())])]
    if todo:
        with ThreadPoolExecutor(max_workers=len(todo)) as ex:
            list(ex.map(lambda s: _compile(nvcc, s, verbose), todo))
    objs = [_obj_of(s) for s in srcs]
    if force or _stale(LIB, objs):
        tmp = LIB + f".tmp{os.getpid()}"
        subprocess.run([nvcc, *ARCH, *LFLAGS, "-shared", "-o", tmp, *objs], check=True)
        os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
