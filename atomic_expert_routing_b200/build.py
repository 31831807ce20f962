"""Build libomnimoe.so (the C-ABI CUDA library) in-tree for sm_100a with nvcc."""
from __future__ import annotations

import glob
import os
import re
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(os.path.dirname(HERE), "include")
LIB = os.path.join(HERE, "libomnimoe.so")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def sources() -> list[str]:
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


OBJ = os.path.join(HERE, "_build")


def _headers() -> list[str]:
    return (glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h")) +
            glob.glob(os.path.join(INCLUDE, "*.h")))


def _obj(src: str) -> str:
    return os.path.join(OBJ, os.path.basename(src)[:-3] + ".o")


def report(src: str) -> str:
    """ptxas resource report (registers, spills, shared memory per kernel) of
    the last compile of ``src``."""
    return os.path.join(OBJ, os.path.basename(src)[:-3] + ".ptxas.txt")


_RESOURCE_LINE = re.compile(r"^(ptxas info\s*:|\s+\d+ bytes stack frame)")


def _stale_obj(src: str, newest_header: float) -> bool:
    o = _obj(src)
    if not os.path.exists(o):
        return True
    t = os.path.getmtime(o)
    return os.path.getmtime(src) > t or newest_header > t


def _stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    return any(os.path.getmtime(p) > t for p in sources() + _headers())


def build(force: bool = False, verbose_ptxas: bool = False) -> str:
    """Compile each source to an object (in parallel, only those out of date)
    and link the shared library."""
    if not force and not _stale():
        return LIB
    from concurrent.futures import ThreadPoolExecutor

    nvcc = os.environ.get("NVCC", "nvcc")
    os.makedirs(OBJ, exist_ok=True)
    newest = max((os.path.getmtime(h) for h in _headers()), default=0.0)
    todo = [s for s in sources() if force or _stale_obj(s, newest)]

    def compile_one(src: str) -> None:
        o = _obj(src)
        tmp = o + f".tmp{os.getpid()}"
        cmd = [nvcc, *ARCH, "-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC",
               "-Xptxas=-v", "-I", INCLUDE, "-c", "-o", tmp, src]
        r = subprocess.run(cmd, capture_output=True, text=True)
        # the resource lines go to the report; anything else (warnings,
        # errors) is shown as the compiler printed it
        other = "".join(ln for ln in r.stderr.splitlines(True) if not _RESOURCE_LINE.match(ln))
        sys.stderr.write(r.stdout + (r.stderr if verbose_ptxas else other))
        if r.returncode != 0:
            raise subprocess.CalledProcessError(r.returncode, cmd)
        with open(report(src), "w") as fh:
            fh.write(r.stderr)
        os.replace(tmp, o)

    with ThreadPoolExecutor(max_workers=max(1, min(len(todo), os.cpu_count() or 1))) as ex:
        list(ex.map(compile_one, todo))
    tmp = LIB + f".tmp{os.getpid()}"
    subprocess.run([nvcc, *ARCH, "-shared", "-o", tmp, *[_obj(s) for s in sources()]], check=True)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose_ptxas="-v" in sys.argv))
