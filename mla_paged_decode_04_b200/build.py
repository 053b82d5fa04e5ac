"""Build libmla_decode.so in-tree with nvcc for sm_100a.

Every translation unit under csrc/ is compiled with
``-gencode arch=compute_100a,code=sm_100a -O3 -lineinfo -Xptxas -v`` and the
ptxas report is checked: any register spill in a kernel of this library fails
the build. The objects are linked into one shared library (static cudart).
Run ``python mla_paged_decode_04_b200/build.py`` (a plain script: it does not import
the package, whose import needs the built library) or call ``build()``.

``build(check=True)`` (``build.py --check``) builds the bounds-checking variant,
``libmla_decode_check.so``, from the same sources with ``-DMLA_BOUNDS_CHECK=1``:
its kernels test every global index against its buffer and set
MLA_DEV_BOUNDS instead of making an access outside it (``mla_bounds_checked()``
tells the two apart). It is for debugging, not for timing.
"""
from __future__ import annotations

import os
import re
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD_DIR = os.path.join(ROOT, "_build")
LIB_PATH = os.path.join(HERE, "libmla_decode.so")
CHECK_LIB_PATH = os.path.join(HERE, "libmla_decode_check.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-Xptxas", "-v",
              "--expt-relaxed-constexpr", "-I", INCLUDE, "-I", CSRC]


def _nvcc() -> str:
    cand = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(cand):
        raise RuntimeError("nvcc not found")
    return cand


def _sources():
    return sorted(os.path.join(CSRC, f) for f in os.listdir(CSRC)
                  if f.endswith(".cu") or f.endswith(".cpp"))


def _headers():
    hs = [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".h", ".cuh"))]
    hs.append(os.path.join(INCLUDE, "mla_decode.h"))
    return hs


_SPILL = re.compile(r"(\d+) bytes spill stores, (\d+) bytes spill loads")


def _check_spills(log: str, src: str) -> None:
    fn = None
    for line in log.splitlines():
        m = re.search(r"Compiling entry function '([^']+)'", line)
        if m:
            fn = m.group(1)
        m = _SPILL.search(line)
        if m and (int(m.group(1)) or int(m.group(2))):
            raise RuntimeError(f"register spill in {fn} ({os.path.basename(src)}): {line.strip()}")


def build(force: bool = False, verbose: bool = False, check: bool = False) -> str:
    build_dir = os.path.join(BUILD_DIR, "check") if check else BUILD_DIR
    lib_path = CHECK_LIB_PATH if check else LIB_PATH
    flags = NVCC_FLAGS + (["-DMLA_BOUNDS_CHECK=1"] if check else [])
    os.makedirs(build_dir, exist_ok=True)
    nvcc = _nvcc()
    newest_dep = max(os.path.getmtime(p) for p in _headers() + [__file__])
    objs = []
    changed = force or not os.path.exists(lib_path)
    for src in _sources():
        obj = os.path.join(build_dir, os.path.basename(src) + ".o")
        objs.append(obj)
        if (not force and os.path.exists(obj)
                and os.path.getmtime(obj) >= max(os.path.getmtime(src), newest_dep)):
            continue
        cmd = [nvcc, *ARCH, *flags, "-c", src, "-o", obj]
        if src.endswith(".cpp"):
            cmd = [nvcc, *ARCH, *flags, "-x", "c++", "-c", src, "-o", obj]
        r = subprocess.run(cmd, capture_output=True, text=True)
        log = r.stdout + r.stderr
        if r.returncode != 0:
            raise RuntimeError(f"nvcc failed for {src}:\n{log}")
        with open(obj + ".ptxas.txt", "w") as f:
            f.write(log)
        if verbose:
            print(log)
        _check_spills(log, src)
        changed = True
    if changed or os.path.getmtime(lib_path) < max(os.path.getmtime(o) for o in objs):
        tmp = lib_path + f".tmp{os.getpid()}"
        # static cudart; driver entry points are fetched at run time, so no -lcuda
        cmd = [nvcc, *ARCH, "-shared", "-o", tmp, *objs]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"link failed:\n{r.stdout}{r.stderr}")
        os.replace(tmp, lib_path)
    return lib_path


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv, check="--check" in sys.argv))
