"""Build liblbca.so in place: every csrc/*.cu compiled for sm_100a with nvcc.

    python -m block_compressed_long_b200.build [--force] [--verbose]

Objects go to _build/ at the repository root; the shared library lands next to
this file so that it travels with the package.  Rebuilds only when a source or
header is newer than the library.
"""
from __future__ import annotations

import argparse
import concurrent.futures as cf
import glob
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
OUT = os.path.join(PKG, "liblbca.so")
OBJ = os.path.join(ROOT, "_build")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
         "--expt-relaxed-constexpr", "-I", INCLUDE, "-I", CSRC]


def _nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


# The bounds-checked variant: every cache row range a decode kernel derives is
# tested against the cache's extent; a failure records LBCA_ERR_ARG on the
# status word and the access is moved inside the array (never a trap).  The
# binding loads it when LBCA_CHECKED=1 is set in the environment.
OUT_CHECKED = os.path.join(PKG, "liblbca_checked.so")


def _stale(out: str = OUT) -> bool:
    if not os.path.exists(out):
        return True
    t = os.path.getmtime(out)
    deps = sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h")) + \
        glob.glob(os.path.join(INCLUDE, "*.h"))
    return any(os.path.getmtime(p) > t for p in deps)


def build(force: bool = False, verbose: bool = False, checked: bool = False) -> str:
    out = OUT_CHECKED if checked else OUT
    if not force and not _stale(out):
        return out
    nvcc = _nvcc()
    objdir = os.path.join(OBJ, "checked") if checked else OBJ
    os.makedirs(objdir, exist_ok=True)
    extra = (["-Xptxas", "-v"] if verbose else []) + (["-DLBCA_CHECKED"] if checked else [])

    def compile_one(src):
        obj = os.path.join(objdir, os.path.basename(src) + ".o")
        cmd = [nvcc, *ARCH, *FLAGS, *extra, "-c", src, "-o", obj]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"nvcc failed on {src}:\n{r.stderr}")
        if verbose:
            sys.stderr.write(r.stderr)
        return obj

    with cf.ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as ex:
        objs = list(ex.map(compile_one, sources()))
    tmp = out + f".tmp{os.getpid()}"
    subprocess.check_call([nvcc, *ARCH, "-shared", "-o", tmp, *objs])
    os.replace(tmp, out)
    return out


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose", action="store_true")
    ap.add_argument("--checked", action="store_true", help="the bounds-checked variant")
    args = ap.parse_args()
    print(build(force=args.force, verbose=args.verbose, checked=args.checked))
