"""Build libpa.so in-tree with nvcc for sm_100a.

    python paged_kv_cache_354_b200/_build.py [--force] [--verbose]

Objects go to ``_build/`` at the repository root; the shared library is
written next to this file, where the binding loads it.  Run it as a script
(or load it by path): importing the package first would load the library
this script is about to rebuild.
"""

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
OBJDIR = os.path.join(ROOT, "_build")
LIB = os.path.join(PKG, "libpa.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
COMMON = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC,-O3,-Wall", f"-I{INCLUDE}", f"-I{CSRC}"]


def nvcc():
    path = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(path):
        raise RuntimeError("nvcc not found: the CUDA toolkit is required to build libpa.so")
    return path


def _sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cpp")))


def _headers():
    return glob.glob(os.path.join(CSRC, "*.h")) + glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(
        os.path.join(INCLUDE, "*.h")
    )


def _stale(target, deps):
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(d) > t for d in deps)


def _compile(src, force, verbose, extra, objdir=OBJDIR):
    obj = os.path.join(objdir, os.path.basename(src) + ".o")
    if not force and not _stale(obj, [src, __file__] + _headers()):
        return obj
    cmd = [nvcc(), "-c", src, "-o", obj] + ARCH + COMMON + extra
    if src.endswith(".cu"):
        cmd += ["-Xptxas", "-v"] if verbose else []
    if verbose:
        print(" ".join(cmd), flush=True)
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError(f"nvcc failed on {src}:\n{res.stdout}\n{res.stderr}")
    if verbose and res.stderr:
        print(res.stderr, flush=True)
    return obj


def build(force=False, verbose=False, extra=(), lib=LIB, objdir=OBJDIR):
    """Compile every source under csrc/ and link a shared library (libpa.so
    next to this file unless ``lib`` says otherwise); returns its path.
    ``extra`` nvcc flags (e.g. -D tuning overrides) should go with their own
    ``lib`` and ``objdir``."""
    os.makedirs(objdir, exist_ok=True)
    srcs = _sources()
    with cf.ThreadPoolExecutor(max_workers=min(8, len(srcs))) as ex:
        objs = list(ex.map(lambda s: _compile(s, force, verbose, list(extra), objdir), srcs))
    if force or _stale(lib, objs):
        cmd = [nvcc(), "-shared", "-o", lib] + objs + ARCH + ["-Xcompiler", "-fPIC"]
        res = subprocess.run(cmd, capture_output=True, text=True)
        if res.returncode != 0:
            raise RuntimeError(f"link failed:\n{res.stdout}\n{res.stderr}")
    return lib


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__)
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose", action="store_true")
    args = ap.parse_args(argv)
    print(build(force=args.force, verbose=args.verbose))


if __name__ == "__main__":
    sys.exit(main())
