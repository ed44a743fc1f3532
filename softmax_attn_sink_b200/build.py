"""Build libattn_sink.so in-tree with nvcc for sm_100a.

    python -m softmax_attn_sink_b200.build          # incremental
    python -m softmax_attn_sink_b200.build --force  # rebuild everything
    python -m softmax_attn_sink_b200.build --debug  # the bounds-checking debug library

Each ``csrc/*.cu`` compiles to an object under ``_build/`` (in parallel), then nvcc
links them into ``softmax_attn_sink_b200/libattn_sink.so`` with the CUDA runtime
linked statically, so the library needs nothing but the driver at run time.

``--debug`` builds the same sources with ``-DATTN_SINK_DEBUG`` into ``_build_debug/`` and
``libattn_sink_debug.so``: every global store of an output checks its index range against
the tensor it writes, skips a store that would leave it and sets bit 8 of the device status
word.  Load it instead of the release library by setting ``ATTN_SINK_LIBRARY`` to its path.
"""
from __future__ import annotations

import argparse
import concurrent.futures as cf
import glob
import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
OBJ = os.path.join(HERE, "_build")
LIB = os.path.join(HERE, "libattn_sink.so")
OBJ_DEBUG = os.path.join(HERE, "_build_debug")
LIB_DEBUG = os.path.join(HERE, "libattn_sink_debug.so")
INCLUDE = os.path.join(ROOT, "include")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "--expt-relaxed-constexpr",
         "-I", INCLUDE, "-I", CSRC]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _headers():
    return glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h")) + \
        glob.glob(os.path.join(INCLUDE, "*.h"))


def _stale(obj: str, src: str) -> bool:
    if not os.path.exists(obj):
        return True
    t = os.path.getmtime(obj)
    return any(os.path.getmtime(d) > t for d in [src] + _headers())


def _compile(src: str, obj: str, extra) -> str:
    cmd = [nvcc()] + ARCH + FLAGS + list(extra) + ["-c", src, "-o", obj]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed for {os.path.basename(src)}:\n{' '.join(cmd)}\n{r.stdout}{r.stderr}")
    return r.stderr


def build(force: bool = False, verbose: bool = False, extra=(), debug: bool = False) -> str:
    """Compile every CUDA source for sm_100a and link the shared library; returns its path.

    debug=True builds the bounds-checking library (``-DATTN_SINK_DEBUG``) beside the release one."""
    obj_dir, lib = (OBJ_DEBUG, LIB_DEBUG) if debug else (OBJ, LIB)
    if debug:
        extra = list(extra) + ["-DATTN_SINK_DEBUG"]
    os.makedirs(obj_dir, exist_ok=True)
    srcs = sorted(glob.glob(os.path.join(CSRC, "*.cu")))
    objs = [os.path.join(obj_dir, os.path.basename(s)[:-3] + ".o") for s in srcs]
    todo = [(s, o) for s, o in zip(srcs, objs) if force or _stale(o, s)]
    if todo:
        with cf.ThreadPoolExecutor(max_workers=min(8, len(todo))) as ex:
            futs = {ex.submit(_compile, s, o, extra): s for s, o in todo}
            for f in cf.as_completed(futs):
                msg = f.result()
                if verbose and msg.strip():
                    print(f"[{os.path.basename(futs[f])}]\n{msg}", file=sys.stderr)
    if todo or not os.path.exists(lib) or any(os.path.getmtime(o) > os.path.getmtime(lib) for o in objs):
        cmd = [nvcc()] + ARCH + ["-shared", "-cudart", "static", "-o", lib] + objs
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"link failed:\n{' '.join(cmd)}\n{r.stdout}{r.stderr}")
    return lib


def main() -> None:
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose", "-v", action="store_true", help="print ptxas resource usage")
    ap.add_argument("--debug", action="store_true", help="build the bounds-checking debug library")
    args = ap.parse_args()
    extra = ["-Xptxas", "-v"] if args.verbose else []
    print(build(force=args.force or args.verbose, verbose=args.verbose, extra=extra, debug=args.debug))


if __name__ == "__main__":
    main()
