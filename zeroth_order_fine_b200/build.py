"""Build libzo_b200.so in-tree for sm_100a (nvcc; no JIT, no torch extension).

Each translation unit under csrc/ is compiled to an object under _build/
(rebuilt only when it or a header changed, earlier builds kept by content) and linked into
zeroth_order_fine_b200/libzo_b200.so, which the Python binding loads.  `--debug` builds
libzo_b200_debug.so instead: the same sources with ZO_DEBUG defined (device bounds checks),
loaded when ZO_LIB=debug.
"""
from __future__ import annotations

import concurrent.futures as cf
import glob
import hashlib
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
OUT = os.path.join(HERE, "libzo_b200.so")
OUT_DEBUG = os.path.join(HERE, "libzo_b200_debug.so")
BUILD = os.path.join(ROOT, "_build")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "-Xcompiler", "-O3",
         "--expt-relaxed-constexpr", "-I" + os.path.join(ROOT, "include")]


def _headers_digest() -> str:
    h = hashlib.sha256()
    for f in sorted(glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h"))
                    + glob.glob(os.path.join(ROOT, "include", "*.h"))):
        with open(f, "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def _compile(src: str, hdr: str, flags: list, verbose: bool) -> str:
    with open(src, "rb") as fh:
        tag = hashlib.sha256(fh.read() + hdr.encode() + " ".join(flags).encode()).hexdigest()[:16]
    obj = os.path.join(BUILD, os.path.basename(src) + "." + tag + ".o")
    if os.path.exists(obj):
        return obj
    cmd = [NVCC] + ARCH + flags + ["-c", src, "-o", obj]
    if src.endswith(".cpp"):
        cmd = [NVCC] + flags + ["-x", "cu"] + ARCH + ["-c", src, "-o", obj]
    if verbose:
        print(" ".join(cmd), flush=True)
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed on {src}:\n{r.stdout}\n{r.stderr}")
    return obj


def build(verbose: bool = False, debug: bool = False) -> str:
    os.makedirs(BUILD, exist_ok=True)
    srcs = sorted(glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cpp")))
    hdr = _headers_digest()
    flags = FLAGS + (["-DZO_DEBUG"] if debug else [])
    out = OUT_DEBUG if debug else OUT
    with cf.ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as ex:
        objs = list(ex.map(lambda s: _compile(s, hdr, flags, verbose), srcs))
    # relink whenever the set of objects differs from the one the library was linked from
    # (going back to an earlier source picks up its cached, older object)
    stamp = os.path.join(BUILD, os.path.basename(out) + ".objects")
    linked = "\n".join(os.path.basename(o) for o in objs) + "\n"
    if os.path.exists(out) and os.path.exists(stamp):
        with open(stamp) as fh:
            if fh.read() == linked:
                return out
    cmd = [NVCC] + ARCH + ["-shared", "-o", out + ".tmp"] + objs + ["-lcudart_static", "-ldl", "-lrt", "-lpthread"]
    if verbose:
        print(" ".join(cmd), flush=True)
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
    os.replace(out + ".tmp", out)
    with open(stamp, "w") as fh:
        fh.write(linked)
    return out


if __name__ == "__main__":
    print(build(verbose="-v" in sys.argv, debug="--debug" in sys.argv))
