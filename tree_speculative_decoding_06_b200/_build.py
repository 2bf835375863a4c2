"""Build the CUDA library libtsd.so in-tree (nvcc, sm_100a only)."""
from __future__ import annotations

import hashlib
import os
import subprocess
from concurrent.futures import ThreadPoolExecutor

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
OBJ = os.path.join(PKG, "_build")
LIB = os.path.join(PKG, "libtsd.so")

NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC,-O2", "--expt-relaxed-constexpr",
         "-I", INCLUDE, "-I", CSRC]


def sources():
    return sorted(os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith(".cu"))


def _headers_digest() -> str:
    h = hashlib.sha256()
    for d in (CSRC, INCLUDE):
        for f in sorted(os.listdir(d)):
            if f.endswith((".h", ".cuh")):
                with open(os.path.join(d, f), "rb") as fh:
                    h.update(fh.read())
    return h.hexdigest()[:12]


def _compile(src: str, hdr: str, verbose: bool) -> str:
    with open(src, "rb") as f:
        tag = hashlib.sha256(f.read() + hdr.encode() + " ".join(FLAGS + ARCH).encode()).hexdigest()[:12]
    obj = os.path.join(OBJ, os.path.basename(src)[:-3] + f".{tag}.o")
    if not os.path.exists(obj):
        cmd = [NVCC, *ARCH, *FLAGS, "-c", src, "-o", obj + ".tmp"]
        if verbose:
            cmd += ["-Xptxas", "-v"]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"nvcc failed for {src}:\n{r.stdout}\n{r.stderr}")
        if verbose and r.stderr:
            print(r.stderr)
        os.replace(obj + ".tmp", obj)
    return obj


def build(verbose: bool = False) -> str:
    """Compile every csrc/*.cu for sm_100a and link libtsd.so; returns its path."""
    os.makedirs(OBJ, exist_ok=True)
    hdr = _headers_digest()
    with ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as ex:
        objs = list(ex.map(lambda s: _compile(s, hdr, verbose), sources()))
    stamp = hashlib.sha256("".join(sorted(objs)).encode()).hexdigest()[:12]
    stamp_file = LIB + ".stamp"
    if not (os.path.exists(LIB) and os.path.exists(stamp_file) and open(stamp_file).read() == stamp):
        tmp = LIB + f".{os.getpid()}.tmp"
        cmd = [NVCC, *ARCH, "-shared", "-Xcompiler", "-fPIC", "-o", tmp, *objs]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
        os.replace(tmp, LIB)
        with open(stamp_file, "w") as f:
            f.write(stamp)
    return LIB


if __name__ == "__main__":
    import sys
    print(build(verbose="-v" in sys.argv))
