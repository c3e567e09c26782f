"""Build libnvfp4.so (the CUDA kernels and the C ABI) in-tree for sm_100a.

    python -m nvfp4_microscaling_quantization_b200.build [--force] [-v]

nvcc cross-compiles for sm_100a without a GPU.  Each translation unit is
compiled to an object file of its own (in parallel), then the objects are
linked into the shared library.  The library is built with -fmad=false (no
contraction of a multiply and an add) and IEEE division, reciprocal and
subnormals, so its binary32 steps round as written.
"""
import concurrent.futures
import glob
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
OUT = os.path.join(PKG, "libnvfp4.so")
OBJ_DIR = os.path.join(PKG, "_build")

NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
COMPILE_FLAGS = [
    "-O3", "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo",
    "-fmad=false", "-prec-div=true", "-prec-sqrt=true", "-ftz=false",
    "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
    "-I", INCLUDE, "-I", CSRC,
]
LINK_FLAGS = ["-shared", "-cudart", "static", "-gencode", "arch=compute_100a,code=sm_100a"]


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _deps():
    return glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h")) + \
        glob.glob(os.path.join(INCLUDE, "*.h")) + [os.path.abspath(__file__)]


def _stale():
    if not os.path.exists(OUT):
        return True
    t = os.path.getmtime(OUT)
    return any(os.path.getmtime(d) > t for d in sources() + _deps())


def _compile(src, verbose):
    obj = os.path.join(OBJ_DIR, os.path.basename(src)[:-3] + ".o")
    flags = list(COMPILE_FLAGS) + (["-Xptxas", "-v"] if verbose else [])
    r = subprocess.run([NVCC, *flags, "-c", src, "-o", obj], capture_output=True, text=True)
    return src, obj, r


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and not _stale():
        return OUT
    os.makedirs(OBJ_DIR, exist_ok=True)
    srcs = sources()
    workers = max(1, min(len(srcs), os.cpu_count() or 1))
    objs, failed = [], []
    with concurrent.futures.ThreadPoolExecutor(max_workers=workers) as pool:
        for src, obj, r in pool.map(lambda s: _compile(s, verbose), srcs):
            if r.stdout:
                sys.stdout.write(r.stdout)
            if r.stderr:
                sys.stderr.write(r.stderr)
            if r.returncode != 0:
                failed.append(src)
            objs.append(obj)
    if failed:
        raise subprocess.CalledProcessError(1, f"nvcc -c {' '.join(os.path.basename(f) for f in failed)}")
    subprocess.run([NVCC, *LINK_FLAGS, *objs, "-o", OUT + ".tmp"], check=True)
    os.replace(OUT + ".tmp", OUT)
    return OUT


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
