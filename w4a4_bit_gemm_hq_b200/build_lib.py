"""Build step of libhq: compiles the CUDA sources under csrc/ for sm_100a into
``libhq.so`` beside this file (in-tree, so the library travels with the repo)."""
import os
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libhq.so")
SOURCES = ["abi.cu", "rotate.cu", "rotq.cu", "pack.cu", "gemm.cu", "gemm_small.cu", "noalloc.cu", "calib.cu", "mxfp4.cu"]
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo", "-O3", "-std=c++17",
         "-Xcompiler", "-fPIC", "--expt-relaxed-constexpr", "-Xptxas", "-v"]


def _stale():
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    deps = [os.path.join(CSRC, f) for f in os.listdir(CSRC)]
    deps.append(os.path.join(HERE, "..", "include", "hq.h"))
    return any(os.path.getmtime(d) > t for d in deps)


def build(force=False, verbose=False):
    if not force and not _stale():
        return LIB
    bdir = os.path.join(HERE, "_build")
    os.makedirs(bdir, exist_ok=True)
    objs = [os.path.join(bdir, src.replace(".cu", ".o")) for src in SOURCES]
    # an object is rebuilt when it is older than its source or any header
    headers = [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".cuh", ".h"))]
    headers.append(os.path.join(HERE, "..", "include", "hq.h"))
    t_hdr = max(os.path.getmtime(h) for h in headers)
    todo = [i for i, src in enumerate(SOURCES)
            if force or not os.path.exists(objs[i])
            or os.path.getmtime(objs[i]) < max(t_hdr, os.path.getmtime(os.path.join(CSRC, src)))]

    def compile_one(i):
        cmd = [NVCC, *FLAGS, "-rdc=true", "-c", os.path.join(CSRC, SOURCES[i]), "-o", objs[i]]
        return subprocess.run(cmd, capture_output=True, text=True)

    # the sources compile independently: all at once
    with ThreadPoolExecutor(max_workers=max(1, len(todo))) as ex:
        results = list(ex.map(compile_one, todo))
    for src, r in zip([SOURCES[i] for i in todo], results):
        if verbose or r.returncode:
            sys.stderr.write(r.stdout + r.stderr)
        if r.returncode:
            raise RuntimeError("nvcc failed on " + src)
    tmp = LIB + ".tmp%d" % os.getpid()
    cmd = [NVCC, "-gencode", "arch=compute_100a,code=sm_100a", "-shared", "-rdc=true", *objs, "-o", tmp,
           "-lcudart"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode:
        sys.stderr.write(r.stdout + r.stderr)
        raise RuntimeError("link failed")
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
