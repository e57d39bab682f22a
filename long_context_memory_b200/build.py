"""Build libmsa.so (the C-ABI library) in-tree with nvcc for sm_100a."""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
SOURCES = ["msa_api.cu", "route.cu", "route_static.cu", "attend.cu", "encode.cu", "aux_loss.cu", "tiered.cu"]
LIB = os.path.join(HERE, "libmsa.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")


def needs_build() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    deps = [os.path.join(CSRC, f) for f in os.listdir(CSRC)] + [os.path.join(ROOT, "include", "msa.h")]
    return any(os.path.getmtime(p) > t for p in deps)


def build(verbose: bool = False, ptxas_verbose: bool = False) -> str:
    """Compile every source to an object in parallel (relocatable device code), then link libmsa.so."""
    import concurrent.futures as cf
    import tempfile

    flags = [NVCC, "-O3", "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo", "-rdc=true",
             "-Xcompiler", "-fPIC", "-I", os.path.join(ROOT, "include")]
    if ptxas_verbose:
        flags += ["-Xptxas", "-v"]
    with tempfile.TemporaryDirectory(prefix="msa_build_") as tmp:
        objs = [os.path.join(tmp, os.path.splitext(src)[0] + ".o") for src in SOURCES]
        cmds = [flags + ["-c", os.path.join(CSRC, src), "-o", obj] for src, obj in zip(SOURCES, objs)]
        if verbose:
            for c in cmds:
                print(" ".join(c), flush=True)
        with cf.ThreadPoolExecutor(max_workers=len(cmds)) as ex:
            results = list(ex.map(lambda c: subprocess.run(c, capture_output=True, text=True), cmds))
        for r in results:
            if r.returncode != 0:
                sys.stderr.write(r.stdout + r.stderr)
                raise RuntimeError("nvcc failed building libmsa.so")
            if verbose or ptxas_verbose:
                sys.stderr.write(r.stderr)
        link = [NVCC, "-gencode", "arch=compute_100a,code=sm_100a", "-rdc=true", "-shared", "-Xcompiler", "-fPIC",
                "-cudart", "static", "-o", LIB] + objs
        if verbose:
            print(" ".join(link), flush=True)
        r = subprocess.run(link, capture_output=True, text=True)
        if r.returncode != 0:
            sys.stderr.write(r.stdout + r.stderr)
            raise RuntimeError("nvcc failed linking libmsa.so")
    return LIB


if __name__ == "__main__":
    build(verbose=True, ptxas_verbose="-v" in sys.argv)
    print(LIB)
