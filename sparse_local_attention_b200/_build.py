"""Build libsta.so in-tree with nvcc for sm_100a (no JIT, no torch extension)."""
from __future__ import annotations

import os
import subprocess
from concurrent.futures import ThreadPoolExecutor

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
LIB = os.path.join(PKG, "libsta.so")
SOURCES = ["sta_api.cpp", "sta_permute.cu", "sta_fwd.cu", "sta_bwd.cu", "sta_noalloc.cu"]
HEADERS = ["sm100_ptx.cuh", "sta_kernels.h", "sta_common.cuh"]
NVCC_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-std=c++17", "-lineinfo",
              "-Xcompiler", "-fPIC", "--cudart", "shared", "-Xptxas", "-v"]


def _nvcc() -> str:
    cand = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    return cand if os.path.exists(cand) else "nvcc"


def sources():
    return [os.path.join(CSRC, s) for s in SOURCES if os.path.exists(os.path.join(CSRC, s))]


def _stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    deps = sources() + [os.path.join(CSRC, h) for h in HEADERS] + [os.path.join(ROOT, "include", "sta.h")]
    return any(os.path.getmtime(d) > t for d in deps if os.path.exists(d))


def compile_command(src: str, obj: str) -> list:
    """nvcc command that compiles one source of the library to an object."""
    return [_nvcc(), *NVCC_FLAGS, "-I", os.path.join(ROOT, "include"), "-c", src, "-o", obj]


def link_command(objs, out: str) -> list:
    """nvcc command that links the objects into a shared library."""
    return [_nvcc(), "-gencode", "arch=compute_100a,code=sm_100a", "--cudart", "shared", "-shared", "-o", out, *objs]


def objects() -> dict:
    """{source name: object path} of the last build."""
    return {os.path.basename(s): os.path.join(PKG, "_build", os.path.basename(s) + ".o") for s in sources()}


def build(force: bool = False, verbose: bool = False) -> str:
    """Compile every source under csrc/ into sparse_local_attention_b200/libsta.so."""
    if not force and not _stale():
        return LIB
    objdir = os.path.join(PKG, "_build")
    os.makedirs(objdir, exist_ok=True)

    def compile_one(src):
        obj = os.path.join(objdir, os.path.basename(src) + ".o")
        return src, obj, subprocess.run(compile_command(src, obj), capture_output=True, text=True)

    # the translation units are independent: compile them side by side
    with ThreadPoolExecutor(max_workers=max(1, min(len(SOURCES), os.cpu_count() or 1))) as ex:
        results = list(ex.map(compile_one, sources()))
    objs = []
    for src, obj, r in results:
        if r.returncode != 0:
            raise RuntimeError(f"nvcc failed on {src}:\n{r.stdout}\n{r.stderr}")
        if verbose:
            print(r.stderr)
        objs.append(obj)
    tmp = LIB + ".tmp"
    cmd = link_command(objs, tmp)
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force=True, verbose=True))
