"""Build libtreedec.so in-tree for sm_100a with nvcc.

    python -m long_context_attention_td_b200.build [--force] [--verbose]

The library links the CUDA runtime statically, so it needs nothing from the
Python environment at run time; the Python binding loads it with ctypes.
"""
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libtreedec.so")
SOURCES = ["td_partial.cu", "td_combine.cu", "td_gqa_combine.cu", "td_gqa_keys.cu", "td_prefill.cu",
           "td_api.cu", "td_static.cu"]
HEADERS = ["td_internal.cuh", "td_device.cuh", "td_tc.cuh"]

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
    "--expt-relaxed-constexpr",
]


def _nvcc():
    home = os.environ.get("CUDA_HOME", "/usr/local/cuda")
    cand = os.path.join(home, "bin", "nvcc")
    return cand if os.path.exists(cand) else "nvcc"


def _inputs():
    files = [os.path.join(CSRC, s) for s in SOURCES + HEADERS]
    files.append(os.path.join(INCLUDE, "treedec.h"))
    files.append(os.path.abspath(__file__))
    return files


def up_to_date() -> bool:
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    return all(os.path.getmtime(f) <= t for f in _inputs())


def build(force: bool = False, verbose: bool = False) -> str:
    """Compile every source to an object in parallel, then link the library."""
    if not force and up_to_date():
        return LIB
    from concurrent.futures import ThreadPoolExecutor
    objdir = os.path.join(PKG, "_build")
    os.makedirs(objdir, exist_ok=True)
    tag = "%d" % os.getpid()

    def compile_one(src):
        obj = os.path.join(objdir, src + "." + tag + ".o")
        cmd = [_nvcc(), *NVCC_FLAGS, "-c", "-I", INCLUDE, "-I", CSRC, "-o", obj]
        if verbose:
            cmd += ["-Xptxas", "-v"]
        subprocess.run(cmd + [os.path.join(CSRC, src)], check=True)
        return obj

    with ThreadPoolExecutor(max_workers=min(len(SOURCES), os.cpu_count() or 1)) as ex:
        objs = list(ex.map(compile_one, SOURCES))
    tmp = LIB + ".tmp" + tag
    try:
        subprocess.run([_nvcc(), *NVCC_FLAGS, "-shared", "-o", tmp, *objs], check=True)
    finally:
        for o in objs:
            if os.path.exists(o):
                os.remove(o)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="--verbose" in sys.argv))
