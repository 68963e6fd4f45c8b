"""Build libgdnq.so (the CUDA kernels + C ABI) in-tree for sm_100a with nvcc.

    python -m bit_recurrent_state_gdn_b200.build [--force] [--ptxas-info]

Objects go to ``bit_recurrent_state_gdn_b200/_build/``; the shared library lands next to this
file, where the Python binding loads it from.
"""
from __future__ import annotations

import concurrent.futures as cf
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
OBJ_DIR = os.path.join(PKG, "_build")
LIB = os.path.join(PKG, "libgdnq.so")
SOURCES = ["api.cu", "window_int8.cu", "window_int4.cu", "window_mixed.cu", "window_int8_smooth.cu",
           "window_int4_smooth.cu", "baseline.cu",
           "pw.cu", "prefill.cu"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _flags(ptxas_info: bool) -> list[str]:
    f = ARCH + ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC,-O2",
                "-I", INCLUDE, "-I", CSRC, "--expt-relaxed-constexpr"]
    if ptxas_info:
        f += ["-Xptxas", "-v"]
    return f


def _deps() -> list[str]:
    files = [os.path.join(CSRC, n) for n in os.listdir(CSRC)]
    return files + [os.path.join(INCLUDE, n) for n in ("gdnq.h", "gdnq_pw.h", "gdnq_prefill.h")]


def _stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    return any(os.path.getmtime(p) > t for p in _deps())


def build(force: bool = False, ptxas_info: bool = False, verbose: bool = False) -> str:
    if not force and not ptxas_info and not _stale():
        return LIB
    os.makedirs(OBJ_DIR, exist_ok=True)
    import fcntl

    with open(os.path.join(OBJ_DIR, ".lock"), "w") as lock:  # one builder at a time
        fcntl.flock(lock, fcntl.LOCK_EX)
        if not force and not ptxas_info and not _stale():
            return LIB
        return _build_locked(ptxas_info, verbose)


def _build_locked(ptxas_info: bool, verbose: bool) -> str:
    cc = nvcc()
    flags = _flags(ptxas_info)

    def compile_one(src: str) -> tuple[str, str]:
        obj = os.path.join(OBJ_DIR, src.replace(".cu", ".o"))
        cmd = [cc, *flags, "-c", os.path.join(CSRC, src), "-o", obj]
        res = subprocess.run(cmd, capture_output=True, text=True)
        if res.returncode != 0:
            raise RuntimeError(f"nvcc failed on {src}:\n{res.stdout}\n{res.stderr}")
        return obj, res.stdout + res.stderr

    with cf.ThreadPoolExecutor(max_workers=len(SOURCES)) as ex:
        results = list(ex.map(compile_one, SOURCES))
    if verbose or ptxas_info:
        for _, log in results:
            if log.strip():
                print(log)
    tmp = LIB + ".tmp"
    cmd = [cc, *ARCH, "-shared", "-o", tmp, *[o for o, _ in results], "-lcudart_static", "-lrt",
           "-lpthread", "-ldl"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, ptxas_info="--ptxas-info" in sys.argv,
                verbose="-v" in sys.argv))
