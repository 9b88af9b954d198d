"""Build the CUDA library libgqa_b200.so in-tree for sm_100a (nvcc, no GPU needed).

    python -m attention_gqa_decode_b200.build [--verbose-ptxas]

Each source compiles to its own object in parallel; the objects are linked
into the shared library.  A second library, libgqa_b200_waittest.so, is built
from the same sources with GQA_WAIT_TEST defined: its internal waits give up
after a millisecond instead of a second, and its producers can be told
(gqa_test_set_stall) to leave their first stage unloaded, so that a test can
watch a bounded wait run out and the kernel return GQA_ERR_TIMEOUT.  Only the
tests load it.
"""
from __future__ import annotations

import os
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
SOURCES = ["api.cu", "decode.cu", "decode_split.cu", "prefill.cu", "mla.cu", "mla_tc.cu"]
HEADERS = ["common.cuh"]
LIB = os.path.join(PKG, "libgqa_b200.so")
WAITTEST_LIB = os.path.join(PKG, "libgqa_b200_waittest.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
OBJ_DIR = os.path.join(PKG, "_build")

FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17", "--use_fast_math",
    "-Xcompiler", "-fPIC,-O2",
    "-I", os.path.join(ROOT, "include"),
]


def _stale(lib: str) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    deps = [os.path.join(CSRC, f) for f in SOURCES + HEADERS] + [os.path.join(ROOT, "include", "gqa.h"), __file__]
    return any(os.path.getmtime(d) > t for d in deps)


def _compile(src: str, obj: str, defines, verbose_ptxas: bool) -> None:
    cmd = [NVCC] + FLAGS + [f"-D{d}" for d in defines] + (["-Xptxas", "-v"] if verbose_ptxas else []) + \
        ["-c", "-o", obj, os.path.join(CSRC, src)]
    subprocess.check_call(cmd)


def _build_one(lib: str, tag: str, defines, verbose_ptxas: bool) -> str:
    os.makedirs(OBJ_DIR, exist_ok=True)
    objs = [os.path.join(OBJ_DIR, f"{os.path.splitext(s)[0]}.{tag}.{os.getpid()}.o") for s in SOURCES]
    try:
        with ThreadPoolExecutor(max_workers=len(SOURCES)) as ex:
            for f in [ex.submit(_compile, s, o, defines, verbose_ptxas) for s, o in zip(SOURCES, objs)]:
                f.result()
        tmp = lib + f".tmp{os.getpid()}"
        subprocess.check_call([NVCC, "-gencode", "arch=compute_100a,code=sm_100a", "-shared", "-o", tmp] + objs)
        os.replace(tmp, lib)
    finally:
        for o in objs:
            if os.path.exists(o):
                os.remove(o)
    return lib


def build(force: bool = False, verbose_ptxas: bool = False, waittest: bool = True) -> str:
    """Build libgqa_b200.so (and, unless waittest=False, the test variant) if stale."""
    jobs = []
    if force or verbose_ptxas or _stale(LIB):
        jobs.append((LIB, "lib", [], verbose_ptxas))
    if waittest and (force or _stale(WAITTEST_LIB)):
        jobs.append((WAITTEST_LIB, "waittest", ["GQA_WAIT_TEST"], False))
    with ThreadPoolExecutor(max_workers=2) as ex:
        for f in [ex.submit(_build_one, *j) for j in jobs]:
            f.result()
    return LIB


if __name__ == "__main__":
    print(build(force=True, verbose_ptxas="--verbose-ptxas" in sys.argv))
