"""Build libkvarn.so in-tree with nvcc for sm_100a.

    python -m bit_kv_cache_15_b200.build [--force]

The library is written next to this file; `kvarn.py` loads it from there.
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libkvarn.so")
SOURCES = ["kvarn_api.cu", "quantize.cu", "decode.cu", "baseline.cu"]
HEADERS = ["common.cuh", "kvarn_internal.h", "quant_tile.cuh"]

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "--std=c++17",
    "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
    "--expt-relaxed-constexpr",
    "-Xptxas", "-v",
]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _inputs():
    files = [os.path.join(CSRC, s) for s in SOURCES + HEADERS]
    files.append(os.path.join(ROOT, "include", "kvarn.h"))
    return files


def up_to_date() -> bool:
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    return all(os.path.getmtime(f) <= t for f in _inputs())


# A test-only variant of the library: the decode's first copy of one warp
# never arrives and the copy waits give up after 2^10 polls, so a test can
# check that the kernel returns KVARN_DEV_TIMEOUT and leaves the device usable.
STALL_LIB = os.path.join(HERE, "libkvarn_stalltest.so")
STALL_DEFINES = ["-DKVARN_TEST_STALL_FIRST_UNIT=1", "-DKVARN_WAIT_LIMIT_LOG2=10"]

# The debug variant: the same kernels with their own index arithmetic checked
# on the device (a failed check reports KVARN_DEV_INTERNAL and skips the
# access).  Tests run it against the release library on the same inputs.
DEBUG_LIB = os.path.join(HERE, "libkvarn_debug.so")
DEBUG_DEFINES = ["-DKVARN_DEBUG=1"]


def _compile(src: str, obj: str, defines, verbose: bool) -> None:
    cmd = [nvcc(), *NVCC_FLAGS, *defines, "-I", os.path.join(ROOT, "include"), "-c", os.path.join(CSRC, src),
           "-o", obj]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        sys.stderr.write(r.stdout + r.stderr)
        raise RuntimeError(f"nvcc failed on {src}")
    if verbose:
        sys.stderr.write(r.stderr)


def _link(objs, lib: str) -> None:
    tmp = lib + ".tmp"
    cmd = [nvcc(), "-gencode", "arch=compute_100a,code=sm_100a", "-shared", "-Xcompiler", "-fPIC",
           "-o", tmp, *objs]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        sys.stderr.write(r.stdout + r.stderr)
        raise RuntimeError("link failed")
    os.replace(tmp, lib)


def _fresh(lib: str) -> bool:
    if not os.path.exists(lib):
        return False
    t = os.path.getmtime(lib)
    return all(os.path.getmtime(f) <= t for f in _inputs())


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and up_to_date() and _fresh(STALL_LIB) and _fresh(DEBUG_LIB):
        return LIB
    objdir = os.path.join(HERE, "_build")
    os.makedirs(objdir, exist_ok=True)
    objs = [os.path.join(objdir, src.replace(".cu", ".o")) for src in SOURCES]
    debug_objs = [os.path.join(objdir, src.replace(".cu", "_debug.o")) for src in SOURCES]
    stall_obj = os.path.join(objdir, "decode_stalltest.o")
    jobs = [(src, obj, []) for src, obj in zip(SOURCES, objs)]
    jobs += [(src, obj, DEBUG_DEFINES) for src, obj in zip(SOURCES, debug_objs)]
    jobs.append(("decode.cu", stall_obj, STALL_DEFINES))
    # the nvcc runs are independent: run them side by side
    with ThreadPoolExecutor(max_workers=min(len(jobs), os.cpu_count() or 1)) as ex:
        for f in [ex.submit(_compile, src, obj, defines, verbose) for src, obj, defines in jobs]:
            f.result()
    _link(objs, LIB)
    _link([stall_obj if o.endswith(os.sep + "decode.o") else o for o in objs], STALL_LIB)
    _link(debug_objs, DEBUG_LIB)
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose="-v" in sys.argv)
    print(LIB)
