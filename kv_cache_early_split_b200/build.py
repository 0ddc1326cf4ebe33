"""Build the sm_100a shared library libart_decode.so in-tree with nvcc.

    python -m kv_cache_early_split_b200.build [--force]

The library exports the C ABI of include/art_decode.h.  nvcc cross-compiles
for sm_100a without a GPU.
"""
from __future__ import annotations

import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libart_decode.so")
# art_api.cu holds the C ABI and the CUDA-core kernels; art_tc_gp*.cu / art_tc_q8.cu the tensor-core
# instantiations (bf16 per head count, q8)
SOURCES = [os.path.join(CSRC, f) for f in ("art_api.cu", "art_tc_gp1.cu", "art_tc_gp2.cu", "art_tc_gp4.cu",
                                           "art_tc_gp8.cu", "art_tc_q8.cu")]
DEPS = SOURCES + [
    os.path.join(CSRC, f) for f in sorted(os.listdir(CSRC)) if f.endswith((".cuh", ".h"))
] + [os.path.join(INCLUDE, "art_decode.h")]

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC",
    "-Xcompiler", "-fvisibility=hidden",
    "-Xcompiler", "-fvisibility-inlines-hidden",
    "-Xptxas", "-v",
    "--expt-relaxed-constexpr",
]


def nvcc() -> str:
    for c in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if c and (os.path.sep not in c or os.path.exists(c)):
            return c
    return "nvcc"


# A test build of the same sources in which the tensor-core kernel's bounded waits give up after
# 1000 SM cycles (instead of about a second): every call aborts early and reports ART_ERR_TIMEOUT,
# which lets a test drive the timeout path without a hung copy.  The drains keep their long limit.
SHORT_WAIT_LIB = os.path.join(PKG, "libart_decode_shortwait.so")
SHORT_WAIT_FLAGS = ["-DART_TC_WAIT_LIMIT_CYCLES=1000LL"]


# The debug build: the same sources with the device index checks compiled in (ART_DCHECK): a failed
# check sets the status word's index bit and the call reports ART_ERR_INDEX -- no trap, no fault.
DEBUG_LIB = os.path.join(PKG, "libart_decode_debug.so")
DEBUG_FLAGS = ["-DART_DEBUG"]


def needs_build(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    return any(os.path.getmtime(d) > t for d in DEPS)


def build_short_wait(force: bool = False) -> str:
    """The short-wait test build (see SHORT_WAIT_FLAGS)."""
    return build(force=force, lib=SHORT_WAIT_LIB, extra_flags=SHORT_WAIT_FLAGS)


def build_debug(force: bool = False) -> str:
    """The debug build with device index checks (see DEBUG_FLAGS)."""
    return build(force=force, lib=DEBUG_LIB, extra_flags=DEBUG_FLAGS)


def build(force: bool = False, verbose: bool = False, lib: str = LIB, extra_flags=()) -> str:
    """Compile every source to an object (in parallel), then link the shared library."""
    from concurrent.futures import ThreadPoolExecutor

    if not force and not needs_build(lib):
        return lib
    tag = f".{os.path.basename(lib)[:-3]}.tmp{os.getpid()}"
    objs = [os.path.join(PKG, os.path.basename(src)[:-3] + tag + ".o") for src in SOURCES]
    cmds = [[nvcc(), *NVCC_FLAGS, *extra_flags, "-I", INCLUDE, "-I", CSRC, "-c", src, "-o", obj]
            for src, obj in zip(SOURCES, objs)]
    with ThreadPoolExecutor(len(cmds)) as ex:
        results = list(ex.map(lambda c: subprocess.run(c, capture_output=True, text=True), cmds))
    tmp = lib + tag
    link = [nvcc(), "-gencode", "arch=compute_100a,code=sm_100a", "-shared", *objs, "-o", tmp]
    if all(r.returncode == 0 for r in results):
        results.append(subprocess.run(link, capture_output=True, text=True))
        cmds.append(link)
    log = os.path.join(PKG, "build.log" if lib == LIB else os.path.basename(lib)[:-3] + ".build.log")
    with open(log, "w") as f:
        for c, r in zip(cmds, results):
            f.write(" ".join(c) + "\n" + r.stdout + r.stderr)
    for o in objs:
        if os.path.exists(o):
            os.remove(o)
    bad = [r for r in results if r.returncode != 0]
    if bad:
        sys.stderr.write(bad[0].stdout + bad[0].stderr)
        raise RuntimeError(f"nvcc failed (log: {log})")
    os.replace(tmp, lib)
    if verbose:
        sys.stdout.write("".join(r.stderr for r in results))
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
    if "--short-wait" in sys.argv:
        print(build_short_wait(force="--force" in sys.argv))
    if "--debug" in sys.argv:
        print(build_debug(force="--force" in sys.argv))
