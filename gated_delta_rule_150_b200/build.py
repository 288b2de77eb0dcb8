"""Build the CUDA library (libgdr.so) in-tree for sm_100a.

    python -m gated_delta_rule_150_b200.build

compiles every ``csrc/*.cu`` with nvcc into ``_build/libgdr.so`` next to this
file.  The library links the CUDA runtime statically, so it only needs the
driver at run time.
"""
from __future__ import annotations

import glob
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
OUT_DIR = os.path.join(HERE, "_build")
LIB = os.path.join(OUT_DIR, "libgdr.so")

NVCC_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17",
              "-Xcompiler", "-fPIC", "--expt-relaxed-constexpr"]


def _nvcc() -> str:
    cand = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    return cand if os.path.exists(cand) else "nvcc"


def sources(extra=()) -> list:
    return sorted(glob.glob(os.path.join(CSRC, "*.cu"))) + list(extra)


def _stale(lib: str, srcs) -> bool:
    if not os.path.exists(lib):
        return True
    deps = list(srcs) + glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h"))
    deps += glob.glob(os.path.join(ROOT, "include", "*.h"))
    t = os.path.getmtime(lib)
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, verbose: bool = False, out: str = LIB, extra=()) -> str:
    srcs = sources(extra)
    if not force and not _stale(out, srcs):
        return out
    os.makedirs(os.path.dirname(out), exist_ok=True)
    objs = []
    for src in srcs:
        obj = os.path.join(os.path.dirname(out), os.path.splitext(os.path.basename(src))[0] + ".o")
        cmd = [_nvcc(), *NVCC_FLAGS, "-I", os.path.join(ROOT, "include"), "-I", CSRC,
               "-c", src, "-o", obj]
        if verbose:
            cmd.insert(1, "-Xptxas=-v")
            print(" ".join(cmd), flush=True)
        subprocess.run(cmd, check=True)
        objs.append(obj)
    tmp = out + f".tmp{os.getpid()}"
    subprocess.run([_nvcc(), "-gencode", "arch=compute_100a,code=sm_100a", "-shared",
                    "-Xcompiler", "-fPIC", "-o", tmp, *objs], check=True)
    os.replace(tmp, out)
    return out


# A copy of the library for the bounded-wait test: the state-pass kernels wait,
# at their second chunk, for a barrier nothing arrives on, with a 1 ms limit,
# so that the timeout path (error word, drain, GDR_ERR_TIMEOUT) runs on demand.
# Everything else is the regular library's objects.
WAIT_TEST_LIB = os.path.join(OUT_DIR, "libgdr_waittest.so")
WAIT_TEST_DEFINES = ["-DGDR_TEST_WAIT_LIMIT_NS=1000000"]


def build_wait_test(force: bool = False) -> str:
    build()
    variant_src = os.path.join(CSRC, "state_pass.cu")
    if not force and not _stale(WAIT_TEST_LIB, sources()):
        return WAIT_TEST_LIB
    vdir = os.path.join(OUT_DIR, "waittest")
    os.makedirs(vdir, exist_ok=True)
    vobj = os.path.join(vdir, "state_pass.o")
    subprocess.run([_nvcc(), *NVCC_FLAGS, *WAIT_TEST_DEFINES, "-I", os.path.join(ROOT, "include"),
                    "-I", CSRC, "-c", variant_src, "-o", vobj], check=True)
    objs = [os.path.join(OUT_DIR, os.path.splitext(os.path.basename(src))[0] + ".o")
            for src in sources() if src != variant_src] + [vobj]
    tmp = WAIT_TEST_LIB + f".tmp{os.getpid()}"
    subprocess.run([_nvcc(), "-gencode", "arch=compute_100a,code=sm_100a", "-shared",
                    "-Xcompiler", "-fPIC", "-o", tmp, *objs], check=True)
    os.replace(tmp, WAIT_TEST_LIB)
    return WAIT_TEST_LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
    if "--wait-test" in sys.argv:
        print(build_wait_test(force="--force" in sys.argv))
