"""Builds libdsa_b200.so (the CUDA kernels and the C ABI of include/dsa.h)
in place, for sm_100a."""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
LIB_PATH = os.path.join(HERE, "libdsa_b200.so")
SOURCES = [os.path.join(CSRC, "dsa_lib.cu")]
# the benchmark's L2 bandwidth and FP8 tensor-rate probes: a separate library,
# not part of the ABI
PROBE_SOURCE = os.path.join(CSRC, "probe_l2.cu")
PROBE_PATH = os.path.join(HERE, "libdsa_probe.so")
DEPS = SOURCES + [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith(".cuh")] + [
    os.path.join(ROOT, "include", "dsa.h")]

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
    "-shared", "-cudart", "static",
]


def nvcc() -> str:
    cand = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    return cand if os.path.exists(cand) else "nvcc"


def build_probe(force: bool = False) -> str:
    deps = (PROBE_SOURCE, os.path.join(CSRC, "ptx.cuh"))
    if (not force and os.path.exists(PROBE_PATH)
            and os.path.getmtime(PROBE_PATH) >= max(os.path.getmtime(d) for d in deps)):
        return PROBE_PATH
    tmp = PROBE_PATH + f".tmp{os.getpid()}"
    subprocess.check_call([nvcc(), *NVCC_FLAGS, "-o", tmp, PROBE_SOURCE])
    os.replace(tmp, PROBE_PATH)
    return PROBE_PATH


def build(force: bool = False, verbose_ptxas: bool = False) -> str:
    build_probe(force)
    if (not force and os.path.exists(LIB_PATH)
            and os.path.getmtime(LIB_PATH) >= max(os.path.getmtime(d) for d in DEPS)):
        return LIB_PATH
    tmp = LIB_PATH + f".tmp{os.getpid()}"
    cmd = [nvcc(), *NVCC_FLAGS, "-I", os.path.join(ROOT, "include"), "-I", CSRC,
           *(["-Xptxas", "-v"] if verbose_ptxas else []), "-o", tmp, *SOURCES]
    subprocess.check_call(cmd)
    os.replace(tmp, LIB_PATH)
    return LIB_PATH


if __name__ == "__main__":
    print(build(force=True, verbose_ptxas="-v" in sys.argv))
