"""Builds libwmtp.so in-tree with nvcc for sm_100a (B200).

    python -m long_context_speculative_kv_b200.build [--force] [--verbose-ptxas]
"""
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libwmtp.so")
SOURCES = [os.path.join(CSRC, "capi.cu")]
DEPS = SOURCES + [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".cuh", ".h"))] + [
    os.path.join(INCLUDE, f) for f in os.listdir(INCLUDE) if f.endswith(".h")]

NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
    "-shared",
    "-I", INCLUDE, "-I", CSRC,
]


def _stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    return any(os.path.getmtime(p) > t for p in DEPS)


def build(force: bool = False, ptxas_verbose: bool = False, defines=()) -> str:
    """Compiles libwmtp.so (``defines``: extra -D options, e.g. the kernel-selection thresholds
    of capi.cu for measurement sweeps)."""
    if not force and not defines and not _stale():
        return LIB
    cmd = [NVCC] + FLAGS + (["-Xptxas", "-v"] if ptxas_verbose else []) + [f"-D{d}" for d in defines] + \
        ["-o", LIB + ".tmp"] + SOURCES
    subprocess.run(cmd, check=True)
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, ptxas_verbose="--verbose-ptxas" in sys.argv,
                defines=[a[2:] for a in sys.argv[1:] if a.startswith("-D")]))
