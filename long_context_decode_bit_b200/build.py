"""Build ``libfathom.so`` (the CUDA kernels and the C ABI) in-tree for sm_100a.

``python -m long_context_decode_bit_b200.build [--force] [--ptxas-v] [--test-hooks]``

``--test-hooks`` builds ``libfathom_testhooks.so`` instead: the same sources
with a short ring-wait poll limit, the device-side bounds checks of
``FATHOM_DEBUG_BOUNDS`` (a failed check sets the fault word's bounds bit and
skips the access; ``fathom_device_status`` then returns FATHOM_ERR_BOUNDS),
and two switches for tests: ``FATHOM_TEST_WITHHOLD_ARRIVAL=1`` makes the
scan withhold one ring arrival (a bounded wait runs out), and
``FATHOM_TEST_SHRINK_CAP=1`` makes the checks allow only half of the
candidate entries (a check fails).  The product never loads it.
"""
from __future__ import annotations

import glob
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libfathom.so")
TEST_LIB = os.path.join(PKG, "libfathom_testhooks.so")
# about 65k polls of at most ~1 us each: tens of ms, far above any normal wait
TEST_DEFINES = ["-DFATHOM_TEST_HOOKS", "-DFATHOM_SPIN_LIMIT=65536", "-DFATHOM_DEBUG_BOUNDS"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc() -> str:
    for c in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", shutil.which("nvcc")):
        if c and os.path.exists(c):
            return c
    raise RuntimeError("nvcc not found")


def sources() -> list[str]:
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _stale(lib: str) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    deps = sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + [os.path.join(INCLUDE, "fathom.h")]
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, ptxas_verbose: bool = False, test_hooks: bool = False) -> str:
    lib = TEST_LIB if test_hooks else LIB
    if not force and not _stale(lib):
        return lib
    cmd = [nvcc(), "-O3", "-std=c++17", *ARCH, "-lineinfo", "-shared", "-Xcompiler", "-fPIC",
           "-I", INCLUDE, "-I", CSRC, *(TEST_DEFINES if test_hooks else []), "-o", lib, *sources()]
    if ptxas_verbose:
        cmd.insert(1, "-Xptxas=-v")
    subprocess.run(cmd, check=True)
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, ptxas_verbose="--ptxas-v" in sys.argv,
                test_hooks="--test-hooks" in sys.argv))
