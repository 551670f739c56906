"""Builds libssd.so in-tree for sm_100a with nvcc (no GPU needed to build).

    python -m structured_state_space_fwd_b200.build [--force] [--verbose-ptxas]

Each .cu under csrc/ compiles to an object in _build/, objects are linked
into structured_state_space_fwd_b200/libssd.so with the CUDA runtime linked
statically. A second library, libssd_testhooks.so, differs only in the C ABI
layer, compiled with SSD_TEST_HOOKS: it honours SSD_TEST_STALL_CHAIN=1, which
makes the single-pass kernel's chain waits run out so that tests can check the
device-side timeout path. The shipped libssd.so has no such hook. The build is
skipped when both libraries are newer than every source.
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
BUILD = os.path.join(PKG, "_build")
LIB = os.path.join(PKG, "libssd.so")
TEST_LIB = os.path.join(PKG, "libssd_testhooks.so")
# the translation unit that reads the test hook
HOOKED = "ssd_api.cu"

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC,-O3,-fvisibility=hidden",
         "--expt-relaxed-constexpr", "-I", INCLUDE, "-I", CSRC]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", shutil.which("nvcc")):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: libssd needs the CUDA toolkit to build")


def sources() -> list[str]:
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _deps() -> list[str]:
    return (sources() + glob.glob(os.path.join(CSRC, "*.h")) + glob.glob(os.path.join(CSRC, "*.cuh"))
            + glob.glob(os.path.join(INCLUDE, "*.h")) + [os.path.abspath(__file__)])


def up_to_date() -> bool:
    if not (os.path.exists(LIB) and os.path.exists(TEST_LIB)):
        return False
    t = min(os.path.getmtime(LIB), os.path.getmtime(TEST_LIB))
    return all(os.path.getmtime(p) <= t for p in _deps())


def build(force: bool = False, verbose_ptxas: bool = False) -> str:
    if not force and up_to_date():
        return LIB
    os.makedirs(BUILD, exist_ok=True)
    cc = nvcc()
    procs = []
    objs = []
    test_objs = []
    jobs = [(src, os.path.join(BUILD, os.path.basename(src).replace(".cu", ".o")), []) for src in sources()]
    for src in sources():
        if os.path.basename(src) == HOOKED:
            jobs.append((src, os.path.join(BUILD, "testhooks_" + os.path.basename(src).replace(".cu", ".o")),
                         ["-DSSD_TEST_HOOKS=1"]))
    for src, obj, extra in jobs:
        if extra:
            test_objs.append(obj)
        else:
            objs.append(obj)
        cmd = [cc, *ARCH, *FLAGS, *extra, "-c", src, "-o", obj]
        if verbose_ptxas:
            cmd += ["-Xptxas", "-v"]
        procs.append((src, subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.STDOUT)))
    failed = []
    for src, p in procs:
        out, _ = p.communicate()
        if out:
            sys.stderr.write(out.decode())
        if p.returncode != 0:
            failed.append(src)
    if failed:
        raise RuntimeError(f"nvcc failed for {failed}")
    tmp = LIB + f".tmp{os.getpid()}"
    subprocess.check_call([cc, *ARCH, "-shared", "-cudart", "static", "-o", tmp, *objs])
    os.replace(tmp, LIB)
    hooked = [o for o in objs if os.path.basename(o) != HOOKED.replace(".cu", ".o")] + test_objs
    tmp = TEST_LIB + f".tmp{os.getpid()}"
    subprocess.check_call([cc, *ARCH, "-shared", "-cudart", "static", "-o", tmp, *hooked])
    os.replace(tmp, TEST_LIB)
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose_ptxas="--verbose-ptxas" in sys.argv)
    print(LIB)
