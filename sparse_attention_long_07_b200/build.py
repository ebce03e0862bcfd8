"""Build libdsa.so (the C-ABI library) in-tree with nvcc for sm_100a.

    python sparse_attention_long_07_b200/build.py [--force] [--profile-waits] [--checked]

--checked builds libdsa_checked.so instead: the same kernels compiled with
-DDSA_DEBUG, whose device-side bounds checks record an error and skip any
access outside its buffer (loaded when DSA_LIBRARY_VARIANT=checked).

Run it by path (or load it with load_builder()): importing the package itself
loads the library, which is what this script produces.
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(HERE, "libdsa.so")
LIB_CHECKED = os.path.join(HERE, "libdsa_checked.so")
SOURCES = [os.path.join(CSRC, "dsa.cu")]
DEPS = SOURCES + [os.path.join(CSRC, f) for f in os.listdir(CSRC)] + [os.path.join(INCLUDE, "dsa.h")]

NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17", "--expt-relaxed-constexpr",
    "-Xcompiler", "-fPIC", "-shared", "-cudart", "static",
    "-Xptxas", "-v",
]


def stale(target: str = LIB) -> bool:
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(p) > t for p in DEPS if os.path.exists(p))


def build(force: bool = False, verbose: bool = False, profile_waits: bool = False, checked: bool = False) -> str:
    """Compile libdsa.so.  profile_waits=True adds the per-wait-site cycle
    counters read by dsa_debug_wait_profile (a diagnostic build, not for
    timing); checked=True compiles libdsa_checked.so with the device-side
    bounds checks."""
    target = LIB_CHECKED if checked else LIB
    if not force and not stale(target):
        return target
    tmp = target + f".tmp{os.getpid()}"
    extra = (["-DDSA_PROFILE_WAITS"] if profile_waits else []) + (["-DDSA_DEBUG"] if checked else [])
    cmd = [NVCC, *FLAGS, *extra, "-I", INCLUDE, "-I", CSRC, *SOURCES, "-o", tmp, "-ldl", "-lrt", "-lpthread"]
    res = subprocess.run(cmd, capture_output=True, text=True)
    log = os.path.join(HERE, "build_checked.log" if checked else "build.log")
    with open(log, "w") as f:
        f.write(" ".join(cmd) + "\n" + res.stdout + res.stderr)
    if res.returncode != 0:
        sys.stderr.write(res.stdout + res.stderr)
        raise RuntimeError(f"nvcc failed (see {log})")
    if verbose:
        sys.stdout.write(res.stdout + res.stderr)
    os.replace(tmp, target)
    return target


if __name__ == "__main__":
    print(build(force="--force" in sys.argv or "--profile-waits" in sys.argv, verbose=True,
                profile_waits="--profile-waits" in sys.argv, checked="--checked" in sys.argv))
