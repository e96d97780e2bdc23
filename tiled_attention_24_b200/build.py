"""Build libtiledattn.so (the attention library), libtiledattn_debug.so (the
same with bounds checks and counters, TA_DEBUG = 1) and libtiledattn_probe.so
(the throughput microbenchmarks behind the roofline denominators) in-tree
with nvcc for sm_100a.

    python -m tiled_attention_24_b200.build [--verbose]

The library links the CUDA runtime statically, so it loads (and exports its
symbols) on a machine without a GPU driver; the driver is only needed when a
call reaches the device.
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libtiledattn.so")
SOURCES = ["api.cu"]
PROBE_LIB = os.path.join(PKG, "libtiledattn_probe.so")
DEBUG_LIB = os.path.join(PKG, "libtiledattn_debug.so")
PROBE_SOURCES = ["probe.cu"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc_path() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _deps():
    files = [os.path.join(CSRC, f) for f in os.listdir(CSRC)]
    files += [os.path.join(INCLUDE, f) for f in os.listdir(INCLUDE)]
    files.append(os.path.abspath(__file__))
    return files


def up_to_date(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return False
    t = os.path.getmtime(lib)
    return all(os.path.getmtime(f) <= t for f in _deps())


def build_probe(verbose: bool = False, force: bool = False) -> str:
    """Compile libtiledattn_probe.so (include/tiledattn_probe.h)."""
    if not force and up_to_date(PROBE_LIB):
        return PROBE_LIB
    return build(verbose=verbose, force=True, out=PROBE_LIB, sources=PROBE_SOURCES)


def build_debug(verbose: bool = False, force: bool = False) -> str:
    """Compile libtiledattn_debug.so: the same library with TA_DEBUG = 1 (bounds
    checks of every TMA coordinate and tensor-memory address, counters read by
    attn_debug_counters)."""
    if not force and up_to_date(DEBUG_LIB):
        return DEBUG_LIB
    return build(verbose=verbose, force=True, out=DEBUG_LIB, defines=["TA_DEBUG=1"])


def build(verbose: bool = False, force: bool = False, out: str | None = None, defines=(),
          sources=None) -> str:
    """Compile libtiledattn.so (or `out`, with extra -D `defines`, for tuning
    sweeps of compile-time kernel parameters; `sources` for another library
    of this package)."""
    lib = out or LIB
    if not force and out is None and not defines and up_to_date():
        return LIB
    cmd = [nvcc_path(), *ARCH, "-lineinfo", "-O3", "-std=c++17", "-shared", "-Xcompiler", "-fPIC",
           "-Xcompiler", "-fvisibility=hidden", "--expt-relaxed-constexpr",
           "-I", INCLUDE, "-I", CSRC, "-o", lib + ".tmp"]
    cmd += ["-D" + d for d in defines]
    if verbose:
        cmd += ["-Xptxas", "-v"]
    cmd += [os.path.join(CSRC, s) for s in (sources or SOURCES)]
    res = subprocess.run(cmd, capture_output=True, text=True)
    if verbose or res.returncode != 0:
        sys.stderr.write(res.stdout + res.stderr)
    if res.returncode != 0:
        raise RuntimeError("nvcc failed (%d)" % res.returncode)
    os.replace(lib + ".tmp", lib)
    return lib


if __name__ == "__main__":
    import argparse
    ap = argparse.ArgumentParser()
    ap.add_argument("--verbose", action="store_true")
    ap.add_argument("--out", default=None)
    ap.add_argument("-D", dest="defines", action="append", default=[])
    a = ap.parse_args()
    print(build(verbose=a.verbose, force=True, out=a.out, defines=a.defines))
    if a.out is None and not a.defines:
        print(build_probe(verbose=a.verbose, force=True))
        print(build_debug(verbose=a.verbose, force=True))
