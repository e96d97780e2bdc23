"""The software exponent ("FlashAttention 4" page, software exponent on CUDA
cores: part of the 2^x evaluations run as a polynomial on the FMA pipe instead
of the MUFU unit) under the bf16 forward's full parity suite.

The product library computes every exponential with MUFU ex2 (the split was
slower on B200 at every share measured); the cubic stays a compile-time
option, so this test builds the library with it switched on -- one of every
four element pairs from the cubic at d = 128, two of four at d = 64 -- and
runs tests/test_fwd_gpu.py against that build in a child process
(TILEDATTN_LIB).  The cubic's relative error (7.5e-5, tests/test_exp2_poly.py)
is far below bf16's 2^-9 rounding of P, so the same tolerances apply.
"""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_forward_parity_with_the_cubic_exponent(cuda_lib):
    from tiled_attention_24_b200 import build
    lib = os.path.join(build.PKG, "libtiledattn_poly.so")
    build.build(force=True, out=lib, defines=["TA_POLY_PAIRS=1", "TA_POLY_PAIRS_D64=2"])
    env = dict(os.environ)
    env["TILEDATTN_LIB"] = lib
    r = subprocess.run([sys.executable, "-m", "pytest", os.path.join("tests", "test_fwd_gpu.py"), "-m", "gpu", "-x",
                        "-q", "-p", "no:cacheprovider"], env=env, cwd=ROOT, capture_output=True, text=True,
                       timeout=1200)
    tail = r.stdout[-3000:] + r.stderr[-2000:]
    print(tail)
    assert r.returncode == 0, tail
