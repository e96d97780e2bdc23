"""Static limits of the warp-specialised kernels, checked on the CPU.

1. Register hand-over (`setmaxnreg`): warpgroup 0 (producer, MMA issuer and
   two idle warps) drops to REG_LOW and the two softmax warpgroups rise to
   REG_HIGH.  An increase that the registers given back cannot cover waits
   forever, so 128 * REG_LOW + 256 * REG_HIGH must fit in the registers the
   block is launched with (384 threads x 168: 65536 / 384 rounded down to a
   multiple of 8), and both values must be multiples of 8 in [24, 256].
2. The compiled headline kernels spill nothing: ptxas's resource report for
   fwd_bf16_kernel<128> (dense and variable-length) shows no spill stores.
"""
import os
import re
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "tiled_attention_24_b200", "csrc")


def _src(name):
    with open(os.path.join(CSRC, name)) as f:
        return f.read()


def _eval_reg(expr, D):
    # "72" or "(D == 64) ? 72 : 80"
    m = re.fullmatch(r"\s*\(D == (\d+)\) \? (\d+) : (\d+)\s*", expr)
    if m:
        return int(m.group(2)) if D == int(m.group(1)) else int(m.group(3))
    return int(expr)


@pytest.mark.parametrize("name,dims", [("fwd_bf16.cuh", (64, 128)), ("fwd_fp4.cuh", (128,)), ("fwd_fp8.cuh", (128,))])
def test_setmaxnreg_split_fits_the_launch(name, dims):
    s = _src(name)
    threads = int(re.search(r"static constexpr int THREADS = (\d+);", s).group(1))
    m = re.search(r"static constexpr int REG_LOW = ([^,]+), REG_HIGH = ([^;]+);", s)
    assert m, name
    assert threads == 384 and "__launch_bounds__(384, 1)" in s
    launch = (65536 // threads) // 8 * 8
    for D in dims:
        low, high = _eval_reg(m.group(1), D), _eval_reg(m.group(2), D)
        for r in (low, high):
            assert r % 8 == 0 and 24 <= r <= 256, (name, D, r)
        assert low <= launch <= high
        assert 128 * low + 256 * high <= threads * launch, (name, D, low, high)


@pytest.mark.skipif(shutil.which("nvcc") is None and not os.path.exists("/usr/local/cuda/bin/nvcc"),
                    reason="nvcc not available")
def test_headline_forward_compiles_without_spills(tmp_path):
    from tiled_attention_24_b200 import build
    cmd = [build.nvcc_path(), *build.ARCH, "-O3", "-std=c++17", "--expt-relaxed-constexpr", "-Xptxas", "-v",
           "-I", os.path.join(ROOT, "include"), "-I", CSRC, "-c", os.path.join(CSRC, "api.cu"),
           "-o", str(tmp_path / "api.o")]
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    log = r.stdout + r.stderr
    found = 0
    for m in re.finditer(r"Function properties for (\S+)\n\s*(\d+) bytes stack frame, (\d+) bytes spill stores", log):
        if m.group(1).startswith("_ZN2ta15fwd_bf16_kernelILi128E"):
            found += 1
            assert int(m.group(3)) == 0, (m.group(1), m.group(3))
    assert found == 2  # dense and variable-length instances
