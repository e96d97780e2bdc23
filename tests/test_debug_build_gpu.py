"""The debug build (libtiledattn_debug.so: the same kernels compiled with
TA_DEBUG = 1) on the GPU, in child processes that load it through
TILEDATTN_LIB.

1. Its counters against the oracle.  The lazy rescale ("FlashAttention 4"
   page, smarter online softmax rescaling: the reference max moves only when a
   key block's max exceeds it by more than 8 in log2 units) is counted per
   query row and key block by the bf16 forward; the oracle's deferred form
   with the same threshold and 128-key blocks counts the same moves.  A row
   whose block max came within 1e-3 of the threshold may decide either way in
   the kernel's fp32 logits; every later move of such a row may then differ
   too, so the two totals may differ by at most the remaining blocks of those
   rows.  The causal forward counts the key tiles a CTA never visits: with
   128-row query tiles and 128-key tiles these are exactly the all-masked
   blocks of the causal mask (key j visible to query i iff j <= i + Nkv - Nq),
   counted here from the mask itself.
2. No launch of any kernel family records a bounds violation: every TMA
   coordinate and tensor-memory address passes the checks (the counter and
   the status word both stay clean).
3. The whole GPU suite passes against the debug build (tests/conftest.py
   then also fails a test whose launches recorded a bounds violation).
"""
import json
import os
import subprocess
import sys

import numpy as np
import pytest

from oracle import attention as A
from tests import _debug_child as C

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
BAND = 1e-3  # log2 units: closer than this to the threshold, fp32 logits may decide either way


@pytest.fixture(scope="module")
def debug_env(cuda_lib):
    from tiled_attention_24_b200 import build
    env = dict(os.environ)
    env["TILEDATTN_LIB"] = build.build_debug()
    return env


@pytest.fixture(scope="module")
def child(debug_env):
    r = subprocess.run([sys.executable, os.path.join(ROOT, "tests", "_debug_child.py")], env=debug_env,
                       cwd=ROOT, capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-4000:]
    return json.loads(r.stdout.strip().splitlines()[-1])


def _expected_moves(q, k, v, causal, d):
    """(oracle total of moves, allowed difference)."""
    _, _, moves, margin = A.attention_lazy_rescale(q, k, v, causal, d ** -0.5, Bc=128, tau=8.0, rescale_rows=True)
    Nq, Nkv = q.shape[2], k.shape[2]
    vis = A.visible_mask(Nq, Nkv, causal)
    blocks = np.array([len({j // 128 for j in np.flatnonzero(vis[i])}) for i in range(Nq)])
    near = margin < BAND
    slack = int((near * np.maximum(blocks - 1, 0)[None, None]).sum())
    return int(moves.sum()), slack, int(near.sum())


def _all_masked_tiles(B, H, Nq, Nkv):
    vis = A.visible_mask(Nq, Nkv, True)
    n = 0
    for r0 in range(0, Nq, 128):
        for c0 in range(0, Nkv, 128):
            n += not vis[r0:r0 + 128, c0:c0 + 128].any()
    return B * H * n


@pytest.mark.parametrize("case", C.LAZY, ids=lambda c: f"{c[0]}-causal{int(c[1])}-d{c[2]}-N{c[3]}")
def test_rescale_count_matches_oracle(child, case):
    pattern, causal, d, N = case
    got = child["lazy"][f"{pattern}-{int(causal)}-{d}-{N}"]
    assert got["status"] == 0 and got["counters"][2] == 0
    q, k, v = C.lazy_inputs(pattern, d, N)
    total, slack, near = _expected_moves(q, k, v, causal, d)
    print(f"{pattern} causal={causal} d={d} N={N}: device {got['counters'][0]}, oracle {total} "
          f"({near} rows within {BAND} of the threshold, slack {slack})")
    assert total > 0
    assert abs(got["counters"][0] - total) <= slack
    if not causal:
        assert got["counters"][1] == 0


@pytest.mark.parametrize("shape", C.CAUSAL, ids=lambda s: "B{}-H{}-Nq{}-Nkv{}-d{}".format(*s))
def test_causal_skipped_tiles_and_rescales(child, shape):
    B, H, Nq, Nkv, d = shape
    got = child["causal"]["{}-{}-{}-{}-{}".format(*shape)]
    assert got["status"] == 0 and got["counters"][2] == 0
    assert got["counters"][1] == _all_masked_tiles(B, H, Nq, Nkv)
    q, k, v = C.causal_inputs(*shape)
    total, slack, _ = _expected_moves(q, k, v, True, d)
    assert abs(got["counters"][0] - total) <= slack


def test_every_family_in_bounds(child):
    for name, got in child["families"].items():
        assert got["status"] == 0, (name, got)
        assert got["counters"][2] == 0, (name, got)
    assert len(child["families"]) == 12


def test_gpu_suite_under_debug_build(debug_env):
    r = subprocess.run([sys.executable, "-m", "pytest", "tests", "-m", "gpu", "-x", "-q", "-p", "no:cacheprovider",
                        "--ignore", os.path.join("tests", "test_debug_build_gpu.py")],
                       env=debug_env, cwd=ROOT, capture_output=True, text=True, timeout=1800)
    tail = r.stdout[-3000:] + r.stderr[-2000:]
    print(tail)
    assert r.returncode == 0, tail
