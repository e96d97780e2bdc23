"""attn_decode_noalloc: the split-KV decode for callers that cannot allocate
device memory (code running inside a caller's memory pool or allocator hook,
plug-ins without an allocator, paths that must never enter the driver's
allocator).  It keeps its split partials in a fixed array inside the library
instead of a caller-provided workspace.

Checked through the C ABI on calls in a row with different inputs and shapes
(the later calls must not see anything an earlier one left in the shared
array): each result is bit-identical to attn_decode (the entry point with a
workspace, which runs the same kernels with the same splits) and within the
bf16 tolerances of the fp64 oracle's decode.  One call uses more splits than
there are keys, so some chunks are empty.  Also checks that a request too
large for the fixed array is refused before anything runs.

This file is collected last on purpose (name), so a run that stops at the
first failure has already run every other test.
"""
import ctypes

import pytest
import torch

from oracle import attention as A
from tests._parity import assert_bf16_close
from workloads import make_qkv

pytestmark = pytest.mark.gpu


def _noalloc(lib, q, k, v, scale, splits):
    B, H, _, d = q.shape
    o = torch.empty_like(q)
    lse = torch.empty((B, H, 1), dtype=torch.float32, device=q.device)
    rc = lib.attn_decode_noalloc(ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(k.data_ptr()),
                                 ctypes.c_void_p(v.data_ptr()), ctypes.c_void_p(o.data_ptr()),
                                 ctypes.c_void_p(lse.data_ptr()), B, H, k.shape[2], d, scale, splits,
                                 ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    return rc, o, lse


def test_noalloc_decode_matches_workspace_decode_and_oracle(cuda_lib):
    lib = cuda_lib.load()
    # (B, H, Nkv, d, splits, seed): the largest first, then smaller ones that
    # reuse the front of the array; the third has 16 splits over 5 keys
    cases = [(8, 16, 3000, 128, 16, 31), (3, 5, 777, 64, 7, 32), (2, 3, 5, 128, 16, 33)]
    for B, H, Nkv, d, splits, seed in cases:
        qc, kc, vc = make_qkv("decode", seed=seed, B=B, H=H, Nq=1, Nkv=Nkv, d=d)
        q, k, v = qc.cuda(), kc.cuda(), vc.cuda()
        scale = d ** -0.5
        o_ref, lse_ref = cuda_lib.decode(q, k, v, scale, splits)
        rc, o, lse = _noalloc(lib, q, k, v, scale, splits)
        assert rc == 0, cuda_lib.attn_status_string(rc)
        assert cuda_lib.attn_check_status() == 0
        what = f"noalloc B={B} H={H} Nkv={Nkv} d={d} splits={splits}"
        assert torch.equal(o, o_ref) and torch.equal(lse, lse_ref), what
        O, L = A.decode(qc, kc, vc, scale)
        assert_bf16_close(o, lse, O, L, what)


def test_noalloc_rejects_requests_beyond_its_scratch(cuda_lib):
    lib = cuda_lib.load()
    q = torch.zeros(64, 64, 1, 128, dtype=torch.bfloat16, device="cuda")
    kv = torch.zeros(64, 64, 16, 128, dtype=torch.bfloat16, device="cuda")
    # 64*64 heads x 16 splits x 129 floats = 33.8 MB > 20 MiB
    rc, _, _ = _noalloc(lib, q, kv, kv, 0.1, 16)
    assert rc == -6 and cuda_lib.attn_status_string(rc) == "ATTN_ERR_TOO_LARGE"
