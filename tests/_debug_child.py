"""Runs in a child process with TILEDATTN_LIB pointing at libtiledattn_debug.so
(tests/test_debug_build_gpu.py): launches the bf16 forward on the cases below
and one small call of every other kernel family, reads the debug counters
after each (attn_debug_counters, reset) and the status word
(attn_check_status), and prints one JSON object on its last line.

The inputs come from the functions here, so the parent builds the same ones
for the oracle."""
import json
import os
import sys

import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from workloads import make_qkv, make_varlen  # noqa: E402

# lazy rescale: key blocks scaled by `gains` (block j by gains[min(j, -1)])
# (N = 768 at d = 128: whole query tile pairs; 700: a ragged last pair)
LAZY = [(pattern, causal, d, N) for pattern in ("steps", "mixed") for causal in (False, True) for d in (64, 128)
        for N in ((700, 768) if d == 128 else (700,))]
GAINS = {"steps": [1, 4, 8, 16, 32], "mixed": [1, 3]}
# causal skipping: (B, H, Nq, Nkv, d)
CAUSAL = [(1, 3, 1000, 1000, 128), (2, 2, 300, 1000, 64), (1, 2, 1000, 300, 128), (1, 1, 129, 4000, 64),
          (1, 3, 1024, 1024, 128), (1, 2, 512, 1000, 128)]


def lazy_inputs(pattern, d, N=700):
    q, k, v = make_qkv("prefill", seed=17 + d, B=1, H=2, Nq=N, Nkv=N, d=d)
    k = k.float()
    g = GAINS[pattern]
    for j in range(-(-N // 128)):
        k[:, :, j * 128:(j + 1) * 128] *= g[min(j, len(g) - 1)]
    return q, k.to(torch.bfloat16), v


def causal_inputs(B, H, Nq, Nkv, d):
    return make_qkv("prefill", seed=Nq + Nkv + d, B=B, H=H, Nq=Nq, Nkv=Nkv, d=d)


def _families(ta, dev):
    """One small call per kernel family (the counters must show no bounds
    violation for any of them)."""
    q, k, v = (t.to(dev) for t in make_qkv("prefill", seed=5, B=1, H=2, Nq=300, Nkv=300, d=128))
    yield "int8", lambda: ta.forward_int8(q, k, v, True)
    yield "int4", lambda: ta.forward_int4(q, k, v, False)
    yield "fp8", lambda: ta.forward_fp8(q, k, v, True)
    yield "fp4_direct_p", lambda: ta.forward_fp4(q, k, v, True, p_mode=ta.DIRECT_P)
    yield "fp4_qae", lambda: ta.forward_fp4(q, k, v, False, p_mode=ta.QUANT_AFTER_EXP)
    o, lse = ta.forward(q, k, v, True)
    do = torch.randn_like(q)
    yield "bwd", lambda: ta.backward(q, k, v, o, lse, do, True)
    yield "bwd_fp8p", lambda: ta.backward(q, k, v, o, lse, do, True, p_fp8=True)
    qg, kg, vg = (t.to(dev) for t in make_qkv("prefill", seed=6, B=1, H=8, Nq=200, Nkv=333, d=64))
    yield "gqa_fwd", lambda: ta.forward(qg, kg[:, :2].contiguous(), vg[:, :2].contiguous(), True)
    qd = qg[:, :, :1].contiguous()
    yield "decode", lambda: ta.decode(qd, kg, vg, num_splits=4)
    yield "decode_gqa", lambda: ta.decode(qd, kg[:, :2].contiguous(), vg[:, :2].contiguous(), num_splits=4)
    qv, kv, vv, cq, ck = make_varlen([5, 300, 129], [7, 300, 400], 4, 2, 128, seed=7)
    qv, kv, vv, cq, ck = (t.to(dev) for t in (qv, kv, vv, cq, ck))
    yield "varlen", lambda: ta.forward_varlen(qv, kv, vv, cq, ck, 300, True)
    qdv = make_qkv("prefill", seed=8, B=3, H=4, Nq=1, Nkv=400, d=128)
    ks = torch.tensor([1, 400, 257], dtype=torch.int32, device=dev)
    qdv = [t.to(dev) for t in qdv]
    yield "decode_varlen", lambda: ta.decode_varlen(qdv[0], qdv[1], qdv[2], ks, num_splits=3)


def main():
    import tiled_attention_24_b200 as ta
    assert ta.LIB_PATH.endswith("libtiledattn_debug.so"), ta.LIB_PATH
    dev = torch.device("cuda", 0)
    ta.attn_debug_counters(reset=True)
    out = {"lazy": {}, "causal": {}, "families": {}}

    def record(group, name, fn):
        fn()
        torch.cuda.synchronize()
        status = ta.attn_check_status()
        out[group][name] = {"counters": ta.attn_debug_counters(reset=True), "status": status}

    for pattern, causal, d, N in LAZY:
        q, k, v = (t.to(dev) for t in lazy_inputs(pattern, d, N))
        record("lazy", f"{pattern}-{int(causal)}-{d}-{N}", lambda: ta.forward(q, k, v, causal, d ** -0.5))
    for B, H, Nq, Nkv, d in CAUSAL:
        q, k, v = (t.to(dev) for t in causal_inputs(B, H, Nq, Nkv, d))
        record("causal", f"{B}-{H}-{Nq}-{Nkv}-{d}", lambda: ta.forward(q, k, v, True, d ** -0.5))
    for name, fn in _families(ta, dev):
        record("families", name, fn)
    print(json.dumps(out))


if __name__ == "__main__":
    main()
