"""ctypes binding of libtiledattn_probe (include/tiledattn_probe.h) and the
rate measurements built on it: the tensor-core ceiling per MMA kind and the
MUFU exponential rate, each from one CTA per SM, in SM clock cycles (from the
kernels' own %clock64) and per second (CUDA events around the launch)."""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
PROBE_PATH = os.path.join(_PKG, "libtiledattn_probe.so")

KINDS = {"bf16": 0, "int8": 1, "fp8": 2, "fp4": 3}
A_TMEM, TWO_ACC, TWO_ISSUERS, COMMIT, B_MN, ATTN, TESTWAIT, WAITFENCE, TMEM_TRAFFIC = 1, 2, 4, 8, 16, 32, 64, 128, 256
FLAGPOLL, FLAGFENCE = 512, 1024
K_PER_MMA = {"bf16": 16, "int8": 32, "fp8": 32, "fp4": 64}

_lib = None


def load():
    global _lib
    if _lib is None:
        if not os.path.exists(PROBE_PATH):
            raise RuntimeError(f"{PROBE_PATH} is missing; build it with `python -m tiled_attention_24_b200.build`")
        lib = ctypes.CDLL(PROBE_PATH)
        VP, I = ctypes.c_void_p, ctypes.c_int
        lib.tap_mma_rate.argtypes = [I, I, I, I, I, VP, VP]
        lib.tap_ex2_rate.argtypes = [I, I, I, I, VP, VP, VP]
        lib.tap_mma_tight_rate.argtypes = [I, I, I, I, I, VP, VP]
        lib.tap_mma_tight_rate.restype = I
        lib.tap_softmax_rate.argtypes = [I, I, I, VP, VP, VP]
        for f in (lib.tap_mma_rate, lib.tap_ex2_rate, lib.tap_softmax_rate):
            f.restype = I
        _lib = lib
    return _lib


def _timed(launch, grid, device, repeats):
    """Best of ``repeats`` launches: (event ms, mean cycles over CTAs)."""
    cyc = torch.zeros(grid, dtype=torch.int64, device=device)
    st = torch.cuda.current_stream(device)
    best = None
    for _ in range(repeats):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(st)
        rc = launch(ctypes.c_void_p(cyc.data_ptr()), ctypes.c_void_p(st.cuda_stream))
        b.record(st)
        if rc != 0:
            raise RuntimeError(f"probe launch failed ({rc})")
        torch.cuda.synchronize(device)
        c = cyc.cpu()
        if (c < 0).any():
            raise RuntimeError("probe kernel wait timed out")
        ms = a.elapsed_time(b)
        if best is None or ms < best[0]:
            best = (ms, float(c.double().mean()))
    return best


def mma_rate(kind: str, n: int = 128, iters: int = 8192, device=None, repeats: int = 3, flags: int = 0):
    """Dense MMA throughput of one kind: FLOP (or OP) per clock per SM from the
    cycle counts, and TFLOP/s over the whole GPU from the event time."""
    device = device or torch.device("cuda", torch.cuda.current_device())
    sms = torch.cuda.get_device_properties(device).multi_processor_count
    lib = load()
    ms, cycles = _timed(lambda c, s: lib.tap_mma_rate(KINDS[kind], n, iters, sms, flags, c, s), sms, device, repeats)
    flop_per_cta = 2.0 * iters * 4 * 128 * n * K_PER_MMA[kind] * (2 if flags & TWO_ISSUERS else 1)
    return {"kind": kind, "n": n, "flags": flags, "flop_per_clk_sm": flop_per_cta / cycles,
            "tflops": flop_per_cta * sms / (ms * 1e-3) / 1e12, "sm_ghz": cycles / (ms * 1e6), "ms": ms}


def mma_tight_rate(kind: str, n: int = 128, iters: int = 4096, device=None, repeats: int = 3, flags: int = 0):
    """As ``mma_rate`` with the straight-line, compile-time issue loop."""
    device = device or torch.device("cuda", torch.cuda.current_device())
    sms = torch.cuda.get_device_properties(device).multi_processor_count
    lib = load()
    ms, cycles = _timed(lambda c, s: lib.tap_mma_tight_rate(KINDS[kind], n, iters, sms, flags, c, s), sms, device,
                        repeats)
    flop_per_cta = 2.0 * iters * 8 * 128 * n * K_PER_MMA[kind] * (2 if flags & ATTN else 1) * \
        (2 if flags & TWO_ISSUERS else 1)
    return {"kind": kind, "n": n, "flags": flags, "tight": True, "flop_per_clk_sm": flop_per_cta / cycles,
            "tflops": flop_per_cta * sms / (ms * 1e-3) / 1e12, "sm_ghz": cycles / (ms * 1e6), "ms": ms}


def ex2_rate(threads: int = 1024, ilp: int = 8, iters: int = 4096, device=None, repeats: int = 3):
    """MUFU ex2 results per clock per SM with ``threads`` per SM."""
    device = device or torch.device("cuda", torch.cuda.current_device())
    sms = torch.cuda.get_device_properties(device).multi_processor_count
    sink = torch.empty(sms * threads, dtype=torch.float32, device=device)
    lib = load()
    ms, cycles = _timed(lambda c, s: lib.tap_ex2_rate(threads, ilp, iters, sms, c,
                                                      ctypes.c_void_p(sink.data_ptr()), s), sms, device, repeats)
    return {"threads": threads, "ilp": ilp, "ex2_per_clk_sm": threads * ilp * iters / cycles}


def softmax_rate(threads: int = 256, iters: int = 2048, device=None, repeats: int = 3):
    """Score pairs per clock per SM through the bf16 softmax's per-score work."""
    device = device or torch.device("cuda", torch.cuda.current_device())
    sms = torch.cuda.get_device_properties(device).multi_processor_count
    sink = torch.empty(sms * threads, dtype=torch.float32, device=device)
    lib = load()
    ms, cycles = _timed(lambda c, s: lib.tap_softmax_rate(threads, iters, sms, c,
                                                          ctypes.c_void_p(sink.data_ptr()), s), sms, device, repeats)
    return {"threads": threads, "scores_per_clk_sm": 2.0 * threads * 8 * iters / cycles}
