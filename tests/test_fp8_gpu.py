"""GPU parity of the FP8 (e4m3) path with incoherent processing against the
oracle, through the C ABI.

* quantisers (rotation by the fast Walsh-Hadamard transform, per-row and
  per-channel e4m3): bit-exact codes and fp32 scales;
* forward: within 5e-3 max-abs of the oracle's step-by-step FP8 emulation
  (lazy rescale threshold 8, as the kernel).  A P element within fp32
  evaluation error of an e4m3 rounding midpoint, or a rescale decision that
  close to the threshold, may go either way on the device; the oracle gives
  the interval of outputs over every such choice (``oracle.outcomes``) and
  the device must lie within 5e-3 of it.  Flagged rows and elements are
  reported and bounded.

Every output sits between guard bands that must survive the call
(``tests._guard``).
"""
import numpy as np
import pytest
import torch

from oracle import attention as A
from oracle import fp8 as F
from tests import _guard as G
from tests._parity import assert_within_outcomes, visible_scores
from workloads import WORKLOADS, make_qkv, rotation_signs

pytestmark = pytest.mark.gpu


def _np(t):
    return t.detach().cpu().numpy()


def _values(codes):
    """e4m3 bytes -> values (sign bit 0x80, magnitude from the format table)."""
    c = _np(codes).astype(np.int64)
    mag = c & 0x7F
    assert (mag != 0x7F).all(), "NaN code"
    return np.where(c & 0x80, -1.0, 1.0) * F.UE4M3_VALUES[mag]


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("rotate", [False, True])
@pytest.mark.parametrize("name", ["prefill", "lowp"])
def test_fp8_row_quantiser_bit_exact(cuda_lib, name, rotate, d):
    q, _, v = make_qkv(name, seed=5, B=2, H=3, Nq=257, Nkv=130, d=d)
    q[0, 1, 7] = 0                                    # an all-zero row
    signs = rotation_signs(d, 3) if rotate else None
    codes, sc = G.quantize_fp8(cuda_lib, q.cuda(), 0, None if signs is None else signs.cuda())
    assert cuda_lib.attn_check_status() == 0
    rv, rs = F.quantize_fp8_rows(q, None if signs is None else signs.numpy())
    assert np.array_equal(_np(sc), rs)
    assert np.array_equal(_values(codes), rv)


@pytest.mark.parametrize("d", [64, 128])
def test_fp8_channel_quantiser_bit_exact(cuda_lib, d):
    _, _, v = make_qkv("lowp", seed=6, B=2, H=3, Nq=1, Nkv=333, d=d)
    v[1, 2, :, 5] = 0                                 # an all-zero channel
    codes, sc = G.quantize_fp8(cuda_lib, v.cuda(), 1)
    assert cuda_lib.attn_check_status() == 0
    rv, rs = F.quantize_fp8_channels(v)
    assert np.array_equal(_np(sc), rs)
    assert np.array_equal(_values(codes), rv)


def _check_fp8(ta, q, k, v, causal, scale, rotate, rows=None, what="", seed=0):
    """The device quantises and runs the forward; the oracle quantises the same
    bf16 inputs with the same signs itself and emulates the forward."""
    d = q.shape[-1]
    signs = rotation_signs(d, seed) if rotate else None
    sg = None if signs is None else signs.cuda()
    qc, qs = G.quantize_fp8(ta, q.cuda(), 0, sg)
    kc, ks = G.quantize_fp8(ta, k.cuda(), 0, sg)
    vc, vs = G.quantize_fp8(ta, v.cuda(), 1)
    B, H, Nq, _ = q.shape
    o, lse = G.fwd_fp8(ta, qc, qs, kc, ks, vc, vs, causal, scale, rotate, what)
    assert ta.attn_check_status() == 0
    sn = None if signs is None else signs.numpy()
    rqv, rqs = F.quantize_fp8_rows(q, sn)
    rkv, rks = F.quantize_fp8_rows(k, sn)
    rvv, rvs = F.quantize_fp8_channels(v)
    O, L, R = F.attention_fp8(rqv, rqs, rkv, rks, rvv, rvs, causal, scale,
                              rot_d=d if rotate else 1, outcomes=True, rows=rows, tau=8.0)
    og, lg = _np(o).astype(np.float64), _np(lse).astype(np.float64)
    if rows is not None:
        og, lg = og[:, :, rows], lg[:, :, rows]
    n_scores = B * H * visible_scores(Nq, k.shape[2], causal, rows)
    err, _ = assert_within_outcomes(og, lg, O, L, R, what, n_scores)
    Oe, _ = A.attention(q, k, v, causal, scale, rows=rows)
    cos = float((og * Oe).sum() / (np.linalg.norm(og) * np.linalg.norm(Oe) + 1e-300))
    return err, R.flips, cos


@pytest.mark.parametrize("rotate", [False, True])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("shape", [(1, 2, 128, 128), (1, 1, 300, 333), (2, 2, 129, 1000), (1, 1, 1, 1),
                                   (1, 1, 640, 200), (1, 1, 513, 129)], ids=lambda s: "x".join(map(str, s)))
def test_fp8_forward_small(cuda_lib, shape, causal, rotate):
    B, H, Nq, Nkv = shape
    q, k, v = make_qkv("prefill", seed=21, B=B, H=H, Nq=Nq, Nkv=Nkv, d=128)
    _check_fp8(cuda_lib, q, k, v, causal, 128 ** -0.5, rotate, what=f"{shape} causal={causal} rot={rotate}")


def test_fp8_rotation_on_outlier_inputs(cuda_lib):
    """Both settings match their emulation; the rotation brings the output
    closer to exact attention on inputs with outlier channels."""
    q, k, v = make_qkv("lowp", seed=1, B=1, H=4, Nq=1024, Nkv=1024)
    _, _, cos_plain = _check_fp8(cuda_lib, q, k, v, False, 128 ** -0.5, False, what="lowp plain")
    _, _, cos_rot = _check_fp8(cuda_lib, q, k, v, False, 128 ** -0.5, True, what="lowp rotated")
    print(f"lowp 1024: cosine vs fp64 plain {cos_plain:.5f}, rotated {cos_rot:.5f}")
    assert cos_rot > 0.99 and cos_rot >= cos_plain


def test_fp8_full_lowp_workload_sampled_rows(cuda_lib):
    w = WORKLOADS["lowp"]
    q, k, v = make_qkv(w, seed=0)
    rows = np.array(sorted({0, 1, 127, 128, 255, 256, 8191} | set(np.random.default_rng(4).choice(8192, 16).tolist())))
    _, flips, cos = _check_fp8(cuda_lib, q, k, v, False, w.scale, True, rows=rows, what="fp8 lowp full")
    print(f"fp8 lowp full: cosine vs fp64 {cos:.5f}, boundary elements {flips}")
    assert cos > 0.99


def test_fp8_package_forward(cuda_lib):
    q, k, v = make_qkv("prefill", seed=23, B=1, H=2, Nq=256, Nkv=384, d=128)
    o, lse = cuda_lib.forward_fp8(q.cuda(), k.cuda(), v.cuda(), causal=True)
    assert cuda_lib.attn_check_status() == 0
    Oe, Le = A.attention(q, k, v, True, 128 ** -0.5)
    assert np.abs(_np(o) - Oe).max() < 0.1
    assert np.isfinite(_np(lse)).all()


def test_fp8_quantisers_exact_on_rounding_ties(cuda_lib):
    """Rows and channels whose quotients land exactly on e4m3 rounding
    midpoints (amax = 448 * 2^k, so s = 2^k, and x = midpoint * 2^k), the case
    where a divide-free quotient could round the other way: codes and scales
    bit-exact against the oracle."""
    from oracle.lowp import UE4M3_VALUES
    grid = np.asarray(UE4M3_VALUES, dtype=np.float64)
    mids = (grid[1:] + grid[:-1]) / 2
    mids = mids[(mids > 2.0 ** -6) & (mids < 448)]
    rows = []
    for k in (-4, 0, 3):
        for sign in (1.0, -1.0):
            r = np.zeros(128)
            r[0] = 448.0 * 2.0 ** k
            sel = mids[np.linspace(0, mids.size - 1, 127).astype(int)]
            r[1:] = sign * sel * 2.0 ** k
            rows.append(r)
    x64 = np.stack(rows)
    x = torch.tensor(x64, dtype=torch.float32).reshape(1, 2, -1, 128).to(torch.bfloat16)
    assert (x.float().numpy().reshape(-1, 128) == x64).all()    # midpoints are exact in bf16
    codes, sc = G.quantize_fp8(cuda_lib, x.cuda(), 0)
    assert cuda_lib.attn_check_status() == 0
    rv, rs = F.quantize_fp8_rows(x, None)
    assert np.array_equal(_np(sc), rs)
    assert np.array_equal(_values(codes), rv)
    # channels: token n of channel c holds pattern[n] * 2^k(c), pattern[0] = 448
    pat = np.concatenate([[448.0], mids[np.linspace(0, mids.size - 1, 127).astype(int)]])
    kc = np.array([(-4, 0, 3)[c % 3] for c in range(128)])
    sgn = np.where(np.arange(128) % 2, -1.0, 1.0)
    v64 = pat[:, None] * (2.0 ** kc)[None, :] * sgn[None, :]
    v = torch.tensor(np.stack([v64, -v64]), dtype=torch.float32).reshape(1, 2, 128, 128).to(torch.bfloat16)
    assert (v.float().numpy().reshape(2, 128, 128) == np.stack([v64, -v64])).all()
    codes, sc = G.quantize_fp8(cuda_lib, v.cuda(), 1)
    assert cuda_lib.attn_check_status() == 0
    rv, rs = F.quantize_fp8_channels(v)
    assert np.array_equal(_np(sc), rs)
    assert np.array_equal(_values(codes), rv)
