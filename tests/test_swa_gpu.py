"""Sliding-window GQA attention with RoPE (samba_swa_fwd) against the fp64 oracle,
plus the band-edge properties that pin the window bookkeeping exactly."""
import math

import numpy as np
import pytest

from oracle import samba_oracle as O
from sliding_window_attention_samba_b200 import inputs as I
from tests.helpers import TOL, attn_err, dev, host, rel_err

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def L():
    import torch
    from sliding_window_attention_samba_b200 import _lib
    torch.cuda.init()
    return _lib


def run_swa(L_, q, k, v, window, rope_base, pos0, dt, scale=0.0):
    import torch
    Bn, Ln, Hq, d = q.shape
    Hkv = k.shape[2]
    o = torch.empty(Bn, Ln, Hq, d, device="cuda", dtype=torch.bfloat16 if dt == "bf16" else torch.float32)
    ws_n = L_.samba_swa_workspace_size(Bn, Ln, Hq, Hkv, d, rope_base, 1 if dt == "bf16" else 0)
    ws = torch.empty(max(ws_n, 1), dtype=torch.uint8, device="cuda")
    L_.samba_swa_fwd(dev(q, dt), dev(k, dt), dev(v, dt), o, Bn, Ln, Hq, Hkv, d, window, rope_base, pos0, scale,
                     1 if dt == "bf16" else 0, ws, ws_n)
    torch.cuda.synchronize()
    assert L_.samba_get_error() == 0
    return host(o)


def oracle_swa(q, k, v, window, rope_base, pos0, rows=None):
    Ln = q.shape[1]
    pos = np.arange(pos0, pos0 + Ln)
    qr, kr = O.rope(q, pos, rope_base), O.rope(k, pos, rope_base)
    return O.swa(qr, kr, v, window)


@pytest.mark.parametrize("dt,Bn,Ln,Hq,Hkv,d,w,base", [
    ("f32", 1, 256, 4, 2, 16, 64, 10000.0),
    ("f32", 2, 300, 4, 4, 32, 37, 10000.0),
    ("f32", 1, 129, 2, 1, 64, 1000, 0.0),
    ("bf16", 1, 1024, 32, 4, 64, 256, 10000.0),
    ("bf16", 2, 333, 8, 2, 64, 100, 10000.0),
    ("bf16", 1, 5, 4, 1, 64, 2048, 10000.0),
])
def test_swa_matches_oracle(L, dt, Bn, Ln, Hq, Hkv, d, w, base):
    r = I.swa_inputs(3, Bn, Ln, Hq, Hkv, d, dt)
    o = run_swa(L, r["q"], r["k"], r["v"], w, base, 0, dt)
    ref = oracle_swa(r["q"], r["k"], r["v"], w, base, 0)
    # bf16 with RoPE: the rotated q/k are stored in bf16 before the tensor-core
    # products, which only the l-inf / normwise reading separates from kernel error
    err = attn_err if (dt == "bf16" and base != 0.0) else rel_err
    assert err(o, ref) <= TOL[dt]


def test_swa_config_shapes_peaked(L):
    # q scaled x3 so that softmax is peaked (score std 3): window-edge mistakes cannot hide
    # under a flat softmax; the band edge itself is pinned exactly by the tests below
    r = I.swa_inputs(3, 1, 2600, 32, 4, 64, "bf16")
    q = I.round_to(r["q"] * 3.0, "bf16")
    o = run_swa(L, q, r["k"], r["v"], 2048, 10000.0, 0, "bf16")
    rows = [0, 1, 2047, 2048, 2049, 2599]
    ref = oracle_swa(q, r["k"], r["v"], 2048, 10000.0, 0)
    assert attn_err(o[:, rows], ref[:, rows]) <= TOL["bf16"]
    assert attn_err(o, ref) <= TOL["bf16"]


@pytest.mark.parametrize("kernel", ["", "2", "1"])
def test_swa_config_shapes_peaked_x30(L, kernel):
    """q scaled x30 (score std 30: most rows put nearly all weight on one or two
    keys), at the config shapes (32/4 heads of 64, window 2048) past the window,
    through the four-head, two-head and one-head tensor-core kernels.  Without RoPE:
    both sides then score the same bf16 q and k, while with RoPE the bf16 storage
    of the rotated q/k moves logits of std 30 by ~0.1, which flips near-ties
    between the two largest keys and is not a kernel error."""
    import os
    r = I.swa_inputs(13, 1, 2600, 32, 4, 64, "bf16")
    q = I.round_to(r["q"] * 30.0, "bf16")
    old = os.environ.get("SAMBA_SWA_KERNEL")
    if kernel:
        os.environ["SAMBA_SWA_KERNEL"] = kernel
    try:
        o = run_swa(L, q, r["k"], r["v"], 2048, 0.0, 0, "bf16")
    finally:
        if kernel:
            if old is None:
                del os.environ["SAMBA_SWA_KERNEL"]
            else:
                os.environ["SAMBA_SWA_KERNEL"] = old
    ref = oracle_swa(q, r["k"], r["v"], 2048, 0.0, 0)
    rows = [0, 1, 2, 2047, 2048, 2049, 2599]
    assert rel_err(o[:, rows], ref[:, rows]) <= TOL["bf16"]
    assert rel_err(o, ref) <= TOL["bf16"]


@pytest.mark.parametrize("dt", ["f32", "bf16"])
def test_swa_window_one_returns_v_exactly(L, dt):
    r = I.swa_inputs(4, 1, 200, 8, 2, 64, dt)
    o = run_swa(L, r["q"], r["k"], r["v"], 1, 10000.0, 0, dt)
    for h in range(8):
        assert np.array_equal(o[:, :, h], r["v"][:, :, h // 4].astype(np.float64))


@pytest.mark.parametrize("dt,w,Ln", [("f32", 64, 300), ("f32", 5, 300), ("bf16", 20, 64), ("bf16", 5, 64)])
def test_swa_uniform_weights_band_mean(L, dt, w, Ln):
    # bf16: v_s = s < 64 and the half-integer band means are exact in bf16, so an
    # off-by-one in the band (a 0.5 shift) cannot round away
    q = np.zeros((1, Ln, 2, 16), np.float32)
    k = I.draw_normal(5, "k", (1, Ln, 1, 16), 1.0, dt)
    v = np.tile(np.arange(Ln, dtype=np.float32)[None, :, None, None], (1, 1, 1, 16))
    o = run_swa(L, q, k, v, w, 10000.0, 0, dt)
    expect = np.array([(max(0, t - w + 1) + t) / 2 for t in range(Ln)])
    # an off-by-one in the band shifts the mean by 0.5, far above bf16 rounding of values < 300
    tol = 1e-3 if dt == "f32" else 0.2
    assert np.max(np.abs(o[0, :, 0, 0] - expect)) < tol
    assert np.max(np.abs(o[0, :, 1, 0] - expect)) < tol


def test_swa_perturbation_locality_exact(L):
    Ln, w, s = 500, 64, 211
    r = I.swa_inputs(6, 1, Ln, 4, 2, 64, "bf16")
    o1 = run_swa(L, r["q"], r["k"], r["v"], w, 10000.0, 0, "bf16")
    k2, v2 = r["k"].copy(), r["v"].copy()
    k2[0, s] = I.round_to(k2[0, s] + 1.0, "bf16")
    v2[0, s] = I.round_to(v2[0, s] - 2.0, "bf16")
    o2 = run_swa(L, r["q"], k2, v2, w, 10000.0, 0, "bf16")
    changed = np.nonzero(np.any(o1 != o2, axis=(0, 2, 3)))[0]
    assert changed.min() == s and changed.max() == s + w - 1


def test_swa_rope_shift_invariance_large_positions(L):
    r = I.swa_inputs(7, 1, 300, 4, 2, 64, "f32")
    o0 = run_swa(L, r["q"], r["k"], r["v"], 128, 10000.0, 0, "f32")
    for P in (1000, 1 << 20, (1 << 30) - 400):
        oP = run_swa(L, r["q"], r["k"], r["v"], 128, 10000.0, P, "f32")
        assert rel_err(oP, o0) <= 1e-4


def test_swa_gqa_equals_repeated_kv(L):
    r = I.swa_inputs(8, 1, 257, 8, 2, 32, "f32")
    o = run_swa(L, r["q"], r["k"], r["v"], 50, 10000.0, 0, "f32")
    o_mha = run_swa(L, r["q"], np.repeat(r["k"], 4, 2), np.repeat(r["v"], 4, 2), 50, 10000.0, 0, "f32")
    assert rel_err(o, o_mha) <= 1e-6


@pytest.mark.parametrize("Bn,Ln,w", [(1, 1000, 2048), (2, 777, 128), (1, 2500, 300), (1, 130, 1)])
def test_swa_tensor_core_kernel_matches_cuda_core_kernel(L, Bn, Ln, w):
    """The tcgen05 kernel (default for bf16, head_dim 64) against the CUDA-core
    kernel on the same bf16 inputs: both accumulate in fp32; they differ by the
    bf16 rounding of P on the tensor-core path."""
    import os
    r = I.swa_inputs(9, Bn, Ln, 8, 2, 64, "bf16")
    o_tc = run_swa(L, r["q"], r["k"], r["v"], w, 10000.0, 0, "bf16")
    os.environ["SAMBA_SWA_KERNEL"] = "simt"
    try:
        o_simt = run_swa(L, r["q"], r["k"], r["v"], w, 10000.0, 0, "bf16")
    finally:
        del os.environ["SAMBA_SWA_KERNEL"]
    assert attn_err(o_tc, o_simt) <= 1e-2


@pytest.mark.parametrize("Bn,Ln,w,qh", [(1, 1000, 2048, 32), (2, 777, 128, 8), (1, 2500, 300, 16), (1, 130, 1, 8)])
def test_swa_four_head_kernel_matches_two_head_kernel(L, Bn, Ln, w, qh):
    """The four-heads-per-CTA kernel (64-key tiles, default when a kv group has a
    multiple of four query heads) against the two-heads-per-CTA kernel (128-key
    tiles) on the same bf16 inputs: same arithmetic per score, different tile
    boundaries for the online softmax."""
    import os
    r = I.swa_inputs(14, Bn, Ln, qh, qh // 8 if qh >= 8 else 1, 64, "bf16")
    o4 = run_swa(L, r["q"], r["k"], r["v"], w, 10000.0, 0, "bf16")
    os.environ["SAMBA_SWA_KERNEL"] = "2"
    try:
        o2 = run_swa(L, r["q"], r["k"], r["v"], w, 10000.0, 0, "bf16")
    finally:
        del os.environ["SAMBA_SWA_KERNEL"]
    assert attn_err(o4, o2) <= 1e-2
    ref = oracle_swa(r["q"], r["k"], r["v"], w, 10000.0, 0)
    assert attn_err(o4, ref) <= TOL["bf16"]
