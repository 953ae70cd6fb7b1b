"""RMSNorm, short convolution and the dense projections (every epilogue, both
GEMM kernels) against the fp64 oracle."""
import os

import numpy as np
import pytest

from oracle import samba_oracle as O
from sliding_window_attention_samba_b200 import inputs as I
from tests.helpers import TOL, dev, host, rel_err, sum_slack

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def L():
    import torch
    from sliding_window_attention_samba_b200 import _lib
    torch.cuda.init()
    return _lib


def DT(dt):
    return 1 if dt == "bf16" else 0


@pytest.mark.parametrize("dt,rows,dim", [("f32", 37, 64), ("bf16", 1000, 2048), ("bf16", 3, 8)])
def test_rmsnorm(L, dt, rows, dim):
    import torch
    x = I.draw_normal(1, "x", (rows, dim), 3.0, dt)
    g = I.draw_normal(1, "g", (dim,), 1.0, "f32")
    out = torch.empty(rows, dim, device="cuda", dtype=dev(x, dt).dtype)
    L.samba_rmsnorm(dev(x, dt), dev(g), out, rows, dim, 1e-5, DT(dt))
    assert rel_err(host(out), O.rmsnorm(x, g, 1e-5)) <= TOL[dt]


@pytest.mark.parametrize("dt,Bn,Ln,D,k,bias", [("f32", 1, 256, 128, 4, False), ("f32", 2, 70, 64, 4, True),
                                                ("bf16", 2, 4096, 4096, 4, False), ("bf16", 1, 2, 64, 4, True),
                                                ("bf16", 1, 33, 32, 3, False)])
def test_causal_conv(L, dt, Bn, Ln, D, k, bias):
    import torch
    x2 = I.draw_normal(2, "x", (Bn, Ln, 2 * D), 1.0, dt)  # strided x half, as in the block
    w = I.draw_normal(2, "w", (D, k), 0.5, "f32")
    b = I.draw_normal(2, "b", (D,), 0.5, "f32") if bias else None
    u = torch.empty(Bn, Ln, D, device="cuda", dtype=dev(x2, dt).dtype)
    st = torch.empty(Bn, D, k - 1, device="cuda", dtype=u.dtype)
    L.samba_causal_conv1d(dev(x2, dt), 2 * D, dev(w), dev(b), u, st, Bn, Ln, D, k, DT(dt))
    pre, so = O.causal_dwconv(x2[..., :D], w, b)
    assert rel_err(host(u), O.silu(pre)) <= TOL[dt]
    assert np.array_equal(host(st), so)  # state is a bit copy of the inputs


def _linear(L, dt, M, N, K, epi, force_simt=False):
    import torch
    x = I.draw_normal(3, "x", (M, K), 1.0, dt)
    W = I.draw_normal(3, "W", (N, K), 0.05, dt)
    W2 = I.draw_normal(3, "W2", (N, K), 0.05, dt)
    bias = I.draw_normal(3, "b", (N,), 1.0, "f32")
    resid = I.draw_normal(3, "r", (M, N), 1.0, dt)
    out = torch.empty(M, N, device="cuda", dtype=torch.bfloat16 if dt == "bf16" else torch.float32)
    old = os.environ.get("SAMBA_GEMM_KERNEL")
    if force_simt:
        os.environ["SAMBA_GEMM_KERNEL"] = "simt"
    try:
        L.samba_linear(dev(x, dt), dev(W, dt), dev(W2, dt), dev(bias), dev(resid, dt), out, M, N, K, epi, DT(dt))
        torch.cuda.synchronize()
    finally:
        if force_simt:
            if old is None:
                del os.environ["SAMBA_GEMM_KERNEL"]
            else:
                os.environ["SAMBA_GEMM_KERNEL"] = old
    assert L.samba_get_error() == 0
    h = O.linear(x, W)
    ref = {0: h, 1: resid + h, 2: h * O.silu(O.linear(x, W2)), 3: O.softplus(h + bias)}[epi]
    # the residual epilogue is checked on the branch part (the sum is dominated by
    # resid); the single rounding of the stored sum is not error of the branch
    if epi == 1:
        got = host(out)
        return rel_err(got - resid, h, slack=sum_slack(got, dt))
    return rel_err(host(out), ref)


@pytest.mark.parametrize("epi", [0, 1, 2, 3])
@pytest.mark.parametrize("M,N,K", [(300, 256, 2048), (128, 160, 4096), (1000, 512, 128), (77, 2048, 1024),
                                   (200, 176, 256)])
def test_linear_tensor_core_bf16(L, epi, M, N, K):
    assert _linear(L, "bf16", M, N, K, epi) <= TOL["bf16"]


@pytest.mark.parametrize("epi", [0, 2, 3])
def test_linear_simt_bf16(L, epi):
    assert _linear(L, "bf16", 200, 192, 256, epi, force_simt=True) <= TOL["bf16"]


@pytest.mark.parametrize("epi", [0, 1, 2, 3])
def test_linear_f32(L, epi):
    assert _linear(L, "f32", 130, 96, 72, epi) <= TOL["f32"]


def test_linear_tc_equals_simt_closely(L):
    import torch
    M, N, K = 256, 256, 512
    x = dev(I.draw_normal(4, "x", (M, K), 1.0, "bf16"), "bf16")
    W = dev(I.draw_normal(4, "W", (N, K), 0.05, "bf16"), "bf16")
    a = torch.empty(M, N, device="cuda", dtype=torch.bfloat16)
    b = torch.empty_like(a)
    L.samba_linear(x, W, None, None, None, a, M, N, K, 0, 1)
    os.environ["SAMBA_GEMM_KERNEL"] = "simt"
    try:
        L.samba_linear(x, W, None, None, None, b, M, N, K, 0, 1)
    finally:
        del os.environ["SAMBA_GEMM_KERNEL"]
    torch.cuda.synchronize()
    # both accumulate in fp32; outputs differ by at most a couple of bf16 ulps
    assert rel_err(host(a), host(b)) <= 1e-2


_SKINNY_SHAPES = [(1, 2048, 8192), (7, 160, 4096), (32, 8192, 2048), (64, 4096, 128), (32, 2560, 2048)]


@pytest.mark.parametrize("epi,M,N,K", [(e, *s) for e in (0, 1, 2, 3) for s in _SKINNY_SHAPES
                                       if not (e == 2 and s[1] % 128)])  # SwiGLU widths: multiples of 128
def test_linear_skinny_decode_bf16(L, epi, M, N, K):
    """M <= 64 (decode batch): swap-AB tensor-core tiles, split-K over a thread-block
    cluster reduced through distributed shared memory."""
    assert _linear(L, "bf16", M, N, K, epi) <= TOL["bf16"]
