"""The 3.8B model's shapes: head_dim 256 attention with 11 query heads over one
kv head (tcgen05, 64-key tiles, four 64-wide atoms per row), projections whose
widths and reduction lengths are not multiples of the 256 / 64 tiles
(x_proj N = 208, dt_proj K = 176), and a whole block, against the oracle."""
import numpy as np
import pytest

from oracle import samba_oracle as O
from sliding_window_attention_samba_b200 import inputs as I
from tests.helpers import TOL, attn_err, dev, host, rel_err, sum_slack
from tests.test_block_gpu import GpuBlock, check_branches

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def L():
    import torch
    from sliding_window_attention_samba_b200 import _lib
    torch.cuda.init()
    return _lib


@pytest.mark.parametrize("Bn,Ln,window,pos0", [(1, 640, 256, 0), (2, 300, 2048, 5), (1, 2304, 2048, 0),
                                               (1, 129, 64, 1000)])
def test_swa_head_dim_256_gqa11(L, Bn, Ln, window, pos0):
    import torch
    Hq, Hkv, hd = 11, 1, 256
    r = I.swa_inputs(40, Bn, Ln, Hq, Hkv, hd, "bf16")
    q, k, v = dev(r["q"], "bf16"), dev(r["k"], "bf16"), dev(r["v"], "bf16")
    o = torch.empty_like(q)
    n = L.samba_swa_workspace_size(Bn, Ln, Hq, Hkv, hd, 10000.0, 1)
    ws = torch.empty(n, dtype=torch.uint8, device="cuda")
    L.samba_swa_fwd(q, k, v, o, Bn, Ln, Hq, Hkv, hd, window, 10000.0, pos0, 0.0, 1, ws, n)
    torch.cuda.synchronize()
    assert L.samba_get_error() == 0
    pos = np.arange(pos0, pos0 + Ln)
    ref = O.swa(O.rope(r["q"], pos, 1e4), O.rope(r["k"], pos, 1e4), r["v"], window)
    assert attn_err(host(o), ref) <= TOL["bf16"]


@pytest.mark.parametrize("M,N,K,epi", [(300, 208, 5632, 0), (1000, 5632, 176, 3), (257, 176, 2816, 0),
                                       (130, 2816, 9984, 1)])
def test_projection_tails(L, M, N, K, epi):
    import torch
    x = I.draw_normal(41, "x", (M, K), 1.0, "bf16")
    W = I.draw_normal(41, "W", (N, K), 0.05, "bf16")
    bias = I.draw_normal(41, "b", (N,), 1.0, "f32")
    resid = I.draw_normal(41, "r", (M, N), 1.0, "bf16")
    out = torch.empty(M, N, device="cuda", dtype=torch.bfloat16)
    L.samba_linear(dev(x, "bf16"), dev(W, "bf16"), None, dev(bias), dev(resid, "bf16"), out, M, N, K, epi, 1)
    torch.cuda.synchronize()
    assert L.samba_get_error() == 0
    h = O.linear(x, W)
    if epi == 1:
        got = host(out)
        assert rel_err(got - resid, h, slack=sum_slack(got, "bf16")) <= TOL["bf16"]
    else:
        ref = O.softplus(h + bias) if epi == 3 else h
        assert rel_err(host(out), ref) <= TOL["bf16"]


def test_block_38b_shapes(L):
    shape = I.WIDE38
    W = I.block_weights(shape, 42)
    x = I.block_input(shape, 42, 1, 2304)
    g = GpuBlock(L, shape, W, 1, 2304)
    out, br, rs = g.prefill(x)
    check_branches(shape, W, x, out, br, rs, TOL["bf16"])


def test_decode_steps_38b_shapes(L):
    """samba_step at the 3.8B widths (11 query heads over one kv head of 256):
    prefill 300 tokens, then 3 decode steps, against the oracle's prefill of the
    longer sequence; positions exact."""
    from tests.test_block_gpu import step_err
    shape = I.WIDE38
    W = I.block_weights(shape, 43)
    P, S = 300, 3
    x = I.block_input(shape, 43, 2, P + S)
    g = GpuBlock(L, shape, W, 2, P + S)
    g.prefill(x[:, :P], taps=False)
    full = O.block_fwd(x, W, shape)
    for i in range(S):
        y = host(g.step(x[:, P + i]))
        assert step_err(y, x[:, P + i], full, P + i, "bf16") <= TOL["bf16"], i
    assert np.array_equal(host(g.pos), np.full(2, P + S))
