"""Parity at the workloads' full sizes, in the launch configurations bench.py
times, on outputs the fp64 oracle can compute one by one:

* the 4-block L = 131072 prefill stack: the first 2304 tokens of every block's
  output (causality makes a prefix exact), past the 2048 window;
* the B = 4, L = 4096 block: one full batch row (rows are independent);
* decode at B = 32 after a 4096-token prefill: one batch row, 3 steps;
* the mixers at L = 2^20: sampled scan channels and sampled SWA rows.  The GPU
  sees full-size tensors; the sampled channels (scan) or the query row and its
  key band (SWA) hold seeded host values, and since channels and rows outside a
  band do not interact, those outputs depend on host values only.
"""
import numpy as np
import pytest

from oracle import samba_oracle as O
from sliding_window_attention_samba_b200 import inputs as I
from tests.helpers import TOL, attn_err, block_weights_dev, dev, host, path_err, rel_err, stream_slack
from tests.test_block_gpu import branch_err, step_err

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def L():
    import torch
    from sliding_window_attention_samba_b200 import _lib
    torch.cuda.init()
    return _lib


def _state(torch, s, Bn, tdt):
    ssm = torch.zeros(Bn, s.d_inner, s.d_state, device="cuda")
    conv = torch.zeros(Bn, s.d_inner, s.d_conv - 1, device="cuda", dtype=tdt)
    kr = torch.zeros(Bn, s.window, s.n_kv, s.head_dim, device="cuda", dtype=tdt)
    vr = torch.zeros_like(kr)
    pos = torch.zeros(Bn, dtype=torch.int64, device="cuda")
    return ssm, conv, kr, vr, pos


def test_prefill_stack_L131072_prefix(L):
    """Every block of the stack runs on the GPU's own stream; the oracle runs the
    same 4 blocks on its own fp64 stream.  Compared: each block's four branch
    outputs (tapped before their residual adds) and its contribution (output
    minus input, each side's own input), first 2304 tokens."""
    import torch
    shape, Bn, Ln, nb, seed = I.WORKLOADS["prefill_bf16_L131072_x4"]
    P = 2304
    x = I.block_input(shape, seed, Bn, Ln)
    cfg = L.make_config(shape)
    n = L.samba_block_workspace_size(cfg, Bn, Ln)
    ws = torch.empty(n, dtype=torch.uint8, device="cuda")
    cur = dev(x, "bf16")
    nxt = torch.empty_like(cur)
    br = [torch.empty_like(cur) for _ in range(4)]
    taps = L.make_taps(br)
    xo = x[:, :P].astype(np.float64)
    for li in range(nb):
        W = I.block_weights(shape, seed, layer=li)
        Wd = block_weights_dev(W, "bf16")
        gin = host(cur[:, :P])  # this block's input on the GPU's own stream
        L.samba_block_fwd(cfg, L.make_weights(Wd), cur, nxt, None, taps, Bn, Ln, ws, n)
        torch.cuda.synchronize()
        assert L.samba_get_error() == 0
        assert torch.isfinite(nxt).all()
        ref = O.block_fwd(xo, W, shape)
        for i in range(4):
            assert branch_err(i, host(br[i][:, :P]), ref["branch"][i], "bf16") <= TOL["bf16"], (li, i)
        assert path_err(host(nxt[:, :P]) - gin, ref["x_out"] - xo, "bf16",
                        slack=stream_slack(ref["resid"], "bf16")) <= TOL["bf16"], li
        xo = ref["x_out"]
        cur, nxt = nxt, cur
        del Wd


def test_block_B4_L4096_one_full_row(L):
    import torch
    shape, Bn, Ln, _, seed = I.WORKLOADS["block_bf16_B4_L4096"]
    W = I.block_weights(shape, seed)
    x = I.block_input(shape, seed, Bn, Ln)
    cfg = L.make_config(shape)
    n = L.samba_block_workspace_size(cfg, Bn, Ln)
    ws = torch.empty(n, dtype=torch.uint8, device="cuda")
    xd = dev(x, "bf16")
    out = torch.empty_like(xd)
    L.samba_block_fwd(cfg, L.make_weights(block_weights_dev(W, "bf16")), xd, out, None, None, Bn, Ln, ws, n)
    torch.cuda.synchronize()
    assert L.samba_get_error() == 0
    row = 2
    ref = O.block_fwd(x[row:row + 1], W, shape)
    got = host(out[row:row + 1])
    assert path_err(got - x[row:row + 1], ref["x_out"] - x[row:row + 1], "bf16",
                    slack=stream_slack(ref["resid"], "bf16")) <= TOL["bf16"]


def test_decode_B32_after_4096_prefill(L):
    import torch
    shape, Bn, P, _, seed = I.WORKLOADS["decode_bf16_B32"]
    S = 3
    W = I.block_weights(shape, seed)
    x = I.block_input(shape, seed, Bn, P + S)
    cfg = L.make_config(shape)
    Wd = block_weights_dev(W, "bf16")  # the struct holds raw pointers: keep the tensors alive
    wst = L.make_weights(Wd)
    n = max(L.samba_block_workspace_size(cfg, Bn, P), L.samba_step_workspace_size(cfg, Bn))
    ws = torch.empty(n, dtype=torch.uint8, device="cuda")
    st_t = _state(torch, shape, Bn, torch.bfloat16)
    st = L.make_state(*st_t)
    xp = dev(x[:, :P], "bf16")
    L.samba_block_fwd(cfg, wst, xp, torch.empty_like(xp), st, None, Bn, P, ws, n)
    ys = []
    for i in range(S):
        xt = dev(x[:, P + i], "bf16")
        yt = torch.empty_like(xt)
        L.samba_step(cfg, wst, xt, yt, st, Bn, ws, n)
        ys.append(host(yt))
    torch.cuda.synchronize()
    assert L.samba_get_error() == 0
    assert np.array_equal(host(st_t[4]), np.full(Bn, P + S))
    row = 17
    ref = O.block_fwd(x[row:row + 1], W, shape)
    for i in range(S):
        assert step_err(ys[i][row:row + 1], x[row:row + 1, P + i], ref, P + i, "bf16") <= TOL["bf16"], i


def test_scan_L1M_sampled_channels(L):
    import torch
    Ln, D, N = 1 << 20, 4096, 16
    chans = [0, 1, 777, 2048, 4095]
    seed = I.MIXER_SWEEP_SEED
    g = torch.Generator(device="cuda")
    g.manual_seed(1)
    bf = torch.bfloat16
    u = torch.randn(1, Ln, D, generator=g, device="cuda").to(bf)
    dt = torch.randn(1, Ln, D, generator=g, device="cuda").to(bf)
    z = torch.randn(1, Ln, D, generator=g, device="cuda").to(bf)
    host_in = {}
    for name, t in (("u", u), ("dt", dt), ("z", z)):
        vals = I.draw_normal(seed, f"fullscan.{name}", (Ln, len(chans)), 1.0, "bf16")
        host_in[name] = vals
        t[0, :, chans] = torch.from_numpy(vals).to("cuda", bf)
    Bh = I.draw_normal(seed, "fullscan.B", (1, Ln, N), 1.0, "bf16")
    Ch = I.draw_normal(seed, "fullscan.C", (1, Ln, N), 1.0, "bf16")
    bias = I.dt_bias_init(seed, "scan.dt_bias", D)
    A_log = I.a_log_init(D, N)
    y = torch.empty_like(u)
    hT = torch.empty(1, D, N, device="cuda")
    L.samba_selective_scan(u, dt, dev(bias), 1, dev(A_log), dev(Bh, "bf16"), dev(Ch, "bf16"),
                           dev(np.ones(D, np.float32)), z, None, hT, y, 1, Ln, D, N, 1)
    torch.cuda.synchronize()
    assert L.samba_get_error() == 0
    yg = host(y[0, :, chans])
    hg = host(hT[0, chans])
    delta = O.softplus(host_in["dt"][None] + bias[chans])
    yo, ho = O.selective_scan(host_in["u"][None], delta, -np.exp(A_log[chans].astype(np.float64)), Bh, Ch,
                              np.ones(len(chans)), host_in["z"][None])
    assert rel_err(yg, yo[0]) <= TOL["bf16"]
    assert rel_err(hg, ho[0]) <= TOL["bf16"]
    for j in range(len(chans)):  # late positions pin the carry across ~16K chunks
        assert rel_err(yg[-4096:, j], yo[0, -4096:, j]) <= TOL["bf16"], j


def test_swa_L1M_sampled_rows(L):
    import torch
    Ln, Hq, Hkv, hd, w = 1 << 20, 32, 4, 64, 2048
    rows = [0, 1, 2047, 2048, 500000, Ln - 1]
    seed = I.MIXER_SWEEP_SEED
    g = torch.Generator(device="cuda")
    g.manual_seed(2)
    bf = torch.bfloat16
    q = torch.randn(1, Ln, Hq, hd, generator=g, device="cuda").to(bf)
    k = torch.randn(1, Ln, Hkv, hd, generator=g, device="cuda").to(bf)
    v = torch.randn(1, Ln, Hkv, hd, generator=g, device="cuda").to(bf)

    def rows_of(name, lo, hi, heads):
        """Seeded values of token rows lo..hi-1 (counter-based: a row's values do
        not depend on which band asked for it)."""
        width = heads * hd
        vals = I.normals(I.tensor_key(seed, name), (hi - lo) * width, start=lo * width)
        return I.round_to(vals, "bf16").reshape(1, hi - lo, heads, hd)

    bands = {}
    for t in rows:
        lo = max(0, t - w + 1)
        bands[t] = (lo, rows_of("fullswa.q", t, t + 1, Hq), rows_of("fullswa.k", lo, t + 1, Hkv),
                    rows_of("fullswa.v", lo, t + 1, Hkv))
        q[:, t:t + 1] = torch.from_numpy(bands[t][1]).to("cuda", bf)
        k[:, lo:t + 1] = torch.from_numpy(bands[t][2]).to("cuda", bf)
        v[:, lo:t + 1] = torch.from_numpy(bands[t][3]).to("cuda", bf)
    o = torch.empty_like(q)
    n = L.samba_swa_workspace_size(1, Ln, Hq, Hkv, hd, 10000.0, 1)
    ws = torch.empty(n, dtype=torch.uint8, device="cuda")
    L.samba_swa_fwd(q, k, v, o, 1, Ln, Hq, Hkv, hd, w, 10000.0, 0, 0.0, 1, ws, n)
    torch.cuda.synchronize()
    assert L.samba_get_error() == 0
    grp = Hq // Hkv
    for t in rows:
        lo, qh, kh, vh = bands[t]
        qr = O.rope(qh, [t], 10000.0)
        kr = O.rope(kh, np.arange(lo, t + 1), 10000.0)
        ref = np.zeros((Hq, hd))
        for h in range(Hq):
            sc = kr[0, :, h // grp] @ qr[0, 0, h] / np.sqrt(hd)
            p = np.exp(sc - sc.max())
            ref[h] = (p / p.sum()) @ vh[0, :, h // grp].astype(np.float64)
        assert attn_err(host(o[0, t]), ref) <= TOL["bf16"], t
