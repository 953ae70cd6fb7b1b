"""Samba block prefill (samba_block_fwd) and decode step (samba_step) against
the fp64 oracle: per-sub-layer branch outputs, the residual stream, the decode
state handoff, prefill+step == longer prefill, and state save/restore."""
import numpy as np
import pytest

from oracle import samba_oracle as O
from sliding_window_attention_samba_b200 import inputs as I
from tests.helpers import TOL, block_weights_dev, dev, host, path_err, rel_err, stream_slack

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def L():
    import torch
    from sliding_window_attention_samba_b200 import _lib
    torch.cuda.init()
    return _lib


class GpuBlock:
    """Device-side block: weights, config, workspace, decode state."""

    def __init__(self, L_, shape, W, Bn, Lmax):
        import torch
        self.L, self.shape, self.Bn = L_, shape, Bn
        self.dt = shape.dtype
        self.tdt = torch.bfloat16 if self.dt == "bf16" else torch.float32
        self.Wd = block_weights_dev(W, self.dt)
        self.cfg = L_.make_config(shape)
        self.w = L_.make_weights(self.Wd)
        n = max(L_.samba_block_workspace_size(self.cfg, Bn, Lmax), L_.samba_step_workspace_size(self.cfg, Bn))
        self.ws = torch.empty(n, dtype=torch.uint8, device="cuda")
        s = shape
        self.ssm = torch.zeros(Bn, s.d_inner, s.d_state, device="cuda")
        self.conv = torch.zeros(Bn, s.d_inner, s.d_conv - 1, device="cuda", dtype=self.tdt)
        self.k_ring = torch.zeros(Bn, s.window, s.n_kv, s.head_dim, device="cuda", dtype=self.tdt)
        self.v_ring = torch.zeros_like(self.k_ring)
        self.pos = torch.zeros(Bn, dtype=torch.int64, device="cuda")
        self.st = L_.make_state(self.ssm, self.conv, self.k_ring, self.v_ring, self.pos)

    def prefill(self, x, taps=True, state=True):
        import torch
        Bn, Ln, Dm = x.shape
        xd = dev(x, self.dt)
        out = torch.empty_like(xd)
        br = [torch.empty_like(xd) for _ in range(4)] if taps else [None] * 4
        rs = [torch.empty_like(xd) for _ in range(3)] if taps else [None] * 3
        t = self.L.make_taps(br, rs) if taps else None
        self.L.samba_block_fwd(self.cfg, self.w, xd, out, self.st if state else None, t, Bn, Ln, self.ws,
                               self.ws.numel())
        torch.cuda.synchronize()
        assert self.L.samba_get_error() == 0
        return host(out), [host(b) for b in br] if taps else None, [host(r) for r in rs] if taps else None

    def step(self, xt):
        import torch
        xd = dev(xt, self.dt)
        y = torch.empty_like(xd)
        self.L.samba_step(self.cfg, self.w, xd, y, self.st, self.Bn, self.ws, self.ws.numel())
        return y


def branch_err(i, got, ref, dt):
    """A branch output of a block (tapped before its residual add)."""
    return path_err(got, ref, dt)


def check_branches(shape, W, x, out, br, rs, tol):
    """GPU branch outputs (tapped before each residual add) and residual stream
    against the oracle's own fp64 stream; a branch sees the stream through an
    RMSNorm, so the GPU's rounding of the stream stays a relative error of the
    branch input.  The stream values are checked with the allowance for their own
    storage rounding (one half-ulp per residual add that produced them)."""
    x = x.astype(np.float64)
    dt = shape.dtype
    ref = O.block_fwd(x, W, shape)
    errs = [branch_err(i, br[i], ref["branch"][i], dt) for i in range(4)]
    assert max(errs) <= tol, errs
    for i in range(3):
        assert path_err(rs[i], ref["resid"][i], dt, slack=stream_slack(ref["resid"], dt, i)) <= tol, i
    assert path_err(out - x, ref["x_out"] - x, dt, slack=stream_slack(ref["resid"], dt)) <= tol
    return errs


def step_err(y, xt, full, t, dt):
    """Decode output y at position t against the oracle's prefill of the longer
    sequence: the block's contribution y - x_t, with the stream's storage
    allowance taken from the oracle's own streams at t."""
    res = [r[:, t] for r in full["resid"]]
    return path_err(y - xt, full["x_out"][:, t] - xt, dt, slack=stream_slack(res, dt))


def test_block_tiny_f32(L):
    shape, Bn, Ln, _, seed = I.WORKLOADS["tiny_f32_L256"]
    W = I.block_weights(shape, seed, conv_bias=True)
    x = I.block_input(shape, seed, Bn, Ln)
    g = GpuBlock(L, shape, W, Bn, Ln)
    out, br, rs = g.prefill(x)
    check_branches(shape, W, x, out, br, rs, TOL["f32"])


def test_block_tiny_f32_ragged_batch(L):
    shape = I.TINY
    W = I.block_weights(shape, 11)
    x = I.block_input(shape, 11, 3, 77)
    g = GpuBlock(L, shape, W, 3, 77)
    out, br, rs = g.prefill(x)
    check_branches(shape, W, x, out, br, rs, TOL["f32"])


def test_block_wide_bf16_prefix(L):
    """2048-wide block at B=2, L=2304 (past the 2048 window)."""
    shape = I.WIDE
    W = I.block_weights(shape, 1)
    x = I.block_input(shape, 1, 2, 2304)
    g = GpuBlock(L, shape, W, 2, 2304)
    out, br, rs = g.prefill(x)
    check_branches(shape, W, x[:1], out[:1], [b[:1] for b in br], [r[:1] for r in rs], TOL["bf16"])


@pytest.mark.parametrize("P,S", [(70, 6), (5, 3), (63, 4)])
def test_prefill_then_step_tiny_f32(L, P, S):
    shape = I.TINY
    W = I.block_weights(shape, 0, conv_bias=True)
    x = I.block_input(shape, 0, 2, P + S)
    full = O.block_fwd(x, W, shape, want_state=True)
    g = GpuBlock(L, shape, W, 2, P + S)
    g.prefill(x[:, :P], taps=False)
    for i in range(S):
        y = host(g.step(x[:, P + i]))
        assert step_err(y, x[:, P + i], full, P + i, "f32") <= TOL["f32"], i
    assert rel_err(host(g.ssm), full["state"]["ssm"]) <= TOL["f32"]
    assert np.array_equal(host(g.pos), full["state"]["pos"])


def test_prefill_state_handoff_wide_bf16(L):
    shape = I.WIDE
    W = I.block_weights(shape, 4)
    P = 2100  # wraps the 2048-slot ring
    x = I.block_input(shape, 4, 1, P + 2)
    g = GpuBlock(L, shape, W, 1, P + 2)
    g.prefill(x[:, :P], taps=False)
    r = O.block_fwd(x[:, :P], W, shape, want_state=True)
    ref = r["state"]
    assert np.array_equal(host(g.pos), ref["pos"])
    assert path_err(host(g.ssm), ref["ssm"], "bf16") <= TOL["bf16"]
    assert rel_err(host(g.conv), ref["conv"]) <= TOL["bf16"]  # a bf16 copy of stored inputs
    kr = host(g.k_ring)[0]
    # ring bookkeeping, integer-exact: every slot holds the key of position p with p mod w == slot
    oracle_k = r["attn"]["k"][0]  # [P, n_kv, d]
    flat = oracle_k.reshape(P, -1)
    for slot in range(0, shape.window, 97):
        p_expect = P - 1 - ((P - 1 - slot) % shape.window)
        dist = np.linalg.norm(flat - kr[slot].reshape(1, -1), axis=1)
        assert int(np.argmin(dist)) == p_expect
    # two decode steps continue the sequence
    full = O.block_fwd(x, W, shape)
    for i in range(2):
        y = host(g.step(x[:, P + i]))
        assert step_err(y, x[:, P + i], full, P + i, "bf16") <= TOL["bf16"]


def test_step_state_save_restore_bit_exact_and_graph(L):
    import torch
    shape = I.TINY
    W = I.block_weights(shape, 2)
    x = I.block_input(shape, 2, 4, 90)
    g = GpuBlock(L, shape, W, 4, 90)
    g.prefill(x[:, :60], taps=False)
    snap = [t.clone() for t in (g.ssm, g.conv, g.k_ring, g.v_ring, g.pos)]
    ys1 = [g.step(x[:, 60 + i]).clone() for i in range(10)]
    for t, s in zip((g.ssm, g.conv, g.k_ring, g.v_ring, g.pos), snap):
        t.copy_(s)
    ys2 = [g.step(x[:, 60 + i]).clone() for i in range(10)]
    for a, b in zip(ys1, ys2):
        assert torch.equal(a, b)
    # CUDA graph capture and replay of one step reproduces eager stepping
    for t, s in zip((g.ssm, g.conv, g.k_ring, g.v_ring, g.pos), snap):
        t.copy_(s)
    xin = dev(x[:, 60], g.dt)
    yout = torch.empty_like(xin)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        gr = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gr, stream=s):
            L.samba_step(g.cfg, g.w, xin, yout, g.st, 4, g.ws, g.ws.numel(), stream=s)
    torch.cuda.current_stream().wait_stream(s)
    for t, s_ in zip((g.ssm, g.conv, g.k_ring, g.v_ring, g.pos), snap):
        t.copy_(s_)
    for i in range(10):
        xin.copy_(dev(x[:, 60 + i], g.dt))
        gr.replay()
        torch.cuda.synchronize()
        assert torch.equal(yout, ys1[i]), i


def test_decode_steps_wide_bf16_batch4(L):
    """Batch-4 decode at the 2048-wide shapes (skinny tensor-core projections,
    per-row RoPE positions, ring attention) against the oracle's longer prefill."""
    shape = I.WIDE
    W = I.block_weights(shape, 6)
    P, S = 300, 3
    x = I.block_input(shape, 6, 4, P + S)
    g = GpuBlock(L, shape, W, 4, P + S)
    g.prefill(x[:, :P], taps=False)
    full = O.block_fwd(x, W, shape)
    for i in range(S):
        y = host(g.step(x[:, P + i]))
        assert step_err(y, x[:, P + i], full, P + i, "bf16") <= TOL["bf16"], i


def test_decode_norm_fold_on_off_wide_bf16_batch3(L, monkeypatch):
    """The decode step's norm fold (the three RMSNorms after the first ride on
    the projections around them: the producer writes x (.) g and per-8-feature
    sums of squares, the consumer scales its rows by the RMS) against the plain
    RMSNorm launches (SAMBA_NORM_FOLD=0): both within tolerance of the oracle,
    close to each other, and the folded step bit-reproducible from the same
    state (its sums are reduced in a fixed order)."""
    import torch
    shape = I.WIDE
    W = I.block_weights(shape, 16)
    P, S, Bn = 200, 3, 3
    x = I.block_input(shape, 16, Bn, P + S)
    g = GpuBlock(L, shape, W, Bn, P + S)
    g.prefill(x[:, :P], taps=False)
    full = O.block_fwd(x, W, shape)
    state = (g.ssm, g.conv, g.k_ring, g.v_ring, g.pos)
    snap = [t.clone() for t in state]

    def run():
        for t, s_ in zip(state, snap):
            t.copy_(s_)
        return [g.step(x[:, P + i]).clone() for i in range(S)]
    folded, again = run(), run()
    monkeypatch.setenv("SAMBA_NORM_FOLD", "0")
    plain = run()
    for i in range(S):
        assert torch.equal(folded[i], again[i]), i
        for y in (folded[i], plain[i]):
            assert step_err(host(y), x[:, P + i], full, P + i, "bf16") <= TOL["bf16"], i
        contrib = plain[i].float() - dev(x[:, P + i], g.dt).float()  # the block's part of the output
        d = float((folded[i].float() - plain[i].float()).norm() / contrib.norm())
        assert d <= 1e-2, (i, d)


def _ring_map_exact(ring, oracle_k, cur, w):
    """The ring's slot -> position map after `cur` tokens, bit-exact: every slot
    holds the key of the latest position p < cur with p mod w == slot (slots
    never written yet, when cur < w, are skipped).  A slot's position is read as
    the oracle key nearest to the stored one."""
    Bn = ring.shape[0]
    flat = oracle_k[:, :cur].reshape(Bn, cur, -1)
    for b in range(Bn):
        for slot in range(min(w, cur)):
            p_expect = cur - 1 - ((cur - 1 - slot) % w)
            dist = np.linalg.norm(flat[b] - ring[b, slot].reshape(1, -1), axis=1)
            assert int(np.argmin(dist)) == p_expect, (b, slot, cur)


def test_decode_ring_wraps_32x_tiny_f32(L):
    """2100 decode steps over a 64-slot ring (32.8 wraps) after a 10-token
    prefill, batch 2: every step's output against the oracle's prefill of the
    whole sequence; the position counter and the ring's slot -> position map
    bit-exact at checkpoints around and far past the wraps."""
    import torch
    shape = I.TINY
    w = shape.window
    P, S, Bn = 10, 2100, 2
    W = I.block_weights(shape, 21, conv_bias=True)
    x = I.block_input(shape, 21, Bn, P + S)
    full = O.block_fwd(x, W, shape)
    g = GpuBlock(L, shape, W, Bn, P + S)
    g.prefill(x[:, :P], taps=False)
    xd = dev(x, "f32")
    ys = torch.empty(S, Bn, shape.d_model, device="cuda")
    checks = {w - P - 1, w - P, 1000, S - 1}
    for i in range(S):
        L.samba_step(g.cfg, g.w, xd[:, P + i].contiguous(), ys[i], g.st, Bn, g.ws, g.ws.numel())
        if i in checks:
            cur = P + i + 1
            assert np.array_equal(host(g.pos), np.full(Bn, cur))
            _ring_map_exact(host(g.k_ring), full["attn"]["k"], cur, w)
    torch.cuda.synchronize()
    assert L.samba_get_error() == 0
    yh = host(ys)
    errs = [step_err(yh[i], x[:, P + i], full, P + i, "f32") for i in range(S)]
    assert max(errs) <= TOL["f32"], int(np.argmax(errs))


def test_decode_ring_wraps_wide_bf16(L):
    """800 decode steps of the 2048-wide block over a 256-slot ring (3.5 wraps)
    after a 100-token prefill: sampled steps around each wrap against the
    oracle's prefill of the whole sequence, the ring map bit-exact at the end."""
    import dataclasses
    import torch
    shape = dataclasses.replace(I.WIDE, window=256)
    w = shape.window
    P, S = 100, 800
    W = I.block_weights(shape, 22)
    x = I.block_input(shape, 22, 1, P + S)
    full = O.block_fwd(x, W, shape)
    g = GpuBlock(L, shape, W, 1, P + S)
    g.prefill(x[:, :P], taps=False)
    xd = dev(x, "bf16")
    ys = torch.empty(S, 1, shape.d_model, device="cuda", dtype=torch.bfloat16)
    for i in range(S):
        L.samba_step(g.cfg, g.w, xd[:, P + i].contiguous(), ys[i], g.st, 1, g.ws, g.ws.numel())
    torch.cuda.synchronize()
    assert L.samba_get_error() == 0
    yh = host(ys)
    for i in (0, 1, w - P - 1, w - P, w - P + 1, 2 * w - P, 3 * w - P, S - 1):
        assert step_err(yh[i], x[:, P + i], full, P + i, "bf16") <= TOL["bf16"], i
    cur = P + S
    assert np.array_equal(host(g.pos), np.full(1, cur))
    _ring_map_exact(host(g.k_ring), full["attn"]["k"], cur, w)


@pytest.mark.parametrize("shape_name", ["TINY", "WIDE"])
def test_step_refuses_negative_position(L, shape_name):
    """A corrupted decode state (a negative position) is reported as
    SAMBA_ERR_DEVICE and nothing is written into the rings: the ring write
    (CUDA-core path) or the fused ring columns of the skinny QKV projection
    check the position before forming a slot."""
    import torch
    shape = getattr(I, shape_name)
    W = I.block_weights(shape, 9)
    x = I.block_input(shape, 9, 2, 40)
    g = GpuBlock(L, shape, W, 2, 40)
    g.prefill(x[:, :39], taps=False)
    k0, v0 = g.k_ring.clone(), g.v_ring.clone()
    g.pos[1] = -5
    g.step(x[:, 39])
    torch.cuda.synchronize()
    assert L.samba_get_error() == L.SAMBA_ERR_DEVICE
    assert torch.equal(g.k_ring[1], k0[1]) and torch.equal(g.v_ring[1], v0[1])
    assert L.samba_get_error() == L.SAMBA_OK  # read and cleared; the context stays usable


def test_decode_streaming_attention_B28(L):
    """Enough (kv head, batch row) pairs for the streaming decode attention (one
    CTA per pair walking every valid slot in 64-slot TMA tiles): 28 rows x 4 kv
    heads at the 2048-wide shapes, 150 prefilled tokens (a partial last tile),
    three steps against the oracle's longer prefill, every row."""
    shape = I.WIDE
    W = I.block_weights(shape, 12)
    P, S = 150, 3
    x = I.block_input(shape, 12, 28, P + S)
    g = GpuBlock(L, shape, W, 28, P + S)
    g.prefill(x[:, :P], taps=False)
    full = O.block_fwd(x, W, shape)
    for i in range(S):
        y = host(g.step(x[:, P + i]))
        assert step_err(y, x[:, P + i], full, P + i, "bf16") <= TOL["bf16"], i


def test_decode_wide_bf16_conv_bias(L):
    """The short-conv step folded into the skinny in_proj epilogue, with a conv
    bias (bf16, 2048-wide shapes): prefill + three steps against the oracle's
    longer prefill."""
    shape = I.WIDE
    W = I.block_weights(shape, 13, conv_bias=True)
    P, S = 70, 3
    x = I.block_input(shape, 13, 2, P + S)
    g = GpuBlock(L, shape, W, 2, P + S)
    g.prefill(x[:, :P], taps=False)
    full = O.block_fwd(x, W, shape)
    for i in range(S):
        y = host(g.step(x[:, P + i]))
        assert step_err(y, x[:, P + i], full, P + i, "bf16") <= TOL["bf16"], i


@pytest.mark.parametrize("Bn", [28, 2])
def test_decode_window_4096(L, Bn):
    """A 4096-slot ring in samba_step: at 28 rows x 4 kv heads the streaming
    decode attention (its largest window), at 2 rows the per-slice kernel with
    the partials in samba_step's own workspace; 100 prefilled tokens, two steps."""
    import dataclasses
    shape = dataclasses.replace(I.WIDE, window=4096)
    W = I.block_weights(shape, 14)
    P, S = 100, 2
    x = I.block_input(shape, 14, Bn, P + S)
    g = GpuBlock(L, shape, W, Bn, P + S)
    g.prefill(x[:, :P], taps=False)
    full = O.block_fwd(x, W, shape)
    for i in range(S):
        y = host(g.step(x[:, P + i]))
        assert step_err(y, x[:, P + i], full, P + i, "bf16") <= TOL["bf16"], i


def test_block_wide_bf16_folded_dt(L):
    """SAMBA_SCAN_FOLD_DT=1: the block's scan forms Delta itself from the x_proj
    output (no dt projection launch); every branch against the oracle."""
    shape = I.WIDE
    W = I.block_weights(shape, 15)
    x = I.block_input(shape, 15, 1, 300)
    import os
    os.environ["SAMBA_SCAN_FOLD_DT"] = "1"
    try:
        g = GpuBlock(L, shape, W, 1, 300)
        out, br, rs = g.prefill(x)
    finally:
        del os.environ["SAMBA_SCAN_FOLD_DT"]
    check_branches(shape, W, x, out, br, rs, TOL["bf16"])
