"""Chunked prefill (samba_block_fwd_chunk): a sequence fed in chunks, each
continuing from the decode state the previous one left, against the fp64
oracle over the whole sequence — per-branch outputs of every chunk, the state
after the last chunk, and decode steps after it.  Chunk lists cover chunks
shorter than the conv history, empty chunks, chunks that start inside the
first window (fewer than window-1 earlier keys) and past it."""
import os

import numpy as np
import pytest

from oracle import samba_oracle as O
from sliding_window_attention_samba_b200 import inputs as I
from tests.helpers import TOL, block_weights_dev, dev, host, path_err, rel_err, stream_slack, sum_slack
from tests.test_block_gpu import branch_err, step_err

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def L():
    import torch
    from sliding_window_attention_samba_b200 import _lib
    torch.cuda.init()
    return _lib


class ChunkedBlock:
    def __init__(self, L_, shape, W, Bn, Lmax):
        import torch
        self.L, self.shape, self.Bn, self.dt = L_, shape, Bn, shape.dtype
        self.tdt = torch.bfloat16 if self.dt == "bf16" else torch.float32
        self.Wd = block_weights_dev(W, self.dt)
        self.cfg = L_.make_config(shape)
        self.w = L_.make_weights(self.Wd)
        n = max(L_.samba_block_chunk_workspace_size(self.cfg, Bn, Lmax), L_.samba_step_workspace_size(self.cfg, Bn))
        self.ws = torch.empty(n, dtype=torch.uint8, device="cuda")
        s = shape
        self.ssm = torch.full((Bn, s.d_inner, s.d_state), float("nan"), device="cuda")  # pos0 = 0 must ignore it
        self.conv = torch.full((Bn, s.d_inner, s.d_conv - 1), float("nan"), device="cuda", dtype=self.tdt)
        self.k_ring = torch.zeros(Bn, s.window, s.n_kv, s.head_dim, device="cuda", dtype=self.tdt)
        self.v_ring = torch.zeros_like(self.k_ring)
        self.pos = torch.zeros(Bn, dtype=torch.int64, device="cuda")
        self.st = L_.make_state(self.ssm, self.conv, self.k_ring, self.v_ring, self.pos)
        self.p = 0

    def chunk(self, x):
        """x: [B, Lc, d_model] host values; returns (x_out, four branch taps)."""
        import torch
        Bn, Lc, _ = x.shape
        xd = dev(x, self.dt)
        out = torch.empty_like(xd)
        br = [torch.empty_like(xd) for _ in range(4)]
        self.L.samba_block_fwd_chunk(self.cfg, self.w, xd, out, self.st, self.p, self.L.make_taps(br), Bn, Lc,
                                     self.ws, self.ws.numel())
        torch.cuda.synchronize()
        assert self.L.samba_get_error() == 0
        self.p += Lc
        return host(out), [host(b) for b in br]

    def step(self, xt):
        import torch
        xd = dev(xt, self.dt)
        y = torch.empty_like(xd)
        self.L.samba_step(self.cfg, self.w, xd, y, self.st, self.Bn, self.ws, self.ws.numel())
        return host(y)


def _run_chunks(L, shape, W, x, chunks, tol, steps=2):
    Bn = x.shape[0]
    total = sum(chunks)
    assert x.shape[1] == total + steps
    ref = O.block_fwd(x, W, shape, want_state=True)  # whole sequence, incl. the decode tokens
    refp = O.block_fwd(x[:, :total], W, shape, want_state=True)["state"]
    g = ChunkedBlock(L, shape, W, Bn, max(max(chunks), 1))
    p = 0
    for ci, Lc in enumerate(chunks):
        out, br = g.chunk(x[:, p:p + Lc])
        if Lc:
            for i in range(4):
                assert branch_err(i, br[i], ref["branch"][i][:, p:p + Lc], shape.dtype) <= tol, (ci, i)
            res = [r[:, p:p + Lc] for r in ref["resid"]]
            assert path_err(out - x[:, p:p + Lc], ref["x_out"][:, p:p + Lc] - x[:, p:p + Lc], shape.dtype,
                            slack=stream_slack(res, shape.dtype)) <= tol, ci
        p += Lc
    assert np.array_equal(host(g.pos), np.full(Bn, total))
    assert path_err(host(g.ssm), refp["ssm"], shape.dtype) <= tol
    assert rel_err(host(g.conv), refp["conv"]) <= tol
    n = min(total, shape.window)
    slots = [(total - n + j) % shape.window for j in range(n)]
    assert rel_err(host(g.k_ring)[:, slots], refp["k_ring"][:, slots]) <= tol
    assert rel_err(host(g.v_ring)[:, slots], refp["v_ring"][:, slots]) <= tol
    for i in range(steps):
        y = g.step(x[:, total + i])
        assert step_err(y, x[:, total + i], ref, total + i, shape.dtype) <= tol, i


@pytest.mark.parametrize("chunks", [[70, 90], [1, 2, 33, 0, 64, 60], [200, 56], [0, 5, 1, 1, 1, 130]])
def test_chunked_prefill_tiny_f32(L, chunks):
    shape = I.TINY  # window 64, d_conv 4
    W = I.block_weights(shape, 7, conv_bias=True)
    x = I.block_input(shape, 7, 2, sum(chunks) + 2)
    _run_chunks(L, shape, W, x, chunks, TOL["f32"])


@pytest.mark.parametrize("kernel", ["", "2", "1"])
def test_chunked_prefill_wide_bf16(L, kernel):
    """2048-wide block at B = 1 in chunks of 1000, 1500, 700: the second chunk
    starts 1000 tokens in (1000 earlier keys, not a tile multiple), the third past
    the window (2047 earlier keys).  kernel "2" / "1" run the two-head / one-head
    per CTA tensor-core attention kernels instead of the four-head one."""
    shape = I.WIDE
    W = I.block_weights(shape, 8)
    chunks = [1000, 1500, 700]
    x = I.block_input(shape, 8, 1, sum(chunks) + 2)
    old = os.environ.get("SAMBA_SWA_KERNEL")
    if kernel:
        os.environ["SAMBA_SWA_KERNEL"] = kernel
    try:
        _run_chunks(L, shape, W, x, chunks, TOL["bf16"])
    finally:
        if kernel:
            if old is None:
                del os.environ["SAMBA_SWA_KERNEL"]
            else:
                os.environ["SAMBA_SWA_KERNEL"] = old


def test_chunked_equals_single_call_wide_bf16(L):
    """Chunks of 128-multiples and not: the same rows as one samba_block_fwd call."""
    import torch
    shape = I.WIDE
    W = I.block_weights(shape, 9)
    Bn, chunks = 2, [640, 2048, 77, 1331]
    total = sum(chunks)
    x = I.block_input(shape, 9, Bn, total)
    g = ChunkedBlock(L, shape, W, Bn, max(chunks))
    outs, p = [], 0
    for Lc in chunks:
        outs.append(g.chunk(x[:, p:p + Lc])[0])
        p += Lc
    got = np.concatenate(outs, axis=1)
    cfg = L.make_config(shape)
    n = L.samba_block_workspace_size(cfg, Bn, total)
    ws = torch.empty(n, dtype=torch.uint8, device="cuda")
    xd = dev(x, "bf16")
    out = torch.empty_like(xd)
    L.samba_block_fwd(cfg, g.w, xd, out, None, None, Bn, total, ws, n)
    torch.cuda.synchronize()
    one = host(out)
    # both sides store their output in bf16: one half-ulp each
    assert path_err(got - x, one - x, "bf16", slack=sum_slack(one, "bf16", 2)) <= TOL["bf16"]


def test_chunk_position_mismatch_sets_device_error(L):
    """pos0 that disagrees with the state's positions is caught by the device check
    (reported by samba_get_error, which then clears the error word)."""
    import torch
    shape = I.TINY
    W = I.block_weights(shape, 3)
    x = I.block_input(shape, 3, 1, 40)
    g = ChunkedBlock(L, shape, W, 1, 40)
    g.chunk(x[:, :20])
    xd = dev(x[:, 20:], "f32")
    out = torch.empty_like(xd)
    L.samba_block_fwd_chunk(g.cfg, g.w, xd, out, g.st, 21, None, 1, 20, g.ws, g.ws.numel())
    torch.cuda.synchronize()
    assert L.samba_get_error() == L.SAMBA_ERR_DEVICE
    assert L.samba_get_error() == 0
    assert int(host(g.pos)[0]) == 41  # the state advanced as instructed; its contents are undefined
