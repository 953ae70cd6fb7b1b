"""Workload of tests/test_debug_checks_gpu.py, run in a child process with
SAMBA_DEBUG_CHECKS=1 so that the binding loads libsamba_debug.so (the library
built with device index checks and workspace guard bands).

It runs the two check self-tests, then the library's entry points on seeded
inputs with every user output placed between guard margins: the smoke
workloads (fp32 and 2048-wide bf16 block prefill + decode step against the
oracle), the selective scan with its final state, the sliding-window attention
with RoPE, a chunked prefill and decode steps.  Any failed device check, any
overwritten workspace band (samba_get_error) or user margin fails the run.
Prints one JSON line with the results."""
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

from sliding_window_attention_samba_b200 import _lib as L  # noqa: E402
from sliding_window_attention_samba_b200 import inputs as I  # noqa: E402

GUARD = 4096
PATTERN = 0x6B


class Guarded:
    """A device tensor placed between two GUARD-byte margins of a fixed byte."""

    def __init__(self, shape, dtype):
        nbytes = int(np.prod(shape)) * torch.empty((), dtype=dtype).element_size()
        self.big = torch.full((nbytes + 2 * GUARD,), PATTERN, dtype=torch.uint8, device="cuda")
        self.t = self.big[GUARD:GUARD + nbytes].view(dtype).view(*shape)

    def intact(self) -> bool:
        m = torch.cat([self.big[:GUARD], self.big[-GUARD:]])
        return bool((m == PATTERN).all().item())


def selftests(res):
    assert L.samba_get_error() == L.SAMBA_OK
    res["kind0_rc"] = L.samba_debug_check_selftest(0)
    res["kind0_err"] = L.samba_get_error()
    res["kind0_site"] = L.samba_last_check_site()
    n = L.samba_debug_selftest_workspace_size()
    ws = torch.empty(n, dtype=torch.uint8, device="cuda")
    res["kind1_rc"] = L.samba_debug_check_selftest(1, ws, n)
    res["kind1_err"] = L.samba_get_error()
    res["kind1_site"] = L.samba_last_check_site()
    res["after_err"] = L.samba_get_error()


def scan_guarded(res):
    Bn, Ln, D, N = 2, 300, 64, 16
    rng = np.random.default_rng(5)
    u = torch.from_numpy(rng.standard_normal((Bn, Ln, D))).cuda().bfloat16()
    dt = torch.from_numpy(rng.uniform(0.01, 0.2, (Bn, Ln, D))).cuda().bfloat16()
    Bm = torch.from_numpy(rng.standard_normal((Bn, Ln, N))).cuda().bfloat16()
    Cm = torch.from_numpy(rng.standard_normal((Bn, Ln, N))).cuda().bfloat16()
    z = torch.from_numpy(rng.standard_normal((Bn, Ln, D))).cuda().bfloat16()
    A_log = torch.from_numpy(np.log(rng.uniform(0.5, 8.0, (D, N)))).cuda().float()
    Dk = torch.from_numpy(rng.standard_normal(D)).cuda().float()
    y = Guarded((Bn, Ln, D), torch.bfloat16)
    hT = Guarded((Bn, D, N), torch.float32)
    L.samba_selective_scan(u, dt, None, False, A_log, Bm, Cm, Dk, z, None, hT.t, y.t, Bn, Ln, D, N, L.SAMBA_BF16)
    res["scan_err"] = L.samba_get_error()
    res["scan_margins"] = y.intact() and hT.intact()


def swa_guarded(res):
    Bn, Ln, Hq, Hkv, hd, w = 1, 400, 8, 2, 64, 128
    rng = np.random.default_rng(6)
    q = torch.from_numpy(rng.standard_normal((Bn, Ln, Hq, hd))).cuda().bfloat16()
    k = torch.from_numpy(rng.standard_normal((Bn, Ln, Hkv, hd))).cuda().bfloat16()
    v = torch.from_numpy(rng.standard_normal((Bn, Ln, Hkv, hd))).cuda().bfloat16()
    o = Guarded((Bn, Ln, Hq, hd), torch.bfloat16)
    n = L.samba_swa_workspace_size(Bn, Ln, Hq, Hkv, hd, 10000.0, L.SAMBA_BF16)
    ws = torch.empty(n, dtype=torch.uint8, device="cuda")
    L.samba_swa_fwd(q, k, v, o.t, Bn, Ln, Hq, Hkv, hd, w, 10000.0, 0, 0.0, L.SAMBA_BF16, ws, n)
    res["swa_err"] = L.samba_get_error()
    res["swa_margins"] = o.intact()


def block_chunks_steps_guarded(res):
    shape = I.WIDE
    Bn, P, C, steps = 2, 160, 96, 3
    W = I.block_weights(shape, 3)
    vec = {"norm0", "norm1", "norm2", "norm3", "conv_w", "conv_b", "dt_bias", "A_log", "D"}
    Wd = {kk: None if vv is None else torch.from_numpy(vv).cuda().to(torch.float32 if kk in vec else torch.bfloat16)
          for kk, vv in W.items()}
    cfg, w = L.make_config(shape), L.make_weights(Wd)
    x = torch.from_numpy(I.block_input(shape, 3, Bn, P + C + steps)).cuda().bfloat16()
    ssm = Guarded((Bn, shape.d_inner, 16), torch.float32)
    conv = Guarded((Bn, shape.d_inner, shape.d_conv - 1), torch.bfloat16)
    kr = Guarded((Bn, shape.window, shape.n_kv, shape.head_dim), torch.bfloat16)
    vr = Guarded((Bn, shape.window, shape.n_kv, shape.head_dim), torch.bfloat16)
    pos = Guarded((Bn,), torch.int64)
    st = L.make_state(ssm.t, conv.t, kr.t, vr.t, pos.t)
    n = max(L.samba_block_workspace_size(cfg, Bn, P), L.samba_block_chunk_workspace_size(cfg, Bn, C),
            L.samba_step_workspace_size(cfg, Bn))
    ws = torch.empty(n, dtype=torch.uint8, device="cuda")
    o1 = Guarded((Bn, P, shape.d_model), torch.bfloat16)
    L.samba_block_fwd(cfg, w, x[:, :P].contiguous(), o1.t, st, None, Bn, P, ws, n)
    o2 = Guarded((Bn, C, shape.d_model), torch.bfloat16)
    L.samba_block_fwd_chunk(cfg, w, x[:, P:P + C].contiguous(), o2.t, st, P, None, Bn, C, ws, n)
    outs = []
    for i in range(steps):
        yt = Guarded((Bn, shape.d_model), torch.bfloat16)
        L.samba_step(cfg, w, x[:, P + C + i].contiguous(), yt.t, st, Bn, ws, n)
        outs.append(yt)
    res["block_err"] = L.samba_get_error()
    res["block_margins"] = all(g.intact() for g in [ssm, conv, kr, vr, pos, o1, o2] + outs)
    res["block_pos"] = pos.t.cpu().tolist()


def main():
    assert L.DEBUG_CHECKS, "run with SAMBA_DEBUG_CHECKS=1"
    torch.cuda.set_device(0)
    res = {"enabled": L.samba_debug_checks_enabled(), "lib": os.path.basename(L.LIB_PATH)}
    selftests(res)
    scan_guarded(res)
    swa_guarded(res)
    block_chunks_steps_guarded(res)
    import __graft_entry__ as g
    g.smoke()  # oracle parity of the fp32 and bf16 block + step; asserts samba_get_error() == 0
    res["smoke"] = "ok"
    print(json.dumps(res))


if __name__ == "__main__":
    main()
