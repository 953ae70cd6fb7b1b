"""Selective scan (samba_selective_scan) against the fp64 oracle."""
import math

import numpy as np
import pytest

from oracle import samba_oracle as O
from sliding_window_attention_samba_b200 import inputs as I
from tests.helpers import TOL, dev, host, rel_err

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def L():
    import torch
    from sliding_window_attention_samba_b200 import _lib
    torch.cuda.init()
    return _lib


def run_scan(L_, r, dt, softplus=True, with_z=True, h0=None, want_hT=True):
    import torch
    Bn, Ln, D = r["u"].shape
    N = r["B"].shape[-1]
    u, dtt, Bm, Cm = dev(r["u"], dt), dev(r["dt_raw"], dt), dev(r["B"], dt), dev(r["C"], dt)
    z = dev(r["z"], dt) if with_z else None
    y = torch.empty(Bn, Ln, D, device="cuda", dtype=u.dtype)
    hT = torch.empty(Bn, D, N, device="cuda") if want_hT else None
    L_.samba_selective_scan(u, dtt, dev(r["dt_bias"]), softplus, dev(r["A_log"]), Bm, Cm, dev(r["D"]), z,
                            dev(h0) if h0 is not None else None, hT, y, Bn, Ln, D, N,
                            1 if dt == "bf16" else 0)
    torch.cuda.synchronize()
    assert L_.samba_get_error() == 0
    return host(y), (host(hT) if want_hT else None)


def oracle_scan(r, softplus=True, with_z=True, h0=None):
    delta = r["dt_raw"] + r["dt_bias"]
    if softplus:
        delta = O.softplus(delta)
    A = -np.exp(r["A_log"].astype(np.float64))
    return O.selective_scan(r["u"], delta, A, r["B"], r["C"], r["D"], r["z"] if with_z else None, h0)


@pytest.mark.parametrize("dt,Bn,Ln,D", [("f32", 1, 256, 128), ("f32", 2, 200, 64), ("bf16", 1, 4096, 4096),
                                        ("bf16", 3, 129, 256), ("bf16", 1, 1, 32), ("f32", 1, 63, 32),
                                        ("bf16", 2, 700, 48), ("f32", 1, 130, 16), ("bf16", 1, 64, 16),
                                        ("bf16", 1, 65, 16), ("bf16", 1, 4097, 1040)])
def test_scan_matches_oracle(L, dt, Bn, Ln, D):
    r = I.scan_inputs(0, Bn, Ln, D, 16, dt, with_h0=True)
    y, hT = run_scan(L, r, dt, h0=r["h0"])
    yo, ho = oracle_scan(r, h0=r["h0"])
    assert rel_err(y, yo) <= TOL[dt]
    assert rel_err(hT, ho) <= TOL[dt]


@pytest.mark.parametrize("dt", ["f32", "bf16"])
def test_scan_no_gate_no_softplus(L, dt):
    r = I.scan_inputs(5, 2, 300, 64, 16, dt)
    r["dt_raw"] = I.round_to(np.abs(r["dt_raw"]) * 0.05, dt)  # Delta given directly (>0)
    r["dt_bias"] = np.zeros_like(r["dt_bias"])
    y, hT = run_scan(L, r, dt, softplus=False, with_z=False)
    yo, ho = oracle_scan(r, softplus=False, with_z=False)
    assert rel_err(y, yo) <= TOL[dt] and rel_err(hT, ho) <= TOL[dt]


def test_scan_lti_closed_form_on_gpu(L):
    Ln, D, N = 500, 32, 16
    dlt, uv = 0.02, 0.5
    Bv = np.linspace(-1, 1, N)
    Cv = np.cos(np.arange(N))
    r = {"u": np.full((1, Ln, D), uv, np.float32), "dt_raw": np.full((1, Ln, D), dlt, np.float32),
         "B": np.tile(Bv, (1, Ln, 1)).astype(np.float32), "C": np.tile(Cv, (1, Ln, 1)).astype(np.float32),
         "z": None, "dt_bias": np.zeros(D, np.float32), "A_log": I.a_log_init(D, N), "D": np.zeros(D, np.float32)}
    y, _ = run_scan(L, r, "f32", softplus=False, with_z=False)
    a = np.exp(-dlt * np.arange(1, N + 1))
    Bv32, Cv32 = r["B"][0, 0].astype(np.float64), r["C"][0, 0].astype(np.float64)
    for t in (0, 1, 63, 64, 65, 499):
        h = np.float32(dlt) * Bv32 * np.float32(uv) * (1 - a ** (t + 1)) / (1 - a)
        assert abs(y[0, t, 0] - h @ Cv32) <= 1e-4 * max(1.0, abs(h @ Cv32))


def test_scan_impulse_prefix_is_exactly_zero(L):
    r = I.scan_inputs(2, 1, 400, 64, 16, "bf16")
    r["u"][:, :237] = 0.0
    y, _ = run_scan(L, r, "bf16")
    assert np.all(y[0, :237] == 0.0)
    assert np.any(y[0, 237] != 0.0)


def test_scan_chunk_split_carries_state(L):
    r = I.scan_inputs(7, 2, 1000, 128, 16, "f32")
    y_full, h_full = run_scan(L, r, "f32")
    cut = 333
    first = {k: (v[:, :cut] if (v is not None and v.ndim == 3 and k != "h0") else v) for k, v in r.items()}
    rest = {k: (v[:, cut:] if (v is not None and v.ndim == 3 and k != "h0") else v) for k, v in r.items()}
    y1, h1 = run_scan(L, first, "f32")
    y2, h2 = run_scan(L, rest, "f32", h0=h1.astype(np.float32))
    assert rel_err(np.concatenate([y1, y2], 1), y_full) <= 1e-5
    assert rel_err(h2, h_full) <= 1e-5


def test_scan_empty_sequence_copies_state(L):
    import torch
    h0 = np.random.default_rng(0).standard_normal((2, 64, 16)).astype(np.float32)
    hT = torch.empty(2, 64, 16, device="cuda")
    u = torch.zeros(16, device="cuda")
    L.samba_selective_scan(u, u, None, 1, torch.zeros(64, 16, device="cuda"), u, u, None, None, dev(h0), hT, u,
                           2, 0, 64, 16, 0)
    torch.cuda.synchronize()
    assert np.array_equal(host(hT), h0)


def test_scan_batch_rows_independent_bit_exact(L):
    r = I.scan_inputs(9, 3, 257, 64, 16, "bf16")
    y3, h3 = run_scan(L, r, "bf16")
    one = {k: (v[1:2] if (v is not None and v.ndim == 3) else v) for k, v in r.items()}
    y1, h1 = run_scan(L, one, "bf16")
    assert np.array_equal(y3[1:2], y1) and np.array_equal(h3[1:2], h1)


@pytest.mark.parametrize("Ln", [31, 32, 33, 64, 65, 96, 130, 4097])
def test_scan_ragged_lengths_bf16(L, Ln):
    """Lengths around the 64-token chunk and the 8-token warp sub-chunks."""
    r = I.scan_inputs(8, 1, Ln, 64, 16, "bf16", with_h0=True)
    y, hT = run_scan(L, r, "bf16", h0=r["h0"])
    yo, ho = oracle_scan(r, h0=r["h0"])
    assert rel_err(y, yo) <= TOL["bf16"] and rel_err(hT, ho) <= TOL["bf16"]


def test_scan_bounded_wait_times_out_and_recovers(L):
    """Failure detection without a fault: the test hook makes the scan's loader
    stop after 3 of 8 chunks and shortens the wait limit to 5 ms.  The consumer's
    wait for chunk 3 runs out, the kernel latches SAMBA_ERR_TIMEOUT, drains its
    own output stores and returns; the context stays usable, and the next call
    without the hook matches the oracle."""
    r = I.scan_inputs(6, 1, 512, 64, 16, "bf16", with_h0=True)
    L.samba_debug_scan_stall(3, 5_000_000)
    try:
        import torch
        Bn, Ln, D = r["u"].shape
        u, dtt = dev(r["u"], "bf16"), dev(r["dt_raw"], "bf16")
        y = torch.empty_like(u)
        L.samba_selective_scan(u, dtt, dev(r["dt_bias"]), 1, dev(r["A_log"]), dev(r["B"], "bf16"),
                               dev(r["C"], "bf16"), dev(r["D"]), dev(r["z"], "bf16"), dev(r["h0"]), None, y,
                               Bn, Ln, D, 16, 1)
        assert L.samba_get_error() == L.SAMBA_ERR_TIMEOUT
    finally:
        L.samba_debug_scan_stall(-1)
    assert L.samba_get_error() == 0  # the word was cleared by the read
    y, hT = run_scan(L, r, "bf16", h0=r["h0"])
    yo, ho = oracle_scan(r, h0=r["h0"])
    assert rel_err(y, yo) <= TOL["bf16"]
    assert rel_err(hT, ho) <= TOL["bf16"]


@pytest.mark.parametrize("Bn,Ln,D,R", [(1, 4096, 4096, 128), (2, 300, 64, 128), (1, 129, 32, 64), (2, 65, 48, 16)])
def test_scan_xdbl_matches_oracle(L, Bn, Ln, D, R):
    """The scan with the dt projection folded in (samba_selective_scan_xdbl):
    Delta = softplus(dt_low W_dt^T + b) formed inside the kernel on tensor-core
    tiles from the x_proj output [dt_low | B | C], against the oracle's
    projection, softplus and scan in fp64 on the same (bf16) values."""
    import torch
    r = I.scan_inputs(7, Bn, Ln, D, 16, "bf16", with_h0=True)
    dt_low = I.draw_normal(7, "scan.dt_low", (Bn, Ln, R), 1.0, "bf16")
    W_dt = I.draw_normal(7, "scan.W_dt", (D, R), R ** -0.5, "bf16")
    x_dbl = np.concatenate([dt_low, r["B"], r["C"]], axis=-1)
    y = torch.empty(Bn, Ln, D, device="cuda", dtype=torch.bfloat16)
    hT = torch.empty(Bn, D, 16, device="cuda")
    L.samba_selective_scan_xdbl(dev(r["u"], "bf16"), dev(x_dbl, "bf16"), R, dev(W_dt, "bf16"), dev(r["dt_bias"]),
                                dev(r["A_log"]), dev(r["D"]), dev(r["z"], "bf16"), dev(r["h0"]), hT, y, Bn, Ln, D,
                                16, 1)
    torch.cuda.synchronize()
    assert L.samba_get_error() == 0
    delta = O.softplus(O.linear(dt_low.astype(np.float64), W_dt.astype(np.float64)) + r["dt_bias"])
    A = -np.exp(r["A_log"].astype(np.float64))
    yo, ho = O.selective_scan(r["u"], delta, A, r["B"], r["C"], r["D"], r["z"], r["h0"])
    assert rel_err(host(y), yo) <= TOL["bf16"]
    assert rel_err(host(hT), ho) <= TOL["bf16"]


def test_scan_xdbl_rejects_unsupported(L):
    """Outside the folded kernel's range the entry point refuses before any launch."""
    import torch
    from sliding_window_attention_samba_b200._lib import SambaError
    u = torch.zeros(1, 64, 64, device="cuda", dtype=torch.bfloat16)
    x = torch.zeros(1, 64, 176 + 32, device="cuda", dtype=torch.bfloat16)
    W = torch.zeros(64, 176, device="cuda", dtype=torch.bfloat16)
    A = torch.zeros(64, 16, device="cuda")
    y = torch.empty_like(u)
    with pytest.raises(SambaError) as e:  # dt_rank 176 > 128
        L.samba_selective_scan_xdbl(u, x, 176, W, None, A, None, None, None, None, y, 1, 64, 64, 16, 1)
    assert e.value.code == L.SAMBA_ERR_UNSUPPORTED
