"""samba_swa_fwd_noalloc: the attention entry point for callers that cannot
allocate device memory (its RoPE scratch lives in a fixed array inside the
library instead of a caller workspace).  Checked through the C ABI against the
workspace-taking samba_swa_fwd on two calls in a row; this file is collected
last so that a failure here never hides another test."""
import numpy as np
import pytest

from sliding_window_attention_samba_b200 import inputs as I
from tests.helpers import TOL, dev, host, rel_err

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def L():
    import torch
    from sliding_window_attention_samba_b200 import _lib
    torch.cuda.init()
    return _lib


def _pair(L_, dt, Bn, Ln, Hq, Hkv, d, w, base, pos0, seed):
    import torch
    r = I.swa_inputs(seed, Bn, Ln, Hq, Hkv, d, dt)
    q, k, v = dev(r["q"], dt), dev(r["k"], dt), dev(r["v"], dt)
    code = 1 if dt == "bf16" else 0
    o_ws = torch.empty_like(q)
    o_na = torch.full_like(q, float("nan"))
    n = L_.samba_swa_workspace_size(Bn, Ln, Hq, Hkv, d, base, code)
    ws = torch.empty(max(n, 1), dtype=torch.uint8, device="cuda")
    L_.samba_swa_fwd(q, k, v, o_ws, Bn, Ln, Hq, Hkv, d, w, base, pos0, 0.0, code, ws, n)
    L_.samba_swa_fwd_noalloc(q, k, v, o_na, Bn, Ln, Hq, Hkv, d, w, base, pos0, 0.0, code)
    torch.cuda.synchronize()
    assert L_.samba_get_error() == 0
    return host(o_na), host(o_ws)


@pytest.mark.parametrize("dt,Bn,Ln,Hq,Hkv,d,w,base,pos0", [
    ("bf16", 1, 1024, 32, 4, 64, 256, 10000.0, 0),
    ("f32", 2, 300, 4, 2, 16, 64, 10000.0, 12345),
    ("bf16", 1, 200, 8, 2, 64, 50, 0.0, 0),
    ("bf16", 1, 1500, 11, 1, 256, 2048, 10000.0, 7),  # head_dim 256: 11.9 MiB of scratch
])
def test_noalloc_matches_workspace_entry_two_calls(L, dt, Bn, Ln, Hq, Hkv, d, w, base, pos0):
    # two calls in a row with different inputs: the shared scratch keeps the first
    # call's contents, and the second call must not depend on them
    for seed in (11, 12):
        got, ref = _pair(L, dt, Bn, Ln, Hq, Hkv, d, w, base, pos0, seed)
        assert not np.isnan(got).any()
        assert rel_err(got, ref) <= TOL[dt]


def test_noalloc_back_to_back_calls_with_other_shapes(L):
    # consecutive calls with a different head_dim, table size, rope base and
    # position: each call rebuilds the table and the rotated copies it reads, so
    # none depends on what the previous call left in the shared scratch
    cases = [("bf16", 1, 600, 11, 1, 256, 512, 10000.0, 3, 21),
             ("bf16", 2, 333, 8, 2, 64, 100, 500000.0, 1000, 22),
             ("f32", 1, 257, 4, 2, 32, 64, 10000.0, 0, 23),
             ("bf16", 1, 600, 11, 1, 256, 512, 20000.0, 99, 24)]
    for dt, Bn, Ln, Hq, Hkv, d, w, base, pos0, seed in cases:
        got, ref = _pair(L, dt, Bn, Ln, Hq, Hkv, d, w, base, pos0, seed)
        assert not np.isnan(got).any()
        assert rel_err(got, ref) <= TOL[dt], (d, base)


def test_noalloc_rejects_sizes_beyond_the_fixed_scratch(L):
    import torch
    # bf16, 36 heads of 64: 4608 bytes of rotated q/k per token; 4096 tokens need 18 MiB > 16 MiB
    q = torch.empty(1, 4096, 32, 64, device="cuda", dtype=torch.bfloat16)
    k = torch.empty(1, 4096, 4, 64, device="cuda", dtype=torch.bfloat16)
    o = torch.empty_like(q)
    with pytest.raises(L.SambaError) as e:
        L.samba_swa_fwd_noalloc(q, k, k, o, 1, 4096, 32, 4, 64, 2048, 10000.0, 0, 0.0, 1)
    assert e.value.code == 2  # SAMBA_ERR_UNSUPPORTED
