"""Pins of the fp64 oracle against facts fixed independently of it: hand-worked
examples, closed forms, brute force, special cases and library routines.

Each test names the property and the passage it follows.  A plausible slip in
the oracle (a dropped term, a wrong sign or index, a transposed operand, an
off-by-one window edge) fails at least one of them."""
import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import samba_oracle as O
from sliding_window_attention_samba_b200 import inputs as I

GOLD = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "hand_examples.json")))
RNG = np.random.default_rng(1234)


def rnd(*shape, s=1.0):
    return RNG.standard_normal(shape) * s


# ---------------------------------------------------------------- generator
def test_splitmix64_published_first_output():
    # SplitMix64 seeded with 0: first output is 0xE220A8397B1DCDAF (published test vector).
    z = np.array([0x9E3779B97F4A7C15], dtype=np.uint64)
    assert int(I._mix_arr(z)[0]) == 0xE220A8397B1DCDAF


def test_torch_generator_matches_unsigned_definition():
    # The int64 torch form of the counter generator gives the same bits as the
    # unsigned SplitMix64 definition, at offsets past 2^32 too.
    key = I.tensor_key(5, "w")
    for start in (0, 7, (1 << 33) + 3):
        ctr = np.arange(start + 1, start + 65, dtype=np.uint64)
        with np.errstate(over="ignore"):
            z = np.uint64(key) + ctr * np.uint64(0x9E3779B97F4A7C15)
        ref = ((I._mix_arr(z) >> np.uint64(11)).astype(np.float64) + 1.0) * 2.0 ** -53
        assert np.array_equal(I.uniforms(key, start, 64), ref)
    a = I.normals(key, 100, start=0)
    b = I.normals(key, 60, start=40)
    assert np.array_equal(a[40:], b)  # element i depends only on its own counters


def test_bf16_rounding_ties_to_even():
    x = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -2.5, 1.0 + 2 ** -7], dtype=np.float32)
    bits = I.to_bf16_bits(x)
    assert list(bits) == [0x3F80, 0x3F80, 0x3F82, 0xC020, 0x3F81]


def test_normals_moments():
    v = I.normals(I.tensor_key(0, "x"), 200000)
    assert abs(v.mean()) < 0.01 and abs(v.std() - 1) < 0.01


def test_dt_bias_softplus_range_loguniform():
    # "Delta bias initialised so that Delta lies in [1e-3, 1e-1]" (Samba 3.4).
    b = I.dt_bias_init(0, "t", 20000)
    d = O.softplus(b)
    assert d.min() >= 1e-3 * (1 - 1e-6) and d.max() <= 1e-1 * (1 + 1e-6)
    q = (np.log(d) - np.log(1e-3)) / (np.log(1e-1) - np.log(1e-3))
    hist, _ = np.histogram(q, bins=10, range=(0, 1))
    assert hist.min() > 1700 and hist.max() < 2300


# ---------------------------------------------------------------- elementwise
def test_softplus_identities():
    x = rnd(1000, s=10)
    assert np.allclose(O.softplus(x) - O.softplus(-x), x, atol=1e-12)
    assert abs(O.softplus(0.0) - math.log(2)) < 1e-15
    assert abs(O.softplus(50.0) - 50.0) < 1e-15


def test_silu_special_values():
    assert O.silu(0.0) == 0.0
    assert abs(O.silu(40.0) - 40.0) < 1e-12 and abs(O.silu(-40.0)) < 1e-12
    x = rnd(100)
    assert np.allclose(O.silu(x) - O.silu(-x), x, atol=1e-12)  # x s(x) + x s(-x) ... = x


# ---------------------------------------------------------------- rmsnorm
def test_rmsnorm_hand_example():
    g = GOLD["rmsnorm_34"]
    out = O.rmsnorm(np.array(g["x"]), np.array(g["g"]), eps=0.0)
    assert np.allclose(out, g["out"], rtol=1e-14)


def test_rmsnorm_constant_closed_form():
    c, eps = 0.37, 1e-5
    out = O.rmsnorm(np.full((3, 8), c), np.full(8, 2.0), eps)
    assert np.allclose(out, 2.0 * c / math.sqrt(c * c + eps), rtol=1e-14)


# ---------------------------------------------------------------- linear / mlp
def test_linear_orientation_brute_force():
    x, W = rnd(2, 3), rnd(4, 3)
    ref = np.array([[sum(x[i, k] * W[j, k] for k in range(3)) for j in range(4)] for i in range(2)])
    assert np.allclose(O.linear(x, W), ref, rtol=1e-14)


def test_swiglu_brute_force_and_zero_gate():
    x, W1, W2, W3 = rnd(2, 3), rnd(5, 3), rnd(5, 3), rnd(3, 5)
    ref = np.zeros((2, 3))
    for i in range(2):
        hid = []
        for j in range(5):
            a = sum(x[i, k] * W1[j, k] for k in range(3))
            g = sum(x[i, k] * W2[j, k] for k in range(3))
            hid.append(a * g / (1 + math.exp(-g)))
        for m in range(3):
            ref[i, m] = sum(hid[j] * W3[m, j] for j in range(5))
    assert np.allclose(O.swiglu_mlp(x, W1, W2, W3), ref, rtol=1e-12)
    assert np.all(O.swiglu_mlp(x, W1, np.zeros_like(W2), W3) == 0)  # SiLU(0) = 0 gates all off


# ---------------------------------------------------------------- conv
def test_conv_hand_example_taps():
    g = GOLD["conv_taps"]
    x = np.array(g["x"])[None, :, None]
    w = np.array(g["w"])[None, :]
    out, st = O.causal_dwconv(x, w)
    assert np.array_equal(out[0, :, 0], np.array(g["out"]))
    assert np.array_equal(st[0, 0], x[0, -3:, 0])


def test_conv_constant_input_and_state_continuation():
    D, L = 5, 12
    w = rnd(D, 4)
    out, _ = O.causal_dwconv(np.ones((1, L, D)), w)
    for t in range(L):
        assert np.allclose(out[0, t], w[:, 3 - min(t, 3):].sum(axis=1), rtol=1e-14)
    x = rnd(2, L, D)
    full, st_full = O.causal_dwconv(x, w)
    a, st = O.causal_dwconv(x[:, :7], w)
    b, st2 = O.causal_dwconv(x[:, 7:], w, state=st)
    assert np.allclose(np.concatenate([a, b], 1), full, rtol=1e-14)
    assert np.array_equal(st2, st_full)


# ---------------------------------------------------------------- selective scan
def test_scan_hand_example():
    g = GOLD["scan_ln2"]
    u = np.array(g["u"])[None, :, None]
    delta = np.full_like(u, g["delta"])
    A = -np.exp(np.array([[g["A_log"]]]))
    one = np.ones((1, 3, 1))
    y, h = O.selective_scan(u, delta, A, one, one, np.array([g["D"]]))
    assert np.allclose(y[0, :, 0], g["y"], rtol=1e-14)
    assert abs(h[0, 0, 0] - g["h_final"]) < 1e-14


def _scan_materialised(u, delta, A, Bm, Cm, Dsk, z, h0):
    """y_t = sum_n C_tn [ exp(A_n sum_{r<=t} d_r) h0_n + sum_{s<=t} exp(A_n sum_{s<r<=t} d_r) d_s B_sn u_s ] + D u_t."""
    Bn, L, D = u.shape
    N = A.shape[1]
    y = np.zeros((Bn, L, D))
    for b in range(Bn):
        cs = np.cumsum(delta[b], axis=0)  # [L, D], cs[t] = sum_{r<=t}
        for t in range(L):
            for c in range(D):
                acc = 0.0
                for n in range(N):
                    if h0 is not None:
                        acc += Cm[b, t, n] * math.exp(A[c, n] * cs[t, c]) * h0[b, c, n]
                    for s in range(t + 1):
                        seg = cs[t, c] - cs[s, c]
                        acc += Cm[b, t, n] * math.exp(A[c, n] * seg) * delta[b, s, c] * Bm[b, s, n] * u[b, s, c]
                y[b, t, c] = acc + Dsk[c] * u[b, t, c]
    if z is not None:
        y = y * z / (1 + np.exp(-z))
    return y


def test_scan_equals_materialised_kernel_form():
    Bn, L, D, N = 2, 24, 3, 4
    u, Bm, Cm, z = rnd(Bn, L, D), rnd(Bn, L, N), rnd(Bn, L, N), rnd(Bn, L, D)
    delta = np.exp(RNG.uniform(np.log(1e-3), np.log(0.5), (Bn, L, D)))
    A = -np.exp(RNG.uniform(-1, 2, (D, N)))
    Dsk, h0 = rnd(D), rnd(Bn, D, N)
    y, _ = O.selective_scan(u, delta, A, Bm, Cm, Dsk, z, h0)
    ref = _scan_materialised(u, delta, A, Bm, Cm, Dsk, z, h0)
    assert np.allclose(y, ref, rtol=1e-11, atol=1e-12)


def test_scan_lti_closed_form():
    L, D, N = 50, 2, 16
    dlt, Bv, Cv, uv = 0.05, rnd(N), rnd(N), 0.7
    A = -np.tile(np.arange(1, N + 1, dtype=float), (D, 1))
    y, h = O.selective_scan(np.full((1, L, D), uv), np.full((1, L, D), dlt), A,
                            np.tile(Bv, (1, L, 1)), np.tile(Cv, (1, L, 1)), np.zeros(D))
    a = np.exp(dlt * A[0])
    for t in range(L):
        ht = dlt * Bv * uv * (1 - a ** (t + 1)) / (1 - a)
        assert np.allclose(y[0, t], ht @ Cv, rtol=1e-12)
    assert np.allclose(h[0, 0], dlt * Bv * uv * (1 - a ** L) / (1 - a), rtol=1e-12)


def test_scan_impulse_is_exactly_causal():
    L, D, N, s = 30, 4, 16, 17
    u = np.zeros((1, L, D)); u[0, s] = rnd(D)
    delta = np.exp(RNG.uniform(np.log(1e-3), np.log(1e-1), (1, L, D)))
    y, _ = O.selective_scan(u, delta, -np.exp(rnd(D, N)), rnd(1, L, N), rnd(1, L, N), np.ones(D), rnd(1, L, D))
    assert np.all(y[0, :s] == 0.0) and np.all(y[0, s] != 0.0)


def test_scan_chunk_split_invariance():
    Bn, L, D, N, L1 = 2, 40, 3, 16, 13
    args = [rnd(Bn, L, D), np.exp(RNG.uniform(-7, -1, (Bn, L, D))), -np.exp(rnd(D, N)),
            rnd(Bn, L, N), rnd(Bn, L, N)]
    Dsk, z = rnd(D), rnd(Bn, L, D)
    y, h = O.selective_scan(*args, Dsk, z)
    first = [a if a.ndim == 2 else a[:, :L1] for a in args]
    rest = [a if a.ndim == 2 else a[:, L1:] for a in args]
    y1, h1 = O.selective_scan(*first, Dsk, z[:, :L1])
    y2, h2 = O.selective_scan(*rest, Dsk, z[:, L1:], h0=h1)
    assert np.allclose(np.concatenate([y1, y2], 1), y, rtol=1e-12, atol=1e-14)
    assert np.allclose(h2, h, rtol=1e-12)


def test_scan_memoryless_and_zero_step_limits():
    Bn, L, D, N = 1, 10, 3, 16
    u, Bm, Cm, Dsk = rnd(Bn, L, D), rnd(Bn, L, N), rnd(Bn, L, N), rnd(D)
    delta = np.full((Bn, L, D), 0.3)
    y, _ = O.selective_scan(u, delta, np.full((D, N), -1e300), Bm, Cm, Dsk)
    ref = np.einsum("btn,btn->bt", Cm, Bm)[:, :, None] * 0.3 * u + Dsk * u
    assert np.allclose(y, ref, rtol=1e-13)
    y0, h0 = O.selective_scan(u, np.zeros_like(u), -np.ones((D, N)), Bm, Cm, Dsk)
    assert np.array_equal(y0, Dsk * u) and np.all(h0 == 0)


# ---------------------------------------------------------------- RoPE
def test_rope_hand_example_and_complex_form():
    g = GOLD["rope_unit"]
    out = O.rope(np.array(g["x"])[None, None, :], [g["pos"]], 10000.0)
    assert np.allclose(out[0, 0], g["out"], rtol=1e-15)
    L, H, d = 7, 3, 16
    x, pos = rnd(L, H, d), np.array([0, 1, 5, 100, 4095, 65536, 1048575])
    theta = 10000.0 ** (-np.arange(d // 2) * 2.0 / d)
    zc = (x[..., :d // 2] + 1j * x[..., d // 2:]) * np.exp(1j * pos[:, None, None] * theta)
    ref = np.concatenate([zc.real, zc.imag], axis=-1)
    assert np.allclose(O.rope(x, pos, 10000.0), ref, rtol=1e-12, atol=1e-12)


def test_rope_relative_position_property():
    d = 64
    q, k = rnd(1, 1, d), rnd(1, 1, d)
    for p, s, P in [(10, 3, 1000), (2047, 0, 123457), (5, 5, 999999)]:
        a = O.rope(q, [p], 1e4)[0, 0] @ O.rope(k, [s], 1e4)[0, 0]
        b = O.rope(q, [p + P], 1e4)[0, 0] @ O.rope(k, [s + P], 1e4)[0, 0]
        assert abs(a - b) < 1e-9


# ---------------------------------------------------------------- SWA
def _sdpa_band(q, k, v, window):
    """torch scaled_dot_product_attention (fp64) with the explicit band mask
    0 <= t - s < window and K/V heads expanded per group."""
    Bn, L, Hq, d = q.shape
    grp = Hq // k.shape[2]
    qt = torch.tensor(q).permute(0, 2, 1, 3)
    kt = torch.tensor(np.repeat(k, grp, 2)).permute(0, 2, 1, 3)
    vt = torch.tensor(np.repeat(v, grp, 2)).permute(0, 2, 1, 3)
    t = torch.arange(L)[:, None]
    s = torch.arange(L)[None, :]
    mask = (t - s >= 0) & (t - s < window)
    return torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=mask).permute(0, 2, 1, 3).numpy()


@pytest.mark.parametrize("window", [1, 3, 16, 37, 200])
def test_swa_equals_library_masked_attention(window):
    q, k, v = rnd(2, 37, 4, 8), rnd(2, 37, 2, 8), rnd(2, 37, 2, 8)
    assert np.allclose(O.swa(q, k, v, window), _sdpa_band(q, k, v, window), rtol=1e-10, atol=1e-12)
    # peaked softmax: window-edge errors are not hidden by a flat distribution
    assert np.allclose(O.swa(30 * q, k, v, window), _sdpa_band(30 * q, k, v, window), rtol=1e-9, atol=1e-11)


def test_swa_full_window_equals_causal_library():
    q, k, v = rnd(1, 20, 2, 8), rnd(1, 20, 1, 8), rnd(1, 20, 1, 8)
    qt = torch.tensor(q).permute(0, 2, 1, 3)
    kt = torch.tensor(np.repeat(k, 2, 2)).permute(0, 2, 1, 3)
    vt = torch.tensor(np.repeat(v, 2, 2)).permute(0, 2, 1, 3)
    ref = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, is_causal=True).permute(0, 2, 1, 3).numpy()
    assert np.allclose(O.swa(q, k, v, 20), ref, rtol=1e-10)
    assert np.allclose(O.swa(q, k, v, 1000), ref, rtol=1e-10)


def test_swa_window_one_returns_v_and_gqa_mapping():
    q, k, v = rnd(1, 9, 6, 4), rnd(1, 9, 3, 4), rnd(1, 9, 3, 4)
    o = O.swa(q, k, v, 1)
    for h in range(6):
        assert np.array_equal(o[:, :, h], v[:, :, h // 2])


def test_swa_uniform_scores_hand_example_and_band_mean():
    g = GOLD["swa_uniform"]
    L, w = g["L"], g["window"]
    v = np.arange(L, dtype=float)[None, :, None, None]
    o = O.swa(np.zeros((1, L, 1, 1)), np.zeros((1, L, 1, 1)), v, w)
    assert np.allclose(o[0, :, 0, 0], g["o"], rtol=1e-14)
    L, w = 300, 64
    v = np.arange(L, dtype=float)[None, :, None, None]
    o = O.swa(np.zeros((1, L, 1, 1)), rnd(1, L, 1, 1), v, w)
    assert np.allclose(o[0, :, 0, 0], [(max(0, t - w + 1) + t) / 2 for t in range(L)], rtol=1e-13)


def test_swa_perturbation_locality():
    L, w, s = 40, 8, 13
    q, k, v = rnd(1, L, 2, 4), rnd(1, L, 1, 4), rnd(1, L, 1, 4)
    o = O.swa(q, k, v, w)
    k2, v2 = k.copy(), v.copy()
    k2[0, s] += 1.0
    v2[0, s] -= 2.0
    o2 = O.swa(q, k2, v2, w)
    changed = np.any(o != o2, axis=(0, 2, 3))
    assert list(np.nonzero(changed)[0]) == list(range(s, s + w))


# ---------------------------------------------------------------- block / decode
def test_block_batch_rows_independent():
    cfg = I.TINY
    W = I.block_weights(cfg, 0)
    x = I.block_input(cfg, 0, 2, 20)
    both = O.block_fwd(x, W, cfg)["x_out"]
    one = O.block_fwd(x[1:2], W, cfg)["x_out"]
    assert np.array_equal(both[1:2], one)


def test_block_composition_of_branches():
    cfg = I.TINY
    W = I.block_weights(cfg, 0, conv_bias=True)
    x = I.block_input(cfg, 0, 1, 16)
    r = O.block_fwd(x, W, cfg)
    assert np.allclose(r["x_out"], x + sum(r["branch"]), rtol=1e-13)
    m = r["mamba"]
    assert np.allclose(m["delta"], O.softplus(m["dt_raw"] + W["dt_bias"]), rtol=1e-14)


@pytest.mark.parametrize("P,S", [(70, 6), (5, 3), (63, 4)])
def test_prefill_then_step_equals_longer_prefill(P, S):
    cfg = I.TINY  # window 64: P=70 wraps the ring, P=63 crosses the edge while stepping
    W = I.block_weights(cfg, 0, conv_bias=True)
    x = I.block_input(cfg, 0, 2, P + S)
    full = O.block_fwd(x, W, cfg, want_state=True)
    st = O.block_fwd(x[:, :P], W, cfg, want_state=True)["state"]
    for i in range(S):
        y, st, _ = O.block_step(x[:, P + i], W, cfg, st)
        assert np.allclose(y, full["x_out"][:, P + i], rtol=1e-11, atol=1e-11)
    for key in ("ssm", "conv", "k_ring", "v_ring"):
        assert np.allclose(st[key], full["state"][key], rtol=1e-10, atol=1e-12), key
    assert np.array_equal(st["pos"], full["state"]["pos"])


def test_ring_slot_map_bit_exact():
    cfg = I.TINY
    W = I.block_weights(cfg, 0)
    L = 3 * cfg.window + 5
    x = I.block_input(cfg, 0, 1, L)
    r = O.block_fwd(x, W, cfg, want_state=True)
    kr = r["attn"]["k"]
    for slot in range(cfg.window):
        # the newest position p < L with p mod w == slot
        p = L - 1 - ((L - 1 - slot) % cfg.window)
        assert np.array_equal(r["state"]["k_ring"][0, slot], kr[0, p])


# ---------------------------------------------------------------- language-model stack
def test_model_stack_composes_the_block():
    # [Mamba, MLP, SWA, MLP'] with MLP' carrying the block's second MLP is the block;
    # the embedding lookup is an identity when the table holds the inputs row by row.
    cfg = I.TINY
    W = I.block_weights(cfg, 5)
    x = I.block_input(cfg, 5, 1, 90)
    W2 = dict(W, norm1=W["norm3"], mlp1_W1=W["mlp2_W1"], mlp1_W2=W["mlp2_W2"], mlp1_W3=W["mlp2_W3"])
    g = RNG.standard_normal(cfg.d_model)
    head = RNG.standard_normal((11, cfg.d_model))
    ids = np.arange(90)[None]
    got = O.model_prefill(ids, [("mamba", W), ("mlp", W), ("swa", W), ("mlp", W2)], x[0], g, head, cfg)
    xo = O.block_fwd(x, W, cfg)["x_out"][:, -1]
    want = (xo / np.sqrt((xo ** 2).mean(-1, keepdims=True) + cfg.norm_eps) * g) @ head.T
    assert np.allclose(got, want, rtol=1e-12, atol=1e-12)


def test_model_without_layers_reads_the_last_token():
    # no layers, one-hot embeddings, identity head: logits are sqrt(d) at the last id
    cfg = I.TINY
    d = cfg.d_model
    ids = np.array([[3, 17, 5], [60, 2, 41]])
    logits = O.model_prefill(ids, [], np.eye(d), np.ones(d), np.eye(d), cfg)
    assert list(logits.argmax(1)) == [5, 41]
    assert np.allclose(logits.max(1), np.sqrt(d / (1 + d * cfg.norm_eps)), rtol=1e-12)
