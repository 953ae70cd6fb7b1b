"""Plain fp64 CPU oracle of the Samba block (test infrastructure only).

This module is test infrastructure.  Only the tests, the smoke check and the
benchmark's CPU-baseline leg may import it; the CUDA path never does, and it
imports nothing from the CUDA path.

Every function is the direct, sequential definition of one step of the layer as
the page "Samba: Simple Hybrid State Space Models for Efficient Unlimited Context
Language Modeling" (a long-form summary of arXiv 2406.07522) states it in §3.2
"Big-Picture Architecture" and §3.4 "Detailed, Sentence-Based Technical
Breakdown".  Cited below as [Samba §3.4, <sub-heading>].  Library primitives
used as steps: numpy matmul / einsum (dot products), exp, log1p.

Inputs arrive already rounded to their storage dtype (fp32 arrays holding bf16 or
fp32 values); everything is then computed in fp64 with no intermediate rounding.

Readings of points the pages leave open (each also listed in the design notes):
  * window edge: a query at t sees keys s with t - w < s <= t (w keys, itself
    included), the band of the blog page's mask 0 <= i - j < w;
  * RMSNorm eps = 1e-5 with a per-channel gain; softmax scale 1/sqrt(head_dim);
  * RoPE: rotate-half pairing (i, i + d/2), theta_i = base^(-2i/d), absolute
    0-based positions, keys cached after rotation;
  * GQA: query head h reads kv head floor(h / (Hq / Hkv));
  * conv taps: u_t = sum_j w[c, j] x_{t-(k-1)+j}, zero history before t = 0;
  * the Mamba gate reads the normed block input: z = X W_g;
  * block order Mamba -> MLP -> SWA -> MLP, each pre-RMSNorm with a residual.

Parity pins: every function here is checked by the "not gpu" tests against
closed forms, brute force, special cases or a hand-worked example; none is
"parity unpinned".
"""
from __future__ import annotations

import math
from typing import Dict, Optional, Tuple

import numpy as np

F64 = np.float64


def _f(x):
    return None if x is None else np.asarray(x, dtype=F64)


# --------------------------------------------------------------------------
# Elementwise functions
# --------------------------------------------------------------------------
def softplus(x):
    """Softplus(x) = log(1 + e^x) [Samba §3.4, "Input-Dependent Selective Gating"],
    evaluated without overflow as max(x, 0) + log1p(exp(-|x|))."""
    x = _f(x)
    return np.maximum(x, 0.0) + np.log1p(np.exp(-np.abs(x)))


def sigmoid(x):
    x = _f(x)
    return 0.5 * (1.0 + np.tanh(0.5 * x))


def silu(x):
    """SiLU(x) = x * sigma(x) [Samba §3.4, "Input Projection and Short Convolution"]."""
    x = _f(x)
    return x * sigmoid(x)


# --------------------------------------------------------------------------
# Dense pieces
# --------------------------------------------------------------------------
def rmsnorm(x, g, eps: float = 1e-5):
    """Pre-norm applied before every Mamba / SWA / MLP layer [Samba §3.2]:
    x / sqrt(mean(x^2) + eps) * g over the last axis."""
    x = _f(x)
    ms = np.mean(x * x, axis=-1, keepdims=True)
    return x / np.sqrt(ms + eps) * _f(g)


def linear(x, W):
    """x W^T for a weight stored [out_features, in_features] (the pages write the
    same map as X W with W in R^{in x out})."""
    return np.matmul(_f(x), _f(W).T)


def swiglu_mlp(x, W1, W2, W3):
    """SwiGLU(x) = ((x W1) * SiLU(x W2)) W3 [Samba §3.4, "SwiGLU Formulation"]."""
    return linear(linear(x, W1) * silu(linear(x, W2)), W3)


# --------------------------------------------------------------------------
# Mamba pieces
# --------------------------------------------------------------------------
def causal_dwconv(x, w, b=None, state=None):
    """Depthwise causal conv along time, no SiLU [Samba §3.4, "Input Projection and
    Short Convolution", eq. U = SiLU(DepthwiseConv(H, W_conv))].

    x: [B, L, D]; w: [D, k]; b: [D] or None; state: [B, D, k-1] holding the k-1
    inputs before t = 0 (oldest first) or None for zeros.
    out[b, t, c] = sum_{j=0}^{k-1} w[c, j] * x[b, t-(k-1)+j, c] (+ b[c]).
    Returns (out, new_state) where new_state holds the last k-1 inputs."""
    x = _f(x)
    w = _f(w)
    Bn, L, D = x.shape
    k = w.shape[1]
    hist = np.zeros((Bn, k - 1, D)) if state is None else np.transpose(_f(state), (0, 2, 1))
    xp = np.concatenate([hist, x], axis=1)  # [B, k-1+L, D]
    out = np.zeros((Bn, L, D))
    for t in range(L):
        for j in range(k):
            out[:, t, :] += w[:, j] * xp[:, t + j, :]
    if b is not None:
        out += _f(b)
    new_state = np.transpose(xp[:, L:, :], (0, 2, 1)).copy()  # last k-1 inputs
    return out, new_state


def selective_scan(u, delta, A, Bm, Cm, Dskip=None, z=None, h0=None):
    """The S6 recurrence, run sequentially over t [Samba §3.4, "The State Space
    Model Update (S6)"]:

        Z_t = exp(Delta_t * A) (.) Z_{t-1} + Delta_t (.) (B_t (x) U_t)
        Y_t = Z_t C_t + D (.) U_t

    with A = -exp(A_log) already applied by the caller (the page writes the decay
    as exp(-Delta (.) exp(A)) with its A being our A_log), Z_0 = h0 (zeros by
    default), and then the gate of "Gated Output": Y (.) SiLU(z) when z is given.

    u, delta, z: [B, L, D]; A: [D, N]; Bm, Cm: [B, L, N]; Dskip: [D]; h0: [B, D, N].
    Returns (y [B, L, D], h_L [B, D, N])."""
    u, delta, A, Bm, Cm = _f(u), _f(delta), _f(A), _f(Bm), _f(Cm)
    Bn, L, D = u.shape
    N = A.shape[1]
    h = np.zeros((Bn, D, N)) if h0 is None else _f(h0).copy()
    y = np.zeros((Bn, L, D))
    for t in range(L):
        dA = np.exp(delta[:, t, :, None] * A[None, :, :])                   # [B, D, N]
        dBu = (delta[:, t, :] * u[:, t, :])[:, :, None] * Bm[:, t, None, :]  # [B, D, N]
        h = dA * h + dBu
        y[:, t, :] = np.einsum("bdn,bn->bd", h, Cm[:, t, :])
    if Dskip is not None:
        y += u * _f(Dskip)
    if z is not None:
        y = y * silu(z)
    return y, h


# --------------------------------------------------------------------------
# Attention pieces
# --------------------------------------------------------------------------
def rope(x, positions, base: float):
    """Rotary position embedding [Samba §3.4, "Positional Encoding"], rotate-half
    pairing: for i < d/2, with a = pos * base^(-2i/d),
      out[i]       = x[i] cos a - x[i + d/2] sin a
      out[i + d/2] = x[i + d/2] cos a + x[i] sin a.
    x: [..., L, H, d]; positions: [L] integers.  base = 0 means no rotation."""
    x = _f(x)
    if base == 0:
        return x.copy()
    d = x.shape[-1]
    half = d // 2
    i = np.arange(half, dtype=F64)
    theta = base ** (-2.0 * i / d)
    ang = np.asarray(positions, dtype=F64)[:, None] * theta[None, :]  # [L, half]
    c = np.cos(ang)[:, None, :]
    s = np.sin(ang)[:, None, :]
    x1, x2 = x[..., :half], x[..., half:]
    return np.concatenate([x1 * c - x2 * s, x2 * c + x1 * s], axis=-1)


def swa(q, k, v, window: int, scale: Optional[float] = None):
    """Causal sliding-window attention with grouped-query heads [Samba §3.4,
    "Window Specification"; §3.2 (SWA layers); GQA per the model-size table]:

        o_{t,h} = sum_{s=max(0, t-w+1)}^{t} softmax_s(q_{t,h} . k_{s,g(h)} * scale) v_{s,g(h)}

    by brute force, one query row at a time.  q: [B, L, Hq, d]; k, v: [B, L, Hkv, d]
    (already rotated).  g(h) = floor(h / (Hq / Hkv))."""
    q, k, v = _f(q), _f(k), _f(v)
    Bn, L, Hq, d = q.shape
    Hkv = k.shape[2]
    grp = Hq // Hkv
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    kk = np.repeat(k, grp, axis=2)  # [B, L, Hq, d]
    vv = np.repeat(v, grp, axis=2)
    o = np.zeros_like(q)
    for t in range(L):
        s0 = max(0, t - window + 1)
        sc = np.einsum("bhd,bshd->bhs", q[:, t], kk[:, s0:t + 1]) * scale
        sc -= sc.max(axis=-1, keepdims=True)
        p = np.exp(sc)
        p /= p.sum(axis=-1, keepdims=True)
        o[:, t] = np.einsum("bhs,bshd->bhd", p, vv[:, s0:t + 1])
    return o


# --------------------------------------------------------------------------
# Layers and the block
# --------------------------------------------------------------------------
def mamba_branch(xn, W, cfg, state=None):
    """Mamba layer on the normed input xn [B, L, d_model] [Samba §3.4, "The Mamba
    Layer"]: H = X W_in; U = SiLU(conv(H)); Delta = Softplus(U W_r W_q + b);
    B = U W_b; C = U W_c; S6 scan; O = (Y (.) SiLU(X W_g)) W_out.
    state: None or dict(ssm [B,D,N], conv [B,D,k-1]).  Returns (O, new_state, extras)."""
    d_inner, N, R = cfg.d_inner, cfg.d_state, cfg.dt_rank
    hz = linear(xn, W["W_in"])
    H, zg = hz[..., :d_inner], hz[..., d_inner:]
    pre, conv_state = causal_dwconv(H, W["conv_w"], W.get("conv_b"), None if state is None else state["conv"])
    U = silu(pre)
    xdbl = linear(U, W["W_x"])
    dt_low, Bm, Cm = xdbl[..., :R], xdbl[..., R:R + N], xdbl[..., R + N:R + 2 * N]
    dt_raw = linear(dt_low, W["W_dt"])
    delta = softplus(dt_raw + _f(W["dt_bias"]))
    A = -np.exp(_f(W["A_log"]))
    y, hT = selective_scan(U, delta, A, Bm, Cm, W["D"], zg, None if state is None else state["ssm"])
    out = linear(y, W["W_out"])
    extras = dict(H=H, z=zg, u=U, dt_raw=dt_raw, delta=delta, B=Bm, C=Cm, y=y)
    return out, dict(ssm=hT, conv=conv_state), extras


def attn_branch(xn, W, cfg, pos0: int = 0):
    """SWA layer on the normed input [Samba §3.4, "The Sliding Window Attention
    (SWA) Layer"]: q, k, v projections, RoPE at absolute positions pos0 + t,
    windowed GQA softmax attention, output projection.  Returns (out, k_rot, v, extras)."""
    Bn, L, _ = xn.shape
    hd = cfg.head_dim
    q = linear(xn, W["Wq"]).reshape(Bn, L, cfg.n_q, hd)
    k = linear(xn, W["Wk"]).reshape(Bn, L, cfg.n_kv, hd)
    v = linear(xn, W["Wv"]).reshape(Bn, L, cfg.n_kv, hd)
    pos = np.arange(pos0, pos0 + L)
    qr, kr = rope(q, pos, cfg.rope_base), rope(k, pos, cfg.rope_base)
    o = swa(qr, kr, v, cfg.window)
    out = linear(o.reshape(Bn, L, cfg.n_q * hd), W["Wo"])
    return out, kr, v, dict(q=qr, k=kr, v=v, o=o)


def block_fwd(x, W, cfg, want_state: bool = False):
    """One Samba block as the workloads define it: Mamba -> MLP -> SWA -> MLP,
    each y = x + f(RMSNorm(x)) [Samba §3.2, "Big-Picture Architecture"].

    Returns dict with x_out, the four branch outputs f(...) (before each residual
    add), the residual stream after each sub-layer, intermediates and, when
    want_state, the decode state after the last token (ring slot = pos mod w)."""
    x0 = _f(x)
    eps = cfg.norm_eps
    f0, mstate, mx = mamba_branch(rmsnorm(x0, W["norm0"], eps), W, cfg)
    x1 = x0 + f0
    f1 = swiglu_mlp(rmsnorm(x1, W["norm1"], eps), W["mlp1_W1"], W["mlp1_W2"], W["mlp1_W3"])
    x2 = x1 + f1
    f2, kr, v, ax = attn_branch(rmsnorm(x2, W["norm2"], eps), W, cfg, 0)
    x3 = x2 + f2
    f3 = swiglu_mlp(rmsnorm(x3, W["norm3"], eps), W["mlp2_W1"], W["mlp2_W2"], W["mlp2_W3"])
    x4 = x3 + f3
    r = dict(x_out=x4, branch=[f0, f1, f2, f3], resid=[x1, x2, x3, x4], mamba=mx, attn=ax)
    if want_state:
        Bn, L = x0.shape[:2]
        w = cfg.window
        k_ring = np.zeros((Bn, w, cfg.n_kv, cfg.head_dim))
        v_ring = np.zeros_like(k_ring)
        for p in range(max(0, L - w), L):
            k_ring[:, p % w] = kr[:, p]
            v_ring[:, p % w] = v[:, p]
        r["state"] = dict(ssm=mstate["ssm"], conv=mstate["conv"], k_ring=k_ring, v_ring=v_ring,
                          pos=np.full(Bn, L, dtype=np.int64))
    return r


def model_prefill(ids, layers, embedding, final_norm, lm_head, cfg):
    """Language-model stack [Samba §3.2 "Big-Picture Architecture": token
    embeddings enter the first layer; each intermediate layer (Mamba, SWA or MLP)
    is preceded by RMSNorm and followed by a residual add; the last layer's output
    is projected to vocabulary logits].  A final RMSNorm (gain final_norm) comes
    before the projection (the pages do not print one; the reading of a pre-norm
    stack).  layers: list of (kind, W), kind in {"mamba", "mlp", "swa"}; an MLP
    layer reads norm1 and mlp1_W1..W3, Mamba norm0, SWA norm2.
    ids: int [B, L].  Returns the logits of the last position, [B, vocab]."""
    x = _f(embedding)[np.asarray(ids)]
    eps = cfg.norm_eps
    for kind, W in layers:
        if kind == "mamba":
            f = mamba_branch(rmsnorm(x, W["norm0"], eps), W, cfg)[0]
        elif kind == "mlp":
            f = swiglu_mlp(rmsnorm(x, W["norm1"], eps), W["mlp1_W1"], W["mlp1_W2"], W["mlp1_W3"])
        elif kind == "swa":
            f = attn_branch(rmsnorm(x, W["norm2"], eps), W, cfg, 0)[0]
        else:
            raise ValueError(kind)
        x = x + f
    return linear(rmsnorm(x[:, -1], final_norm, eps), lm_head)


def empty_state(cfg, batch: int):
    return dict(ssm=np.zeros((batch, cfg.d_inner, cfg.d_state)),
                conv=np.zeros((batch, cfg.d_inner, cfg.d_conv - 1)),
                k_ring=np.zeros((batch, cfg.window, cfg.n_kv, cfg.head_dim)),
                v_ring=np.zeros((batch, cfg.window, cfg.n_kv, cfg.head_dim)),
                pos=np.zeros(batch, dtype=np.int64))


def block_step(x_t, W, cfg, state):
    """One decode step of the block for one new token per sequence: the same
    layer equations for a single t, with the recurrent SSM state, the last k-1
    conv inputs and a window-sized ring KV cache (slot = position mod w).

    x_t: [B, d_model]; state as from block_fwd(..., want_state=True) (modified
    copy returned).  Returns (y_t, new_state, branches)."""
    st = {k: np.array(v, copy=True) for k, v in state.items()}
    x0 = _f(x_t)
    Bn = x0.shape[0]
    eps = cfg.norm_eps
    d_inner, N, R, k = cfg.d_inner, cfg.d_state, cfg.dt_rank, cfg.d_conv
    # --- Mamba, one time step
    xn = rmsnorm(x0, W["norm0"], eps)
    hz = linear(xn, W["W_in"])
    H, zg = hz[:, :d_inner], hz[:, d_inner:]
    window = np.concatenate([st["conv"], H[:, :, None]], axis=2)  # [B, D, k], oldest first
    pre = np.einsum("bdj,dj->bd", window, _f(W["conv_w"]))
    if W.get("conv_b") is not None:
        pre = pre + _f(W["conv_b"])
    st["conv"] = window[:, :, 1:]
    U = silu(pre)
    xdbl = linear(U, W["W_x"])
    dt_low, Bm, Cm = xdbl[:, :R], xdbl[:, R:R + N], xdbl[:, R + N:R + 2 * N]
    delta = softplus(linear(dt_low, W["W_dt"]) + _f(W["dt_bias"]))
    A = -np.exp(_f(W["A_log"]))
    h = np.exp(delta[:, :, None] * A[None]) * st["ssm"] + (delta * U)[:, :, None] * Bm[:, None, :]
    st["ssm"] = h
    y = np.einsum("bdn,bn->bd", h, Cm) + U * _f(W["D"])
    y = y * silu(zg)
    f0 = linear(y, W["W_out"])
    x1 = x0 + f0
    # --- MLP 1
    f1 = swiglu_mlp(rmsnorm(x1, W["norm1"], eps), W["mlp1_W1"], W["mlp1_W2"], W["mlp1_W3"])
    x2 = x1 + f1
    # --- SWA over the ring
    xn = rmsnorm(x2, W["norm2"], eps)
    hd, w = cfg.head_dim, cfg.window
    grp = cfg.n_q // cfg.n_kv
    scale = 1.0 / math.sqrt(hd)
    o = np.zeros((Bn, cfg.n_q, hd))
    for b in range(Bn):
        P = int(st["pos"][b])
        q = rope(linear(xn[b:b + 1], W["Wq"]).reshape(1, cfg.n_q, hd)[None], [P], cfg.rope_base)[0, 0]
        kk = rope(linear(xn[b:b + 1], W["Wk"]).reshape(1, cfg.n_kv, hd)[None], [P], cfg.rope_base)[0, 0]
        vv = linear(xn[b:b + 1], W["Wv"]).reshape(cfg.n_kv, hd)
        st["k_ring"][b, P % w] = kk
        st["v_ring"][b, P % w] = vv
        lo = max(0, P - w + 1)
        slots = [p % w for p in range(lo, P + 1)]
        for hq in range(cfg.n_q):
            g = hq // grp
            sc = st["k_ring"][b, slots, g] @ q[hq] * scale
            sc = np.exp(sc - sc.max())
            sc /= sc.sum()
            o[b, hq] = sc @ st["v_ring"][b, slots, g]
    f2 = linear(o.reshape(Bn, cfg.n_q * hd), W["Wo"])
    x3 = x2 + f2
    # --- MLP 2
    f3 = swiglu_mlp(rmsnorm(x3, W["norm3"], eps), W["mlp2_W1"], W["mlp2_W2"], W["mlp2_W3"])
    x4 = x3 + f3
    st["pos"] = st["pos"] + 1
    return x4, st, [f0, f1, f2, f3]
