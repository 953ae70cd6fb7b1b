"""Seeded synthetic inputs shared by the CUDA path's tests/bench and the CPU oracle.

This module holds no arithmetic of the Samba layer itself: it only draws random
numbers and lays them out.  Both sides receive the very same arrays.

Generator (counter based, so any slice of any tensor can be drawn on its own):

* SplitMix64 (Steele, Lea & Flood, "Fast splittable pseudorandom number
  generators", OOPSLA 2014): ``z = state + k*0x9E3779B97F4A7C15`` followed by the
  published finaliser (xor-shift 30 / mul 0xBF58476D1CE4E5B9 / xor-shift 27 /
  mul 0x94D049BB133111EB / xor-shift 31).
* Each tensor gets its own key: ``key = mix(seed * 0x9E3779B97F4A7C15 ^ fnv1a64(name))``.
* Element i of a normal tensor uses counters 2i+1 and 2i+2 for two uniforms
  ``u = ((x >> 11) + 1) * 2**-53`` in (0, 1] and Box-Muller's cosine branch
  ``sqrt(-2 ln u1) * cos(2 pi u2)`` (Box & Muller 1958), in fp64, evaluated with
  multi-threaded torch CPU ops so that full-size tensors take seconds.
* The fp64 value is scaled, rounded to fp32 (round to nearest even) and, for
  bf16 tensors, rounded again from fp32 to bf16 (round to nearest even).

Shapes, value distributions and initialisation follow the Samba paper summary
(arXiv 2406.07522, "3.4 Detailed Technical Breakdown": A initialised S4D-Real so
that exp(A_log) = 1..16, D = 1, the Delta bias initialised so that the step size
lies in [1e-3, 1e-1]) and the five workloads this repository measures.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, Iterable, Optional, Tuple

import numpy as np

_GAMMA = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)
_MASK64 = (1 << 64) - 1


def _mix_int(z: int) -> int:
    z &= _MASK64
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & _MASK64
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & _MASK64
    return z ^ (z >> 31)


def _fnv1a64(s: str) -> int:
    h = 0xCBF29CE484222325
    for b in s.encode():
        h ^= b
        h = (h * 0x100000001B3) & _MASK64
    return h


def tensor_key(seed: int, name: str) -> int:
    return _mix_int(((seed * 0x9E3779B97F4A7C15) & _MASK64) ^ _fnv1a64(name))


def _mix_arr(z: np.ndarray) -> np.ndarray:
    """SplitMix64 finaliser on uint64 numpy arrays (reference form, small inputs)."""
    with np.errstate(over="ignore"):
        z = (z ^ (z >> np.uint64(30))) * _M1
        z = (z ^ (z >> np.uint64(27))) * _M2
        return z ^ (z >> np.uint64(31))


def _s64(c: int) -> int:
    """An unsigned 64-bit constant as the int64 with the same bits."""
    return c - (1 << 64) if c >= (1 << 63) else c


def _lsr(z, k: int):
    """Logical right shift of int64 tensors (torch shifts are arithmetic)."""
    return (z >> k) & ((1 << (64 - k)) - 1)


def _mix_t(z):
    """SplitMix64 finaliser on int64 torch tensors (wrapping 64-bit arithmetic,
    identical bits to the unsigned definition)."""
    z = (z ^ _lsr(z, 30)) * _s64(0xBF58476D1CE4E5B9)
    z = (z ^ _lsr(z, 27)) * _s64(0x94D049BB133111EB)
    return z ^ _lsr(z, 31)


def uniforms(key: int, start: int, count: int) -> np.ndarray:
    """Uniforms in (0, 1] for counters start+1 .. start+count (fp64)."""
    import torch
    ctr = torch.arange(start + 1, start + count + 1, dtype=torch.int64)
    z = _s64(key) + ctr * _s64(0x9E3779B97F4A7C15)
    x = _mix_t(z)
    return ((_lsr(x, 11).to(torch.float64) + 1.0) * (2.0 ** -53)).numpy()


def normals(key: int, count: int, start: int = 0, chunk: int = 1 << 24) -> np.ndarray:
    """Standard normals (fp64) for elements start .. start+count-1 of a tensor:
    element i uses counters 2i+1, 2i+2 and Box-Muller's cosine branch.  Runs on
    the host cores (torch CPU ops, multi-threaded)."""
    import torch
    out = np.empty(count, dtype=np.float64)
    two_pi = 2.0 * np.pi
    for off in range(0, count, chunk):
        n = min(chunk, count - off)
        ctr = torch.arange(2 * (start + off) + 1, 2 * (start + off + n) + 1, dtype=torch.int64)
        x = _mix_t(_s64(key) + ctr * _s64(0x9E3779B97F4A7C15))
        u = (_lsr(x, 11).to(torch.float64) + 1.0) * (2.0 ** -53)
        u1, u2 = u[0::2], u[1::2]
        out[off:off + n] = (torch.sqrt(-2.0 * torch.log(u1)) * torch.cos(two_pi * u2)).numpy()
    return out


def to_bf16_bits(x32: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 (round to nearest even), returned as uint16 bit patterns."""
    b = np.ascontiguousarray(x32, dtype=np.float32).view(np.uint32)
    nan = (b & 0x7F800000) == 0x7F800000
    rounded = (b + np.uint32(0x7FFF) + ((b >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)
    rounded = np.where(nan & ((b & 0x007FFFFF) != 0), (b >> np.uint32(16)) | np.uint32(0x40), rounded)
    return rounded.astype(np.uint16)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << np.uint32(16)).view(np.float32)


def round_to(x: np.ndarray, dtype: str) -> np.ndarray:
    """Round fp64 values to the storage dtype and return them as fp32 arrays
    (bf16 values are exactly representable in fp32).  fp64 -> fp32 and fp32 ->
    bf16 both round to nearest even."""
    import torch
    x32 = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float64)).to(torch.float32)
    if dtype == "f32":
        return x32.numpy()
    if dtype == "bf16":
        return x32.to(torch.bfloat16).to(torch.float32).numpy()
    raise ValueError(dtype)


def draw_normal(seed: int, name: str, shape: Tuple[int, ...], std: float, dtype: str) -> np.ndarray:
    n = int(np.prod(shape)) if len(shape) else 1
    v = normals(tensor_key(seed, name), n) * std
    return round_to(v, dtype).reshape(shape)


def draw_uniform(seed: int, name: str, shape: Tuple[int, ...]) -> np.ndarray:
    n = int(np.prod(shape))
    return uniforms(tensor_key(seed, name), 0, n).reshape(shape)


# ----------------------------------------------------------------------------
# Workload shapes
# ----------------------------------------------------------------------------
@dataclasses.dataclass(frozen=True)
class BlockShape:
    d_model: int
    d_inner: int
    d_state: int
    d_conv: int
    dt_rank: int
    n_q: int
    n_kv: int
    head_dim: int
    window: int
    d_ff: int
    rope_base: float = 10000.0
    norm_eps: float = 1e-5
    dtype: str = "bf16"


TINY = BlockShape(d_model=64, d_inner=128, d_state=16, d_conv=4, dt_rank=4, n_q=4, n_kv=2,
                  head_dim=16, window=64, d_ff=256, dtype="f32")
WIDE = BlockShape(d_model=2048, d_inner=4096, d_state=16, d_conv=4, dt_rank=128, n_q=32, n_kv=4,
                  head_dim=64, window=2048, d_ff=8192, dtype="bf16")

# the 3.8B model's widths (d_model 2816, MLP 9984, 11 query heads over 1 kv
# head, hence head_dim 256; d_inner = 2 d_model, dt_rank = d_model / 16)
WIDE38 = BlockShape(d_model=2816, d_inner=5632, d_state=16, d_conv=4, dt_rank=176, n_q=11, n_kv=1,
                    head_dim=256, window=2048, d_ff=9984, dtype="bf16")

# name -> (shape, batch, seq_len, n_blocks, seed)
WORKLOADS = {
    "tiny_f32_L256": (TINY, 1, 256, 1, 0),
    "block_bf16_B4_L4096": (WIDE, 4, 4096, 1, 1),
    "prefill_bf16_L131072_x4": (WIDE, 1, 131072, 4, 2),
    "decode_bf16_B32": (WIDE, 32, 4096, 1, 4),
    "chunked_prefill_bf16_L1048576": (WIDE, 1, 1048576, 1, 5),
    "block38_bf16_L131072": (WIDE38, 1, 131072, 1, 6),
}
# chunk length of the chunked prefill (the blog page's "Chunked Prefilling for
# 1M-Token Sequences": chunks of 32,768 tokens)
CHUNKED_PREFILL_CHUNK = 32768
MIXER_SWEEP_L = (4096, 16384, 65536, 262144, 1048576)
MIXER_SWEEP_SEED = 3

DELTA_MIN, DELTA_MAX = 1e-3, 1e-1


def dt_bias_init(seed: int, name: str, d_inner: int) -> np.ndarray:
    """Bias b with softplus(b) = Delta0, Delta0 log-uniform in [1e-3, 1e-1].

    The inverse of softplus(x) = log(1 + e^x) is b = Delta0 + log(-expm1(-Delta0)),
    evaluated in fp64 and stored as fp32."""
    u = draw_uniform(seed, name + ".u", (d_inner,))
    d0 = np.exp(np.log(DELTA_MIN) + u * (np.log(DELTA_MAX) - np.log(DELTA_MIN)))
    return (d0 + np.log(-np.expm1(-d0))).astype(np.float32)


def a_log_init(d_inner: int, d_state: int) -> np.ndarray:
    """S4D-Real: A_log[d, n] = log(n + 1), so A = -exp(A_log) = -(n + 1)."""
    return np.tile(np.log(np.arange(1, d_state + 1, dtype=np.float64)), (d_inner, 1)).astype(np.float32)


def block_weights(shape: BlockShape, seed: int, layer: int = 0, conv_bias: bool = False) -> Dict[str, np.ndarray]:
    """Random-init weights of one block (Mamba, MLP, SWA, MLP).

    Matrices are stored [out_features, in_features] row-major in the block dtype;
    per-channel vectors (norm gains, conv taps, dt bias, A_log, D) are fp32."""
    s = shape
    dt = s.dtype
    p = f"L{layer}."
    std = 0.02
    w: Dict[str, np.ndarray] = {}
    for i in range(4):
        w[f"norm{i}"] = np.ones(s.d_model, dtype=np.float32)
    w["W_in"] = draw_normal(seed, p + "W_in", (2 * s.d_inner, s.d_model), std, dt)
    w["conv_w"] = draw_normal(seed, p + "conv_w", (s.d_inner, s.d_conv), std, "f32")
    w["conv_b"] = draw_normal(seed, p + "conv_b", (s.d_inner,), std, "f32") if conv_bias else None
    w["W_x"] = draw_normal(seed, p + "W_x", (s.dt_rank + 2 * s.d_state, s.d_inner), std, dt)
    w["W_dt"] = draw_normal(seed, p + "W_dt", (s.d_inner, s.dt_rank), std, dt)
    w["dt_bias"] = dt_bias_init(seed, p + "dt_bias", s.d_inner)
    w["A_log"] = a_log_init(s.d_inner, s.d_state)
    w["D"] = np.ones(s.d_inner, dtype=np.float32)
    w["W_out"] = draw_normal(seed, p + "W_out", (s.d_model, s.d_inner), std, dt)
    w["Wq"] = draw_normal(seed, p + "Wq", (s.n_q * s.head_dim, s.d_model), std, dt)
    w["Wk"] = draw_normal(seed, p + "Wk", (s.n_kv * s.head_dim, s.d_model), std, dt)
    w["Wv"] = draw_normal(seed, p + "Wv", (s.n_kv * s.head_dim, s.d_model), std, dt)
    w["Wo"] = draw_normal(seed, p + "Wo", (s.d_model, s.n_q * s.head_dim), std, dt)
    for m in (1, 2):
        w[f"mlp{m}_W1"] = draw_normal(seed, p + f"mlp{m}_W1", (s.d_ff, s.d_model), std, dt)
        w[f"mlp{m}_W2"] = draw_normal(seed, p + f"mlp{m}_W2", (s.d_ff, s.d_model), std, dt)
        w[f"mlp{m}_W3"] = draw_normal(seed, p + f"mlp{m}_W3", (s.d_model, s.d_ff), std, dt)
    return w


def block_input(shape: BlockShape, seed: int, batch: int, seq_len: int, name: str = "x") -> np.ndarray:
    return draw_normal(seed, name, (batch, seq_len, shape.d_model), 1.0, shape.dtype)


def scan_inputs(seed: int, batch: int, seq_len: int, d_inner: int, d_state: int, dtype: str,
                with_z: bool = True, with_h0: bool = False) -> Dict[str, np.ndarray]:
    """Mixer-only selective-scan inputs: u, dt_raw, B, C, z ~ N(0,1); dt bias and
    A_log per the block initialisation; D = 1; optional h0 ~ N(0,1) (fp32)."""
    r: Dict[str, np.ndarray] = {}
    r["u"] = draw_normal(seed, "scan.u", (batch, seq_len, d_inner), 1.0, dtype)
    r["dt_raw"] = draw_normal(seed, "scan.dt", (batch, seq_len, d_inner), 1.0, dtype)
    r["B"] = draw_normal(seed, "scan.B", (batch, seq_len, d_state), 1.0, dtype)
    r["C"] = draw_normal(seed, "scan.C", (batch, seq_len, d_state), 1.0, dtype)
    r["z"] = draw_normal(seed, "scan.z", (batch, seq_len, d_inner), 1.0, dtype) if with_z else None
    r["dt_bias"] = dt_bias_init(seed, "scan.dt_bias", d_inner)
    r["A_log"] = a_log_init(d_inner, d_state)
    r["D"] = np.ones(d_inner, dtype=np.float32)
    r["h0"] = draw_normal(seed, "scan.h0", (batch, d_inner, d_state), 1.0, "f32") if with_h0 else None
    return r


def swa_inputs(seed: int, batch: int, seq_len: int, n_q: int, n_kv: int, head_dim: int,
               dtype: str) -> Dict[str, np.ndarray]:
    """Mixer-only attention inputs: q, k, v ~ N(0,1), layout [B, L, heads, head_dim]."""
    return {
        "q": draw_normal(seed, "swa.q", (batch, seq_len, n_q, head_dim), 1.0, dtype),
        "k": draw_normal(seed, "swa.k", (batch, seq_len, n_kv, head_dim), 1.0, dtype),
        "v": draw_normal(seed, "swa.v", (batch, seq_len, n_kv, head_dim), 1.0, dtype),
    }
