"""Shared test helpers: device marshalling and the error metric.

Error metric (the reading of "max relative error" used throughout):
    err = max( max_i |g_i - o_i| / max_i |o_i| ,  ||g - o||_2 / ||o||_2 )
i.e. the l-infinity relative error of the tensor, and the normwise relative
error must both stay below the threshold.  Thresholds: fp32 paths 1e-4,
bf16-input / fp32-accumulate paths 2e-2.  (An elementwise ratio is undefined
at zeros; floored at the tensor RMS it is dominated by the bf16 rounding of
rotated q/k that every bf16 tensor-core attention performs: 4.6% from that
rounding alone on N(0,1) inputs, against 0.28% l-inf and 0.27% normwise.)
"""
import numpy as np

TOL = {"f32": 1e-4, "bf16": 2e-2}


def linf_rel(g, o) -> float:
    g = np.asarray(g, dtype=np.float64)
    o = np.asarray(o, dtype=np.float64)
    if o.size == 0:
        return 0.0
    return float(np.max(np.abs(g - o)) / max(float(np.max(np.abs(o))), 1e-300))


def rel_err(g, o) -> float:
    """max(l-inf relative, normwise relative) error of g against the reference o."""
    if np.asarray(o).size == 0:
        return 0.0
    return max(linf_rel(g, o), norm_err(g, o))


def norm_err(g, o) -> float:
    g = np.asarray(g, dtype=np.float64)
    o = np.asarray(o, dtype=np.float64)
    return float(np.linalg.norm(g - o) / max(np.linalg.norm(o), 1e-300))


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
