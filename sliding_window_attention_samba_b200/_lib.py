"""ctypes binding of libsamba.so: argument marshalling only.

Every function here has the name and argument order of its C counterpart in
include/samba.h.  Tensors are torch CUDA tensors (device memory and streams are
torch's); they are passed to the library as raw device pointers.  Nothing is
computed here, and there is no fallback: if the shared library is missing the
import fails loudly.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

_HERE = os.path.dirname(os.path.abspath(__file__))
# SAMBA_DEBUG_CHECKS=1 selects the debug-check build (device index checks and
# workspace guard bands; same symbols and results)
DEBUG_CHECKS = os.environ.get("SAMBA_DEBUG_CHECKS", "0") not in ("", "0")
LIB_PATH = os.path.join(_HERE, "libsamba_debug.so" if DEBUG_CHECKS else "libsamba.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with `python -m sliding_window_attention_samba_b200.build"
        f"{' --debug-checks' if DEBUG_CHECKS else ''}` "
        "(the CUDA path has no CPU fallback)")

_L = ctypes.CDLL(LIB_PATH)

c_void_p = ctypes.c_void_p
c_int = ctypes.c_int
c_int64 = ctypes.c_int64
c_size_t = ctypes.c_size_t
c_float = ctypes.c_float

SAMBA_F32, SAMBA_BF16 = 0, 1
(SAMBA_OK, SAMBA_ERR_INVALID_ARG, SAMBA_ERR_UNSUPPORTED, SAMBA_ERR_CUDA, SAMBA_ERR_TIMEOUT,
 SAMBA_ERR_DEVICE, SAMBA_ERR_BOUNDS) = range(7)
EPI_NONE, EPI_RESIDUAL, EPI_SWIGLU, EPI_SOFTPLUS_BIAS = 0, 1, 2, 3
STATUS = {0: "SAMBA_OK", 1: "SAMBA_ERR_INVALID_ARG", 2: "SAMBA_ERR_UNSUPPORTED", 3: "SAMBA_ERR_CUDA",
          4: "SAMBA_ERR_TIMEOUT", 5: "SAMBA_ERR_DEVICE", 6: "SAMBA_ERR_BOUNDS"}


class SambaError(RuntimeError):
    def __init__(self, fn: str, code: int, detail: str = ""):
        super().__init__(f"{fn} returned {STATUS.get(code, code)}" + (f" [{detail}]" if detail else ""))
        self.code = code
        self.detail = detail


class BlockConfig(ctypes.Structure):
    _fields_ = [("d_model", c_int), ("d_inner", c_int), ("d_state", c_int), ("d_conv", c_int),
                ("dt_rank", c_int), ("n_q", c_int), ("n_kv", c_int), ("head_dim", c_int), ("window", c_int),
                ("d_ff", c_int), ("rope_base", c_float), ("norm_eps", c_float), ("dtype", c_int)]


class BlockWeights(ctypes.Structure):
    _fields_ = [("norm_g", c_void_p * 4), ("W_in", c_void_p), ("conv_w", c_void_p), ("conv_b", c_void_p),
                ("W_x", c_void_p), ("W_dt", c_void_p), ("dt_bias", c_void_p), ("A_log", c_void_p),
                ("Dskip", c_void_p), ("W_out", c_void_p), ("Wq", c_void_p), ("Wk", c_void_p), ("Wv", c_void_p),
                ("Wo", c_void_p), ("mlp1_W1", c_void_p), ("mlp1_W2", c_void_p), ("mlp1_W3", c_void_p),
                ("mlp2_W1", c_void_p), ("mlp2_W2", c_void_p), ("mlp2_W3", c_void_p)]


class Model(ctypes.Structure):
    _fields_ = [("cfg", BlockConfig), ("n_layers", c_int), ("kinds", ctypes.POINTER(c_int)),
                ("layers", ctypes.POINTER(BlockWeights)), ("embedding", c_void_p), ("final_norm", c_void_p),
                ("lm_head", c_void_p), ("vocab", c_int)]


LAYER_MAMBA, LAYER_MLP, LAYER_SWA = 0, 1, 2


class LayerState(ctypes.Structure):
    _fields_ = [("ssm", c_void_p), ("conv", c_void_p), ("k_ring", c_void_p), ("v_ring", c_void_p)]


class DecodeState(ctypes.Structure):
    _fields_ = [("ssm", c_void_p), ("conv", c_void_p), ("k_ring", c_void_p), ("v_ring", c_void_p),
                ("pos", c_void_p)]


class BlockTaps(ctypes.Structure):
    _fields_ = [("branch", c_void_p * 4), ("resid", c_void_p * 3)]


def _sig(name, restype, argtypes):
    f = getattr(_L, name)
    f.restype = restype
    f.argtypes = argtypes
    return f


_status_string = _sig("samba_status_string", ctypes.c_char_p, [c_int])
_version = _sig("samba_version", ctypes.c_char_p, [])
_last_cuda_error = _sig("samba_last_cuda_error", ctypes.c_char_p, [])
_set_timing = _sig("samba_set_gemm_timing", c_int, [c_int, c_void_p, c_void_p, c_int])
_timing_count = _sig("samba_gemm_timing_count", c_int, [])
_get_error = _sig("samba_get_error", c_int, [c_void_p])
_scan_stall = _sig("samba_debug_scan_stall", c_int, [c_int, ctypes.c_uint64])
_dbg_enabled = _sig("samba_debug_checks_enabled", c_int, [])
_check_site = _sig("samba_last_check_site", ctypes.c_char_p, [])
_selftest_ws = _sig("samba_debug_selftest_workspace_size", c_size_t, [])
_selftest = _sig("samba_debug_check_selftest", c_int, [c_int, c_void_p, c_size_t, c_void_p])
_scan_ws = _sig("samba_selective_scan_workspace_size", c_size_t, [c_int, c_int, c_int, c_int])
_scan = _sig("samba_selective_scan", c_int,
             [c_void_p, c_void_p, c_void_p, c_int, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
              c_void_p, c_void_p, c_int, c_int, c_int, c_int, c_int, c_void_p, c_size_t, c_void_p])
_scan_xdbl = _sig("samba_selective_scan_xdbl", c_int,
                  [c_void_p, c_void_p, c_int, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                   c_void_p, c_int, c_int, c_int, c_int, c_int, c_void_p])
_swa_ws = _sig("samba_swa_workspace_size", c_size_t, [c_int, c_int, c_int, c_int, c_int, c_float, c_int])
_swa = _sig("samba_swa_fwd", c_int,
            [c_void_p, c_void_p, c_void_p, c_void_p, c_int, c_int, c_int, c_int, c_int, c_int, c_float, c_int64,
             c_float, c_int, c_void_p, c_size_t, c_void_p])
_swa_noalloc = _sig("samba_swa_fwd_noalloc", c_int,
                    [c_void_p, c_void_p, c_void_p, c_void_p, c_int, c_int, c_int, c_int, c_int, c_int, c_float,
                     c_int64, c_float, c_int, c_void_p])
_rmsnorm = _sig("samba_rmsnorm", c_int, [c_void_p, c_void_p, c_void_p, c_int64, c_int, c_float, c_int, c_void_p])
_conv = _sig("samba_causal_conv1d", c_int,
             [c_void_p, c_int64, c_void_p, c_void_p, c_void_p, c_void_p, c_int, c_int, c_int, c_int, c_int,
              c_void_p])
_linear = _sig("samba_linear", c_int,
               [c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_int64, c_int, c_int, c_int, c_int,
                c_void_p])
_block_ws = _sig("samba_block_workspace_size", c_size_t, [ctypes.POINTER(BlockConfig), c_int, c_int])
_block = _sig("samba_block_fwd", c_int,
              [ctypes.POINTER(BlockConfig), ctypes.POINTER(BlockWeights), c_void_p, c_void_p,
               ctypes.POINTER(DecodeState), ctypes.POINTER(BlockTaps), c_int, c_int, c_void_p, c_size_t, c_void_p])
_chunk_ws = _sig("samba_block_chunk_workspace_size", c_size_t, [ctypes.POINTER(BlockConfig), c_int, c_int])
_chunk = _sig("samba_block_fwd_chunk", c_int,
              [ctypes.POINTER(BlockConfig), ctypes.POINTER(BlockWeights), c_void_p, c_void_p,
               ctypes.POINTER(DecodeState), c_int64, ctypes.POINTER(BlockTaps), c_int, c_int, c_void_p, c_size_t,
               c_void_p])
_model_ws = _sig("samba_model_workspace_size", c_size_t, [ctypes.POINTER(Model), c_int, c_int])
_model = _sig("samba_model_prefill", c_int,
              [ctypes.POINTER(Model), c_void_p, c_void_p, c_int, c_int, c_void_p, c_size_t, c_void_p])
_mstep_ws = _sig("samba_model_step_workspace_size", c_size_t, [ctypes.POINTER(Model), c_int])
_mstep = _sig("samba_model_step", c_int,
              [ctypes.POINTER(Model), c_void_p, c_void_p, ctypes.POINTER(LayerState), c_void_p, c_int, c_void_p,
               c_size_t, c_void_p])
_step_ws = _sig("samba_step_workspace_size", c_size_t, [ctypes.POINTER(BlockConfig), c_int])
_step = _sig("samba_step", c_int,
             [ctypes.POINTER(BlockConfig), ctypes.POINTER(BlockWeights), c_void_p, c_void_p,
              ctypes.POINTER(DecodeState), c_int, c_void_p, c_size_t, c_void_p])


def lib_handle():
    return _L


def _p(t) -> Optional[int]:
    """Device pointer of a tensor (None -> NULL)."""
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is not None:
        return stream if isinstance(stream, int) else stream.cuda_stream
    import torch
    return torch.cuda.current_stream().cuda_stream


def _check(fn: str, rc: int):
    if rc != 0:
        detail = _last_cuda_error().decode() if rc == SAMBA_ERR_CUDA else ""
        raise SambaError(fn, rc, detail)


def samba_last_cuda_error() -> str:
    return _last_cuda_error().decode()


def samba_status_string(code: int) -> str:
    return _status_string(code).decode()


def samba_version() -> str:
    return _version().decode()


def samba_set_gemm_timing(epi: int, start_events=(), stop_events=()):
    """Install (epi >= 0) or remove (epi < 0) the projection timing hook.  The
    events are torch.cuda.Event(enable_timing=True) objects that have been
    recorded once (so that their CUDA events exist); keep them alive while
    the hook is installed."""
    if epi < 0:
        _check("samba_set_gemm_timing", _set_timing(-1, None, None, 0))
        return
    n = len(start_events)
    if n != len(stop_events) or n == 0:
        raise ValueError("need equally many start and stop events")
    hs = [int(e.cuda_event) for e in start_events]
    he = [int(e.cuda_event) for e in stop_events]
    if not all(hs) or not all(he):
        raise ValueError("record every event once before installing the hook")
    a = (c_void_p * n)(*hs)
    b = (c_void_p * n)(*he)
    _check("samba_set_gemm_timing", _set_timing(epi, ctypes.cast(a, c_void_p), ctypes.cast(b, c_void_p), n))


def samba_gemm_timing_count() -> int:
    return _timing_count()


def samba_debug_scan_stall(stop_after_chunks: int, wait_limit_ns: int = 0) -> None:
    """Set (stop_after_chunks >= 0) or clear (-1) the scan's failure-detection
    test hook (see include/samba.h)."""
    _check("samba_debug_scan_stall", _scan_stall(stop_after_chunks, wait_limit_ns))


def samba_get_error(stream=None) -> int:
    return _get_error(_stream(stream))


def samba_debug_checks_enabled() -> int:
    return _dbg_enabled()


def samba_last_check_site() -> str:
    return _check_site().decode()


def samba_debug_selftest_workspace_size() -> int:
    return _selftest_ws()


def samba_debug_check_selftest(kind: int, workspace=None, workspace_bytes: int = 0, stream=None) -> int:
    """Returns the status code (SAMBA_ERR_UNSUPPORTED in the release build)."""
    return _selftest(kind, _p(workspace), workspace_bytes, _stream(stream))


def samba_selective_scan_workspace_size(B, L, D, N) -> int:
    return _scan_ws(B, L, D, N)


def samba_selective_scan(u, dt, dt_bias, dt_softplus, A_log, Bm, Cm, Dskip, z, h0, hT, y, B, L, D, N, dtype,
                         workspace=None, workspace_bytes=0, stream=None):
    _check("samba_selective_scan",
           _scan(_p(u), _p(dt), _p(dt_bias), int(dt_softplus), _p(A_log), _p(Bm), _p(Cm), _p(Dskip), _p(z), _p(h0),
                 _p(hT), _p(y), B, L, D, N, dtype, _p(workspace), workspace_bytes, _stream(stream)))


def samba_swa_workspace_size(B, L, Hq, Hkv, head_dim, rope_base, dtype) -> int:
    return _swa_ws(B, L, Hq, Hkv, head_dim, rope_base, dtype)


def samba_selective_scan_xdbl(u, x_dbl, dt_rank, W_dt, dt_bias, A_log, Dskip, z, h0, hT, y, B, L, D, N, dtype,
                              stream=None):
    _check("samba_selective_scan_xdbl",
           _scan_xdbl(_p(u), _p(x_dbl), dt_rank, _p(W_dt), _p(dt_bias), _p(A_log), _p(Dskip), _p(z), _p(h0),
                      _p(hT), _p(y), B, L, D, N, dtype, _stream(stream)))


def samba_swa_fwd(q, k, v, o, B, L, Hq, Hkv, head_dim, window, rope_base, pos0, softmax_scale, dtype,
                  workspace=None, workspace_bytes=0, stream=None):
    _check("samba_swa_fwd",
           _swa(_p(q), _p(k), _p(v), _p(o), B, L, Hq, Hkv, head_dim, window, rope_base, pos0, softmax_scale, dtype,
                _p(workspace), workspace_bytes, _stream(stream)))


def samba_swa_fwd_noalloc(q, k, v, o, B, L, Hq, Hkv, head_dim, window, rope_base, pos0, softmax_scale, dtype,
                          stream=None):
    _check("samba_swa_fwd_noalloc",
           _swa_noalloc(_p(q), _p(k), _p(v), _p(o), B, L, Hq, Hkv, head_dim, window, rope_base, pos0,
                        softmax_scale, dtype, _stream(stream)))


def samba_rmsnorm(x, g, out, rows, dim, eps, dtype, stream=None):
    _check("samba_rmsnorm", _rmsnorm(_p(x), _p(g), _p(out), rows, dim, eps, dtype, _stream(stream)))


def samba_causal_conv1d(x, ld_x, w, bias, u, conv_state, B, L, D, k, dtype, stream=None):
    _check("samba_causal_conv1d",
           _conv(_p(x), ld_x, _p(w), _p(bias), _p(u), _p(conv_state), B, L, D, k, dtype, _stream(stream)))


def samba_linear(x, W, W2, bias, resid, out, M, N, K, epilogue, dtype, stream=None):
    _check("samba_linear",
           _linear(_p(x), _p(W), _p(W2), _p(bias), _p(resid), _p(out), M, N, K, epilogue, dtype, _stream(stream)))


def samba_block_workspace_size(cfg: BlockConfig, B, L) -> int:
    return _block_ws(ctypes.byref(cfg), B, L)


def samba_block_fwd(cfg: BlockConfig, w: BlockWeights, x_in, x_out, st: Optional[DecodeState],
                    taps: Optional[BlockTaps], B, L, workspace, workspace_bytes, stream=None):
    _check("samba_block_fwd",
           _block(ctypes.byref(cfg), ctypes.byref(w), _p(x_in), _p(x_out), ctypes.byref(st) if st else None,
                  ctypes.byref(taps) if taps else None, B, L, _p(workspace), workspace_bytes, _stream(stream)))


def samba_block_chunk_workspace_size(cfg: BlockConfig, B, L) -> int:
    return _chunk_ws(ctypes.byref(cfg), B, L)


def samba_block_fwd_chunk(cfg: BlockConfig, w: BlockWeights, x_in, x_out, st: DecodeState, pos0,
                          taps: Optional[BlockTaps], B, L, workspace, workspace_bytes, stream=None):
    _check("samba_block_fwd_chunk",
           _chunk(ctypes.byref(cfg), ctypes.byref(w), _p(x_in), _p(x_out), ctypes.byref(st) if st else None, pos0,
                  ctypes.byref(taps) if taps else None, B, L, _p(workspace), workspace_bytes, _stream(stream)))


def samba_model_workspace_size(m: Model, B, L) -> int:
    return _model_ws(ctypes.byref(m), B, L)


def samba_model_prefill(m: Model, ids, logits, B, L, workspace, workspace_bytes, stream=None):
    _check("samba_model_prefill",
           _model(ctypes.byref(m), _p(ids), _p(logits), B, L, _p(workspace), workspace_bytes, _stream(stream)))


def samba_model_step_workspace_size(m: Model, B) -> int:
    return _mstep_ws(ctypes.byref(m), B)


def make_layer_states(states: Sequence[dict]):
    """Host array of LayerState from dicts of device tensors (ssm, conv, k_ring, v_ring; absent = NULL)."""
    n = len(states)
    arr = (LayerState * max(n, 1))(*[LayerState(_p(d.get("ssm")), _p(d.get("conv")), _p(d.get("k_ring")),
                                                 _p(d.get("v_ring"))) for d in states])
    return arr


def samba_model_step(m: Model, ids_t, logits, states, pos, B, workspace, workspace_bytes, stream=None):
    _check("samba_model_step",
           _mstep(ctypes.byref(m), _p(ids_t), _p(logits), ctypes.cast(states, ctypes.POINTER(LayerState)), _p(pos),
                  B, _p(workspace), workspace_bytes, _stream(stream)))


def samba_step_workspace_size(cfg: BlockConfig, B) -> int:
    return _step_ws(ctypes.byref(cfg), B)


def samba_step(cfg: BlockConfig, w: BlockWeights, x_t, y_t, st: DecodeState, B, workspace, workspace_bytes,
               stream=None):
    _check("samba_step",
           _step(ctypes.byref(cfg), ctypes.byref(w), _p(x_t), _p(y_t), ctypes.byref(st), B, _p(workspace),
                 workspace_bytes, _stream(stream)))


# ---------------------------------------------------------------------------
# Convenience marshalling for whole blocks (torch tensors -> ctypes structs)
# ---------------------------------------------------------------------------
def make_config(shape) -> BlockConfig:
    return BlockConfig(shape.d_model, shape.d_inner, shape.d_state, shape.d_conv, shape.dt_rank, shape.n_q,
                       shape.n_kv, shape.head_dim, shape.window, shape.d_ff, float(shape.rope_base),
                       float(shape.norm_eps), SAMBA_BF16 if shape.dtype == "bf16" else SAMBA_F32)


def make_weights(wt: dict) -> BlockWeights:
    """wt: dict of device tensors keyed like inputs.block_weights()."""
    w = BlockWeights()
    for i in range(4):
        w.norm_g[i] = _p(wt.get(f"norm{i}"))
    for name in ("W_in", "conv_w", "conv_b", "W_x", "W_dt", "dt_bias", "A_log", "W_out", "Wq", "Wk", "Wv", "Wo",
                 "mlp1_W1", "mlp1_W2", "mlp1_W3", "mlp2_W1", "mlp2_W2", "mlp2_W3"):
        setattr(w, name, _p(wt.get(name)))
    w.Dskip = _p(wt.get("D"))
    return w


def make_model(cfg: BlockConfig, kinds: Sequence[int], layers: Sequence[dict], embedding, final_norm, lm_head,
               vocab: int) -> Model:
    """kinds: LAYER_* per sub-layer; layers: dicts of device tensors keyed like
    inputs.block_weights() (a layer's kind decides which it reads).  The host
    arrays live as attributes of the returned struct; keep the tensors alive."""
    n = len(kinds)
    ka = (c_int * max(n, 1))(*kinds)
    la = (BlockWeights * max(n, 1))(*[make_weights(d) for d in layers])
    m = Model(cfg, n, ctypes.cast(ka, ctypes.POINTER(c_int)), ctypes.cast(la, ctypes.POINTER(BlockWeights)),
              _p(embedding), _p(final_norm), _p(lm_head), vocab)
    m._keep = (ka, la)
    return m


def make_state(ssm, conv, k_ring, v_ring, pos) -> DecodeState:
    return DecodeState(_p(ssm), _p(conv), _p(k_ring), _p(v_ring), _p(pos))


def make_taps(branch: Sequence = (None,) * 4, resid: Sequence = (None,) * 3) -> BlockTaps:
    t = BlockTaps()
    for i in range(4):
        t.branch[i] = _p(branch[i])
    for i in range(3):
        t.resid[i] = _p(resid[i])
    return t
