#!/usr/bin/env python3
"""Samba block prefill benchmark on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl samba|reference]

Workload: long-context prefill, batch 1, L = 131072 tokens through a stack of 4
bf16 Samba blocks (d_model 2048, d_inner 4096, d_state 16, d_conv 4, dt_rank 128,
32/4 heads of 64, window 2048, SwiGLU 8192).  One step = the whole stack over one
sequence.  Metric: prefill tokens/s per block = B*L / (step time / 4), summed over
ranks (each rank runs its own replica: no data-path collective).

Printed JSON line (rank 0): value (device time, inputs resident in HBM), e2e
(same metric through the C ABI with pinned host input/output copied inside the
timed region), roofline of the dominant kernel (CUDA events around its launches
inside the timed region), per-kernel figures (scan HBM GB/s, SWA and projection
TF/s) from an attribution pass over the same kernels, the oracle CPU baseline,
clocks sampled during the timed region; at one GPU also `decode` (batch 32,
65 536 graph-replayed samba_step calls after a 4096-token prefill, against its
HBM roofline) and `sweep` (scan and SWA alone at L = 4K .. 1M).  `--impl
reference` times the fp64 CPU oracle on a bounded sample of the same workload
instead (the same sample as the line's cpu_baseline).
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

from sliding_window_attention_samba_b200 import inputs as I  # noqa: E402

WORKLOAD = "prefill_bf16_L131072_x4"
MUFU_EX2_PER_CLK_SM = 16  # ex2.approx results per clock per SM (sm_100a MUFU)
N_SMS = 148
METRIC = "prefill tokens/s per Samba block at L=128K; scan HBM GB/s & SWA TC util vs peak"
UNIT = "tokens/s"


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="samba", choices=["samba", "reference"])
    ap.add_argument("--seq-len", type=int, default=None, help="override L (parity/debug runs only)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extras", action="store_true",
                    help="prefill line only: skip the decode and mixer-sweep measurements")
    ap.add_argument("--workload", default="prefill",
                    choices=["prefill", "block", "block38", "decode", "sweep", "chunked", "model",
                             "model_decode"],
                    help="prefill: 4-block L=131072 stack (the headline); block: one block at B=4, L=4096; "
                         "block38: one block at the 3.8B model's widths (head_dim 256), L=131072; "
                         "decode: B=32 samba_step stream; "
                         "sweep: scan and SWA alone at L = 4K..1M; "
                         "chunked: one block over L=1M in 32K-token chunks (samba_block_fwd_chunk); "
                         "model: prompt processing of a Samba-1.7B-layout stack vs a GQA Transformer of the "
                         "same width (samba_model_prefill), 128K tokens per step at L = 4K..128K; "
                         "model_decode: decode tokens/s of the same two stacks at batch 16 over 64K generated "
                         "tokens (samba_model_step, CUDA graph replay)")
    ap.add_argument("--max-len", type=int, default=1048576, help="sweep: largest L")
    ap.add_argument("--prefill", type=int, default=None,
                    help="decode: override the 4096-token prefill (profiling runs only)")
    return ap.parse_args()


def load_peaks():
    """(HBM GB/s, burst bf16 TF/s, sustained bf16 TF/s, source): the measured
    figures of MEASURED_PEAKS.json when present, else fallback figures for the
    B200 (6.65 TB/s, 1.59 PF/s burst, ~1.4 PF/s sustained)."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d.get("hbm_gbs", 6650.0), d.get("bf16_tflops", 1590.0), d.get("bf16_tflops_sustained", 1400.0), "measured"
    return 6650.0, 1590.0, 1400.0, "fallback"


def peak_clock_mhz(kind):
    """SM clock (MHz) at which a peak was taken: from MEASURED_PEAKS.json when it
    records one (any numeric field whose name mentions the peak kind and a
    clock), else the clock of the fallback sustained figure
    (~1.4 PF/s at ~1.3 GHz).  None when unknown."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        def walk(d, path=""):
            for k, v in d.items():
                name = (path + "." + k).lower()
                if isinstance(v, dict):
                    yield from walk(v, name)
                elif isinstance(v, (int, float)) and ("mhz" in name or "clock" in name):
                    yield name, float(v)
        cands = list(walk(json.load(open(p))))
        sus = [v for n, v in cands if "sustain" in n and 300 < v < 3000]
        burst = [v for n, v in cands if "sustain" not in n and ("bf16" in n or "gemm" in n) and 300 < v < 3000]
        if kind == "sustained" and sus:
            return sus[0]
        if kind == "burst" and burst:
            return burst[0]
        return None
    return 1300.0 if kind == "sustained" else None


# ---------------------------------------------------------------------------
# clocks during the timed region
# ---------------------------------------------------------------------------
class ClockSampler:
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
         "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
         "clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.idx = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.idx), f"--query-gpu={self.Q}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if not self.proc:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx.append(float(f[2]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        os.unlink(self.path)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


# ---------------------------------------------------------------------------
# the CUDA path
# ---------------------------------------------------------------------------
def graph_kernel_nodes(graph):
    """Kernel nodes of a CUDA graph captured with keep_graph=True (the launches
    one replay makes), or None where the runtime bindings cannot tell."""
    try:
        from cuda.bindings import runtime as rt
        g = rt.cudaGraph_t(init_value=graph.raw_cuda_graph())
        err, _, n = rt.cudaGraphGetNodes(g, 0)
        if err != rt.cudaError_t.cudaSuccess:
            return None
        err, nodes, n = rt.cudaGraphGetNodes(g, n)
        if err != rt.cudaError_t.cudaSuccess:
            return None
        kernel = rt.cudaGraphNodeType.cudaGraphNodeTypeKernel
        return sum(1 for x in nodes[:n] if rt.cudaGraphNodeGetType(x)[1] == kernel)
    except Exception:
        return None


def make_stack(torch, L, shape, n_blocks, seed, dev):
    """Random-init weights of the stack on the device (N(0, 0.02) matrices,
    S4D-Real A, D = 1, Delta bias in [1e-3, 1e-1], unit norm gains)."""
    g = torch.Generator(device=dev)
    blocks = []
    s = shape
    bf = torch.bfloat16
    for li in range(n_blocks):
        g.manual_seed(I.tensor_key(seed, f"stack.L{li}") & ((1 << 63) - 1))

        def mat(o, i):
            return (torch.randn(o, i, generator=g, device=dev) * 0.02).to(bf)

        w = {f"norm{i}": torch.ones(s.d_model, device=dev) for i in range(4)}
        w["W_in"] = mat(2 * s.d_inner, s.d_model)
        w["conv_w"] = torch.randn(s.d_inner, s.d_conv, generator=g, device=dev) * 0.02
        w["conv_b"] = None
        w["W_x"] = mat(s.dt_rank + 2 * s.d_state, s.d_inner)
        w["W_dt"] = mat(s.d_inner, s.dt_rank)
        w["dt_bias"] = torch.from_numpy(I.dt_bias_init(seed, f"stack.L{li}.dt_bias", s.d_inner)).to(dev)
        w["A_log"] = torch.from_numpy(I.a_log_init(s.d_inner, s.d_state)).to(dev)
        w["D"] = torch.ones(s.d_inner, device=dev)
        w["W_out"] = mat(s.d_model, s.d_inner)
        w["Wq"] = mat(s.n_q * s.head_dim, s.d_model)
        w["Wk"] = mat(s.n_kv * s.head_dim, s.d_model)
        w["Wv"] = mat(s.n_kv * s.head_dim, s.d_model)
        w["Wo"] = mat(s.d_model, s.n_q * s.head_dim)
        for m in (1, 2):
            w[f"mlp{m}_W1"] = mat(s.d_ff, s.d_model)
            w[f"mlp{m}_W2"] = mat(s.d_ff, s.d_model)
            w[f"mlp{m}_W3"] = mat(s.d_model, s.d_ff)
        blocks.append((w, L.make_weights(w)))
    return blocks


def gemm_list(s, T):
    """(name, M, N, K, epilogue, flops) of every projection in one block, in launch order."""
    R, N16 = s.dt_rank, s.d_state
    qkvw = (s.n_q + 2 * s.n_kv) * s.head_dim
    g = [("in_proj", T, 2 * s.d_inner, s.d_model, 0),
         ("x_proj", T, R + 2 * N16, s.d_inner, 0),
         ("dt_proj", T, s.d_inner, R, 3),
         ("out_proj", T, s.d_model, s.d_inner, 1),
         ("mlp1_up", T, s.d_ff, s.d_model, 2),
         ("mlp1_down", T, s.d_model, s.d_ff, 1),
         ("qkv", T, qkvw, s.d_model, 0),
         ("o_proj", T, s.d_model, s.n_q * s.head_dim, 1),
         ("mlp2_up", T, s.d_ff, s.d_model, 2),
         ("mlp2_down", T, s.d_model, s.d_ff, 1)]
    return [(n, M, N, K, e, 2.0 * M * N * K * (2 if e == 2 else 1)) for (n, M, N, K, e) in g]


def swa_flops(s, Bn, Ln):
    w = s.window
    pairs = Ln * w - w * (w - 1) / 2 if Ln >= w else Ln * (Ln + 1) / 2
    return 4.0 * s.head_dim * s.n_q * pairs * Bn


def dt_folded(s):
    """The block forms Delta inside the scan kernel (opt-in: SAMBA_SCAN_FOLD_DT=1;
    bf16, dt_rank <= 128, a multiple of 16): no separate dt projection launch."""
    return (os.environ.get("SAMBA_SCAN_FOLD_DT") == "1" and s.dtype == "bf16" and s.dt_rank % 16 == 0
            and 16 <= s.dt_rank <= 128)


def attribution_pass(torch, L, s, blocks, x, T, Bn, Ln, reps=2):
    """Times each kernel of one block separately through the component entry
    points (same kernels, same shapes, same stream) with CUDA events."""
    dev = x.device
    bf = torch.bfloat16
    st = torch.cuda.current_stream()
    w, _ = blocks[0]
    # realistic operand values: N(0,1) activations, step sizes Delta in [1e-3, 1e-1]
    xn = torch.empty(T, s.d_model, device=dev, dtype=bf).normal_()
    hz = torch.empty(T, 2 * s.d_inner, device=dev, dtype=bf).normal_()
    u = torch.empty(T, s.d_inner, device=dev, dtype=bf).normal_()
    xdbl = torch.empty(T, s.dt_rank + 2 * s.d_state, device=dev, dtype=bf).normal_()
    dlt = (torch.rand(T, s.d_inner, device=dev) * 0.099 + 0.001).to(bf)
    y = torch.empty(T, s.d_inner, device=dev, dtype=bf)
    big = torch.empty(T, s.d_ff, device=dev, dtype=bf)
    xo = torch.empty(T, s.d_model, device=dev, dtype=bf)
    q = torch.empty(Bn, Ln, s.n_q, s.head_dim, device=dev, dtype=bf).normal_()
    kk = torch.empty(Bn, Ln, s.n_kv, s.head_dim, device=dev, dtype=bf).normal_()
    vv = torch.empty_like(kk).normal_()
    o = torch.empty_like(q)
    times = {}

    def timed(name, fn):
        for _ in range(reps + 1):  # first call is a warm-up
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(st)
            fn()
            e1.record(st)
            e1.synchronize()
            times.setdefault(name, []).append(e0.elapsed_time(e1) * 1e-3)
        times[name] = times[name][1:]

    timed("rmsnorm", lambda: L.samba_rmsnorm(x, w["norm0"], xn, T, s.d_model, s.norm_eps, 1))
    W = {"in_proj": (w["W_in"], None, xn, hz), "x_proj": (w["W_x"], None, u, xdbl),
         "dt_proj": (w["W_dt"], None, None, dlt), "out_proj": (w["W_out"], None, y, xo),
         "mlp1_up": (w["mlp1_W1"], w["mlp1_W2"], xn, big), "mlp1_down": (w["mlp1_W3"], None, big, xo),
         "qkv": (w["Wq"], None, xn, None), "o_proj": (w["Wo"], None, o, xo)}
    for (name, M, N, K, e, fl) in gemm_list(s, T):
        if name in ("mlp2_up", "mlp2_down") or (name == "dt_proj" and dt_folded(s)):
            continue
        Wm, W2, a_in, out = W[name]
        a_t = torch.empty(M, K, device=dev, dtype=bf).normal_() if a_in is None or a_in.shape[1] != K else a_in
        o_t = torch.empty(M, N, device=dev, dtype=bf) if out is None or out.shape[1] != N else out
        Wt = Wm if Wm.shape == (N, K) else torch.empty(N, K, device=dev, dtype=bf).normal_()
        timed(name, lambda a_t=a_t, Wt=Wt, W2=W2, o_t=o_t, M=M, N=N, K=K, e=e: L.samba_linear(
            a_t, Wt, W2, w["dt_bias"] if e == 3 else None, x if e == 1 else None, o_t, M, N, K, e, 1))
    timed("conv", lambda: L.samba_causal_conv1d(hz, 2 * s.d_inner, w["conv_w"], None, u, None, Bn, Ln, s.d_inner,
                                                 s.d_conv, 1))
    if dt_folded(s):  # the block's scan forms Delta itself from the x_proj output
        timed("scan", lambda: _scan_xdbl(torch, L, s, w, u, xdbl, y, Bn, Ln))
    else:
        timed("scan", lambda: _scan_contig(torch, L, s, w, u, dlt, hz, y, Bn, Ln))
    timed("swa", lambda: L.samba_swa_fwd(q, kk, vv, o, Bn, Ln, s.n_q, s.n_kv, s.head_dim, s.window, 0.0, 0, 0.0, 1))
    return {k: sum(v) / len(v) for k, v in times.items()}


_SCAN_BUFS = {}


def _scan_contig(torch, L, s, w, u, dlt, hz, y, Bn, Ln):
    """Selective scan on contiguous [B, L, D] operands of the block's sizes."""
    key = (Bn, Ln)
    if key not in _SCAN_BUFS:
        dev = u.device
        T = Bn * Ln
        _SCAN_BUFS[key] = (torch.empty(T, s.d_inner, device=dev, dtype=torch.bfloat16).normal_(),
                           torch.empty(T, s.d_state, device=dev, dtype=torch.bfloat16).normal_(),
                           torch.empty(T, s.d_state, device=dev, dtype=torch.bfloat16).normal_())
    z, Bm, Cm = _SCAN_BUFS[key]
    L.samba_selective_scan(u, dlt, None, 0, w["A_log"], Bm, Cm, w["D"], z, None, None, y, Bn, Ln, s.d_inner,
                           s.d_state, 1)


def _scan_xdbl(torch, L, s, w, u, xdbl, y, Bn, Ln):
    """The scan with the dt projection folded in, on the x_proj output."""
    key = ("z", Bn, Ln)
    if key not in _SCAN_BUFS:
        _SCAN_BUFS[key] = torch.empty(Bn * Ln, s.d_inner, device=u.device, dtype=torch.bfloat16).normal_()
    z = _SCAN_BUFS[key]
    L.samba_selective_scan_xdbl(u, xdbl, s.dt_rank, w["W_dt"], w["dt_bias"], w["A_log"], w["D"], z, None, None, y,
                                Bn, Ln, s.d_inner, s.d_state, 1)


def workload_of(args):
    return {"block": "block_bf16_B4_L4096", "block38": "block38_bf16_L131072"}.get(args.workload, WORKLOAD)


def run_cuda(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist
    from sliding_window_attention_samba_b200 import _lib as L

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    shape, Bn, Ln, n_blocks, seed = I.WORKLOADS[workload_of(args)]
    if args.seq_len:
        Ln = args.seq_len
    s = shape
    T = Bn * Ln
    cfg = L.make_config(s)
    blocks = make_stack(torch, L, s, n_blocks, seed + 1000 * rank, dev)
    ws_bytes = L.samba_block_workspace_size(cfg, Bn, Ln)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    gx = torch.Generator(device=dev)
    gx.manual_seed(I.tensor_key(seed + rank, "stack.x") & ((1 << 63) - 1))
    x0 = torch.randn(Bn, Ln, s.d_model, generator=gx, device=dev).to(torch.bfloat16)
    bufs = [torch.empty_like(x0), torch.empty_like(x0)]
    stream = torch.cuda.current_stream()

    def step(x_in, y_out=None):
        """The stack over one sequence; the last block writes y_out if given."""
        cur = x_in
        for i, (_, wst) in enumerate(blocks):
            out = y_out if (y_out is not None and i == len(blocks) - 1) else bufs[i % 2]
            L.samba_block_fwd(cfg, wst, cur, out, None, None, Bn, Ln, ws, ws_bytes)
            cur = out
        return cur

    def barrier():
        if world > 1:
            dist.barrier()

    for _ in range(args.warmup):
        step(x0)
    torch.cuda.synchronize()
    assert L.samba_get_error() == 0, "device error during warm-up"

    # ---- device-timed region (inputs resident; activations >> L2, no flush needed)
    # The dominant kernel (the SwiGLU up-projection, two per block) is bracketed
    # by CUDA events inside the region through the library's timing hook.
    n_up = args.steps * n_blocks * 2
    up_ev = None
    try:
        up_ev = ([torch.cuda.Event(enable_timing=True) for _ in range(n_up)],
                 [torch.cuda.Event(enable_timing=True) for _ in range(n_up)])
        for ev in up_ev[0] + up_ev[1]:
            ev.record(stream)  # creates the CUDA events
        torch.cuda.synchronize()
        L.samba_set_gemm_timing(L.EPI_SWIGLU, up_ev[0], up_ev[1])
    except Exception as ex:  # noqa: BLE001  (the attribution pass still times the kernel)
        print(f"bench: timing hook unavailable ({ex}); roofline from the attribution pass", file=sys.stderr)
        up_ev = None
    clocks = ClockSampler(local_rank)
    clocks.start()
    barrier()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        step(x0)
    e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    clk = clocks.stop()
    t_dev = e0.elapsed_time(e1) * 1e-3
    t_up_live = None
    if up_ev is not None:
        n_rec = L.samba_gemm_timing_count()
        L.samba_set_gemm_timing(-1)
        try:
            if n_rec == n_up:
                d = [a.elapsed_time(b) * 1e-3 for a, b in zip(up_ev[0], up_ev[1])]
                if min(d) > 0:
                    t_up_live = (sum(d) / len(d), len(d))
        except Exception as ex:  # noqa: BLE001
            print(f"bench: timing hook events unreadable ({ex})", file=sys.stderr)
    assert L.samba_get_error() == 0, "device error in the timed region"

    # ---- end to end: every step copies its input from pinned host memory and
    # its output back.  The copies run on their own stream, double-buffered, so
    # step k's output leaves and step k+1's input arrives while step k computes.
    xh = x0.cpu().pin_memory()
    yh = torch.empty_like(xh).pin_memory()
    xd = [torch.empty_like(x0), torch.empty_like(x0)]
    yd = [torch.empty_like(x0), torch.empty_like(x0)]
    cps = torch.cuda.Stream()
    barrier()
    torch.cuda.synchronize()
    f0 = torch.cuda.Event(enable_timing=True)
    f1 = torch.cuda.Event(enable_timing=True)
    h2d = [torch.cuda.Event() for _ in range(args.steps)]
    done = [torch.cuda.Event() for _ in range(args.steps)]
    d2h = [torch.cuda.Event() for _ in range(args.steps)]
    f0.record(cps)

    def load(k):
        with torch.cuda.stream(cps):
            if k >= 2:
                cps.wait_event(done[k - 2])  # step k-2 no longer reads xd[k % 2]
            xd[k % 2].copy_(xh, non_blocking=True)
            h2d[k].record(cps)

    load(0)
    for k in range(args.steps):
        if k + 1 < args.steps:
            load(k + 1)
        stream.wait_event(h2d[k])
        if k >= 2:
            stream.wait_event(d2h[k - 2])  # yd[k % 2] has been read back
        step(xd[k % 2], yd[k % 2])
        done[k].record(stream)
        with torch.cuda.stream(cps):
            cps.wait_event(done[k])
            yh.copy_(yd[k % 2], non_blocking=True)
            d2h[k].record(cps)
    f1.record(cps)
    torch.cuda.synchronize()
    barrier()
    t_e2e = f0.elapsed_time(f1) * 1e-3

    # ---- per-kernel attribution (same kernels and shapes, one block)
    kt = attribution_pass(torch, L, s, blocks, x0.view(T, s.d_model), T, Bn, Ln) if rank == 0 else {}

    t_dev, t_e2e = max_over_ranks(t_dev, world, dev), max_over_ranks(t_e2e, world, dev)
    return dict(t_dev=t_dev, t_e2e=t_e2e, clocks=clk, kt=kt, s=s, Bn=Bn, Ln=Ln, n_blocks=n_blocks,
                h2d=xh.numel() * 2, d2h=yh.numel() * 2, t_up_live=t_up_live)


def max_over_ranks(t, world, device):
    """The slowest rank's time (every rank calls it, in the same order)."""
    if world == 1:
        return t
    import torch
    import torch.distributed as dist
    tt = torch.tensor([t], device=device, dtype=torch.float64)
    dist.all_reduce(tt, op=dist.ReduceOp.MAX)
    return float(tt.item())


def replica_throughput(tokens_per_rank, world, t_max, steps, n_blocks):
    """Whole-job tokens/s per block: the tokens all replicas pushed through each
    block, over the slowest rank's time per step and block."""
    return tokens_per_rank * world / (t_max / steps / n_blocks)


def kernel_report(kt, s, T, Bn, Ln, peaks, t_up_live=None, clocks=None):
    hbm, tf_burst, tf_sus, src = peaks
    gl = gemm_list(s, T)
    g_flops = sum(fl for (n, M, N, K, e, fl) in gl if n in kt)
    g_time = sum(kt[n] for (n, *_r) in gl if n in kt)
    n_g = len([1 for (n, *_r) in gl if n in kt])
    rep = {"gemm": {"tflops": g_flops / g_time / 1e12, "frac_of_" + src + "_bf16_peak": g_flops / g_time / 1e12 / tf_sus,
                    "per_gemm_tflops": {n: round(fl / kt[n] / 1e12, 1) for (n, M, N, K, e, fl) in gl if n in kt}}}
    scan_bytes = T * (8 * s.d_inner + 4 * s.d_state)
    rep["scan"] = {"gbs": scan_bytes / kt["scan"] / 1e9, "frac_of_" + src + "_hbm": scan_bytes / kt["scan"] / 1e9 / hbm,
                   "ms": kt["scan"] * 1e3}
    # The scan's binding unit is the exponential (MUFU) pipe: one ex2 per
    # (token, channel, state) element at 16 per clock per SM (measured on this
    # pool's B200 with a throughput microbenchmark: 4.6e12 ex2/s), at the run's
    # median SM clock.
    mhz = (clocks or {}).get("sm_mhz")
    if mhz:
        ex2_per_s = MUFU_EX2_PER_CLK_SM * N_SMS * mhz * 1e6
        floor = T * s.d_inner * s.d_state / ex2_per_s
        rep["scan"].update({"bound": "alu", "mufu_floor_ms": floor * 1e3, "frac_of_mufu_floor": floor / kt["scan"],
                            "mufu_peak": f"{MUFU_EX2_PER_CLK_SM} ex2/clk/SM x {N_SMS} SMs x {mhz:.0f} MHz"})
    sf = swa_flops(s, Bn, Ln)
    rep["swa"] = {"tflops": sf / kt["swa"] / 1e12, "frac_of_" + src + "_bf16_peak": sf / kt["swa"] / 1e12 / tf_sus,
                  "ms": kt["swa"] * 1e3}
    conv_bytes = T * s.d_inner * 4
    rep["conv"] = {"gbs": conv_bytes / kt["conv"] / 1e9, "ms": kt["conv"] * 1e3}
    rep["rmsnorm"] = {"gbs": T * s.d_model * 4 / kt["rmsnorm"] / 1e9, "ms": kt["rmsnorm"] * 1e3}
    rep["gemm"]["frac_of_" + src + "_burst_bf16_peak"] = g_flops / g_time / 1e12 / tf_burst
    # Dominant kernel: the SwiGLU up-projection (gemm_tc_kernel<2>, ~32% of the
    # step in the launch list).  Timed by CUDA events around each of its launches
    # inside the timed region (the library's timing hook), so against the
    # sustained peak; if the hook gave nothing usable, by the attribution pass
    # (the kernel alone), against the burst peak.  DRAM traffic per launch from an ncu capture of this kernel
    # at M = 16384 (dram__bytes_read.sum 201.9 MB, dram__bytes_write.sum 243.4 MB,
    # with the L2 eviction priorities and TMA-store epilogue of the current kernel), scaled to this M:
    # the activation reads and the output writes grow with M, the 67 MB of
    # weights are read once whatever M is.
    name = "mlp1_up"
    up = [fl for (n, M, N, K, e, fl) in gl if n == name][0]
    w_bytes = 2 * s.d_ff * s.d_model * 2
    scale = T / 16384
    # measured at the 2048-wide shapes only
    traffic = (201.9e6 - w_bytes) * scale + w_bytes + 243.4e6 * scale if s == I.WIDE else None
    t_alone = kt[name]
    live = t_up_live is not None and 0.5 * t_alone <= t_up_live[0] <= 2.0 * t_alone
    t_k, peak, kind = (t_up_live[0], tf_sus, "sustained") if live else (t_alone, tf_burst, "burst")
    achieved = up / t_k / 1e12
    note = None
    if achieved > peak and kind == "sustained":
        # the sustained figure was taken at a lower clock than this run's: it is
        # not this kernel's ceiling, so the burst figure is the denominator
        note = (f"the sustained bf16 figure ({tf_sus} TF/s) is below this kernel's measured rate; "
                f"the burst figure is used as the peak")
        peak, kind = tf_burst, "burst"
    run_mhz = (clocks or {}).get("sm_mhz")
    # per-clock comparison with a peak whose clock is known (the chosen peak's,
    # else the sustained figure's): (achieved / run MHz) / (peak / peak MHz)
    norm_kind = kind if peak_clock_mhz(kind) else "sustained"
    pk_mhz = peak_clock_mhz(norm_kind)
    pk_val = peak if norm_kind == kind else tf_sus
    frac_clk = (achieved / run_mhz) / (pk_val / pk_mhz) if (pk_mhz and run_mhz) else None
    roof = {"bound": "tensor", "achieved": round(achieved, 2), "peak": peak, "unit": "TFLOP/s",
            "frac": round(achieved / peak, 4), "traffic": round(traffic) if traffic else None,
            "frac_clock_normalised": round(frac_clk, 4) if frac_clk else None,
            "clock_normalisation": (f"(achieved / {run_mhz:.0f} MHz median SM clock of this run) / "
                                    f"({norm_kind} peak {pk_val} TF/s / {pk_mhz:.0f} MHz at which it was taken)")
            if frac_clk else "peak clock unknown",
            "denominator_note": note,
            "algorithmic_flops": up,
            "algorithmic_bytes": T * s.d_model * 2 + w_bytes + T * s.d_ff * 2,
            "kernel": "gemm_tc_kernel<2>: SwiGLU up-projection [T, d_model] x [2 d_ff, d_model]^T",
            "timing": (f"CUDA events around each of its {t_up_live[1]} launches inside the timed region"
                       if live else "attribution pass: the kernel alone, CUDA events"),
            "peak_source": src + (" sustained bf16 (kernel timed inside the long step)" if kind == "sustained"
                                  else " burst bf16"),
            "alone_tflops": round(up / t_alone / 1e12, 2),
            "traffic_source": "ncu dram__bytes_read.sum + dram__bytes_write.sum at M=16384, scaled to M"}
    return roof, rep


# ---------------------------------------------------------------------------
# the oracle (CPU baseline / reference arm)
# ---------------------------------------------------------------------------
def cpu_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [d.get("num_threads", 1) for d in threadpool_info() if d.get("user_api") == "blas"]
        return max(n) if n else os.cpu_count()
    except Exception:
        return os.cpu_count()


ORACLE_SAMPLE_LEN = 2304
_ORACLE_IN = {}


def oracle_sample(sample_len=ORACLE_SAMPLE_LEN):
    """fp64 oracle of one block at the workload's shapes on a bounded sample:
    batch 1, the first `sample_len` tokens of the sequence (2304: the last 256
    attend over the full 2048-key window).  Weights and input are drawn once
    per process, outside the timing.  Returns (tokens/s per block, desc)."""
    from oracle import samba_oracle as O
    shape = I.WORKLOADS[WORKLOAD][0]
    if sample_len not in _ORACLE_IN:
        _ORACLE_IN[sample_len] = (I.block_weights(shape, 2), I.block_input(shape, 2, 1, sample_len))
    W, x = _ORACLE_IN[sample_len]
    t0 = time.perf_counter()
    O.block_fwd(x, W, shape)
    dt = time.perf_counter() - t0
    return sample_len / dt, (f"1 block, batch 1, the first {sample_len} tokens of the L=131072 sequence "
                             f"(the last {sample_len - shape.window} at the full {shape.window}-key window); "
                             f"fp64 numpy, BLAS threads = cores")


def decode_bytes_per_step(s, Bn):
    """Algorithmic HBM bytes of one decode step: every weight once, the ring K/V
    read (full window), the SSM state read+written, the conv state read+written."""
    es = 2
    w = (2 * s.d_inner * s.d_model + (s.dt_rank + 2 * s.d_state) * s.d_inner + s.d_inner * s.dt_rank +
         s.d_model * s.d_inner + (s.n_q + 2 * s.n_kv) * s.head_dim * s.d_model + s.d_model * s.n_q * s.head_dim +
         2 * 3 * s.d_ff * s.d_model) * es
    ring = 2 * Bn * s.window * s.n_kv * s.head_dim * es
    ssm = 2 * Bn * s.d_inner * s.d_state * 4
    conv = 2 * Bn * s.d_inner * (s.d_conv - 1) * es
    return w + ring + ssm + conv


DECODE_STEPS = 65536


def measure_decode(steps, warmup, prefill=None):
    """Streaming decode at batch 32 (one block at the 2048-wide shapes, 2048-slot
    ring): prefill 4096 tokens, then `steps` replays of one captured samba_step.
    Returns the measurement as a dict (device time, end to end, roofline)."""
    import torch
    from sliding_window_attention_samba_b200 import _lib as L
    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    shape, Bn, P, _, seed = I.WORKLOADS["decode_bf16_B32"]
    if prefill:
        P = prefill  # profiling runs only: a shorter prefill keeps the device footprint small
    s = shape
    cfg = L.make_config(s)
    (w, wst), = make_stack(torch, L, s, 1, seed, dev)
    bf = torch.bfloat16
    ssm = torch.zeros(Bn, s.d_inner, s.d_state, device=dev)
    conv = torch.zeros(Bn, s.d_inner, s.d_conv - 1, device=dev, dtype=bf)
    kr = torch.zeros(Bn, s.window, s.n_kv, s.head_dim, device=dev, dtype=bf)
    vr = torch.zeros_like(kr)
    pos = torch.zeros(Bn, dtype=torch.int64, device=dev)
    st = L.make_state(ssm, conv, kr, vr, pos)
    ws_bytes = max(L.samba_block_workspace_size(cfg, Bn, P), L.samba_step_workspace_size(cfg, Bn))
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    g = torch.Generator(device=dev)
    g.manual_seed(I.tensor_key(seed, "decode.x") & ((1 << 63) - 1))
    x = torch.randn(Bn, P, s.d_model, generator=g, device=dev).to(bf)
    xo = torch.empty_like(x)
    L.samba_block_fwd(cfg, wst, x, xo, st, None, Bn, P, ws, ws_bytes)
    del x, xo
    xt = torch.randn(Bn, s.d_model, generator=g, device=dev).to(bf)
    yt = torch.empty_like(xt)
    stream = torch.cuda.Stream()
    stream.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(stream):
        L.samba_step(cfg, wst, xt, yt, st, Bn, ws, ws_bytes, stream=stream)  # first call outside capture
        graph = torch.cuda.CUDAGraph(keep_graph=True)
        with torch.cuda.graph(graph, stream=stream):
            L.samba_step(cfg, wst, xt, yt, st, Bn, ws, ws_bytes, stream=stream)
        nk = graph_kernel_nodes(graph)  # the step's kernel launches, read from the captured graph
        graph.instantiate()
        for _ in range(max(3, warmup)):
            graph.replay()
        stream.synchronize()
        assert L.samba_get_error(stream) == 0
        clocks = ClockSampler(0)
        clocks.start()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(steps):
            graph.replay()
        e1.record(stream)
        stream.synchronize()
        clk = clocks.stop()
        t = e0.elapsed_time(e1) * 1e-3
        # end to end: host token in, host token out, every step
        xh = xt.cpu().pin_memory()
        yh = torch.empty_like(xh).pin_memory()
        f0 = torch.cuda.Event(enable_timing=True)
        f1 = torch.cuda.Event(enable_timing=True)
        n_e2e = max(1, min(steps, 2000))
        f0.record(stream)
        for _ in range(n_e2e):
            xt.copy_(xh, non_blocking=True)
            graph.replay()
            yh.copy_(yt, non_blocking=True)
        f1.record(stream)
        stream.synchronize()
        t_e2e = f0.elapsed_time(f1) * 1e-3
    del graph
    assert L.samba_get_error() == 0
    hbm, _, _, src = load_peaks()
    bps = decode_bytes_per_step(s, Bn)
    per_step = t / steps
    return {"tokens_per_s": Bn * steps / t, "ms_per_step": per_step * 1e3, "steps": steps, "batch": Bn,
            "prefill": P, "window": s.window,
            "e2e": {"value": Bn * n_e2e / t_e2e, "unit": "tokens/s", "h2d_bytes_per_step": xh.numel() * 2,
                    "d2h_bytes_per_step": yh.numel() * 2, "steps": n_e2e},
            "roofline": {"bound": "hbm", "achieved": bps / per_step / 1e9, "peak": hbm, "unit": "GB/s",
                         "frac": bps / per_step / 1e9 / hbm, "traffic": None,
                         "kernel": "whole decode step (weights + ring + states per step)",
                         "peak_source": src, "bytes_per_step": bps},
            "clocks": clk, "graph": "one samba_step captured, replayed per step",
            # per step: the first RMSNorm (the other three ride on the
            # projections around them: the norm fold), 9 skinny projections
            # (in_proj with the conv step, x_proj, out_proj, QKV with RoPE and
            # the ring write, o_proj, 2 x SwiGLU up, 2 x down, the last
            # advancing the positions), the recurrence step with the dt
            # projection, the streaming attention: 12 launches; 15 with the
            # fold off (SAMBA_NORM_FOLD=0)
            "gpu_launches": (nk if nk else 12) * steps,
            "launches_per_step": {"value": nk if nk else 12, "source": "graph nodes" if nk else "claimed"}}


def run_decode(args):
    """Streaming decode: prefill P tokens at batch 32, then time samba_step replays."""
    d = measure_decode(args.steps, args.warmup, args.prefill)
    line = {"metric": "decode tokens/s (batch 32, one Samba block, 2048-slot ring)", "value": d["tokens_per_s"],
            "unit": "tokens/s", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": d["ms_per_step"], "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16", "data": "synthetic",
            "config": {"workload": "decode_bf16_B32", "batch": d["batch"], "prefill": d["prefill"],
                       "window": d["window"], "d_model": I.WIDE.d_model, "graph": d["graph"]},
            "e2e": d["e2e"], "roofline": d["roofline"], "clocks": d["clocks"], "gpu_launches": d["gpu_launches"],
            "launches_per_step": d["launches_per_step"]}
    print(json.dumps(line))


def run_chunked(args):
    """One block over a 1M-token sequence fed as 32K-token chunks, each continuing
    from the state the previous chunk left.  Device timing with the sequence
    resident; end to end streams every chunk from pinned host memory and back,
    so the device holds one chunk's input/output and workspace only.  For
    comparison, the same sequence in one samba_block_fwd call when it fits."""
    import torch
    from sliding_window_attention_samba_b200 import _lib as L
    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    wl = "chunked_prefill_bf16_L1048576"
    shape, Bn, Ln, _, seed = I.WORKLOADS[wl]
    if args.seq_len:
        Ln = args.seq_len
    C = min(I.CHUNKED_PREFILL_CHUNK, Ln)
    nch = (Ln + C - 1) // C
    s = shape
    cfg = L.make_config(s)
    (w, wst), = make_stack(torch, L, s, 1, seed, dev)
    bf = torch.bfloat16
    ssm = torch.zeros(Bn, s.d_inner, s.d_state, device=dev)
    conv = torch.zeros(Bn, s.d_inner, s.d_conv - 1, device=dev, dtype=bf)
    kr = torch.zeros(Bn, s.window, s.n_kv, s.head_dim, device=dev, dtype=bf)
    vr = torch.zeros_like(kr)
    pos = torch.zeros(Bn, dtype=torch.int64, device=dev)
    st = L.make_state(ssm, conv, kr, vr, pos)
    ws_bytes = L.samba_block_chunk_workspace_size(cfg, Bn, C)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    g = torch.Generator(device=dev)
    g.manual_seed(I.tensor_key(seed, "chunked.x") & ((1 << 63) - 1))
    x = torch.randn(Bn, Ln, s.d_model, generator=g, device=dev).to(bf)
    out = torch.empty_like(x)
    stream = torch.cuda.current_stream()

    def step():
        for c in range(nch):
            a, b = c * C, min(Ln, (c + 1) * C)
            L.samba_block_fwd_chunk(cfg, wst, x[:, a:b], out[:, a:b], st, a, None, Bn, b - a, ws, ws_bytes)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    assert L.samba_get_error() == 0, "device error during warm-up"
    clocks = ClockSampler(0)
    clocks.start()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    t_dev = e0.elapsed_time(e1) * 1e-3
    assert L.samba_get_error() == 0, "device error in the timed region"
    # end to end, streamed: chunk in from pinned host memory, chunk out to it
    xh = x.cpu().pin_memory()
    yh = torch.empty_like(xh).pin_memory()
    del x, out
    # two device chunk buffers each way; copies on their own stream overlap the
    # previous / next chunk's compute
    xc = [torch.empty(Bn, C, s.d_model, device=dev, dtype=bf) for _ in range(2)]
    yc = [torch.empty_like(xc[0]) for _ in range(2)]
    cps = torch.cuda.Stream()
    jobs = [(c * C, min(Ln, (c + 1) * C)) for _ in range(args.steps) for c in range(nch)]
    h2d = [torch.cuda.Event() for _ in jobs]
    done = [torch.cuda.Event() for _ in jobs]
    d2h = [torch.cuda.Event() for _ in jobs]
    torch.cuda.synchronize()
    f0 = torch.cuda.Event(enable_timing=True)
    f1 = torch.cuda.Event(enable_timing=True)
    f0.record(cps)

    def load(k):
        a, b = jobs[k]
        with torch.cuda.stream(cps):
            if k >= 2:
                cps.wait_event(done[k - 2])
            xc[k % 2][:, :b - a].copy_(xh[:, a:b], non_blocking=True)
            h2d[k].record(cps)

    load(0)
    for k, (a, b) in enumerate(jobs):
        if k + 1 < len(jobs):
            load(k + 1)
        stream.wait_event(h2d[k])
        if k >= 2:
            stream.wait_event(d2h[k - 2])
        L.samba_block_fwd_chunk(cfg, wst, xc[k % 2], yc[k % 2], st, a, None, Bn, b - a, ws, ws_bytes)
        done[k].record(stream)
        with torch.cuda.stream(cps):
            cps.wait_event(done[k])
            yh[:, a:b].copy_(yc[k % 2][:, :b - a], non_blocking=True)
            d2h[k].record(cps)
    f1.record(cps)
    torch.cuda.synchronize()
    t_e2e = f0.elapsed_time(f1) * 1e-3
    assert L.samba_get_error() == 0
    # one call over the whole sequence, if its workspace fits next to the rest
    one = None
    ws1 = L.samba_block_workspace_size(cfg, Bn, Ln)
    free, _ = torch.cuda.mem_get_info()
    if ws1 + 2 * xh.numel() * 2 + (4 << 30) < free:
        del ws
        ws_one = torch.empty(ws1, dtype=torch.uint8, device=dev)
        xd = xh.to(dev)
        yd = torch.empty_like(xd)
        L.samba_block_fwd(cfg, wst, xd, yd, None, None, Bn, Ln, ws_one, ws1)
        torch.cuda.synchronize()
        t_one = _time(torch, lambda: L.samba_block_fwd(cfg, wst, xd, yd, None, None, Bn, Ln, ws_one, ws1), 1,
                      max(1, args.steps))
        one = {"value": Bn * Ln / t_one, "unit": "tokens/s", "workspace_gb": ws1 / 1e9}
        del ws_one, xd, yd
    tok = Bn * Ln * args.steps
    line = {"metric": "chunked prefill tokens/s per Samba block at L=1M (32K-token chunks)", "value": tok / t_dev,
            "unit": "tokens/s", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": t_dev / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": wl, "batch": Bn, "seq_len": Ln, "chunk": C, "n_chunks": nch,
                       "workspace_gb": ws_bytes / 1e9, "d_model": s.d_model, "window": s.window,
                       "l2": "activations per chunk >> 126 MB L2; no flush needed"},
            "e2e": {"value": tok / t_e2e, "unit": "tokens/s", "h2d_bytes_per_step": xh.numel() * 2,
                    "d2h_bytes_per_step": yh.numel() * 2,
                    "mode": "each chunk copied in from pinned host memory and out again on a copy stream that "
                            "overlaps the neighbouring chunks' compute (double-buffered)"},
            "single_call": one, "clocks": clk, "gpu_launches": (21 * nch - 1) * args.steps}
    print(json.dumps(line))


def make_layers(torch, s, layout, seed, dev):
    """Random-init weights of a layout of sub-layers (N(0, 0.02) matrices, S4D-Real
    A, D = 1, Delta bias in [1e-3, 1e-1], unit norm gains); each dict holds only
    what its kind reads."""
    g = torch.Generator(device=dev)
    bf = torch.bfloat16
    out = []
    for li, kind in enumerate(layout):
        g.manual_seed(I.tensor_key(seed, f"model.L{li}") & ((1 << 63) - 1))

        def mat(o, i):
            return (torch.randn(o, i, generator=g, device=dev) * 0.02).to(bf)

        if kind == "mamba":
            w = {"norm0": torch.ones(s.d_model, device=dev), "W_in": mat(2 * s.d_inner, s.d_model),
                 "conv_w": torch.randn(s.d_inner, s.d_conv, generator=g, device=dev) * 0.02,
                 "W_x": mat(s.dt_rank + 2 * s.d_state, s.d_inner), "W_dt": mat(s.d_inner, s.dt_rank),
                 "dt_bias": torch.from_numpy(I.dt_bias_init(seed, f"model.L{li}.dt_bias", s.d_inner)).to(dev),
                 "A_log": torch.from_numpy(I.a_log_init(s.d_inner, s.d_state)).to(dev),
                 "D": torch.ones(s.d_inner, device=dev), "W_out": mat(s.d_model, s.d_inner)}
        elif kind == "swa":
            w = {"norm2": torch.ones(s.d_model, device=dev), "Wq": mat(s.n_q * s.head_dim, s.d_model),
                 "Wk": mat(s.n_kv * s.head_dim, s.d_model), "Wv": mat(s.n_kv * s.head_dim, s.d_model),
                 "Wo": mat(s.d_model, s.n_q * s.head_dim)}
        else:
            w = {"norm1": torch.ones(s.d_model, device=dev), "mlp1_W1": mat(s.d_ff, s.d_model),
                 "mlp1_W2": mat(s.d_ff, s.d_model), "mlp1_W3": mat(s.d_model, s.d_ff)}
        out.append(w)
    return out


def run_model(args):
    """Prompt processing of two stacks of the same width built from this
    library's kernels: the paper's Samba-1.7B layout (8 x [Mamba, MLP, Mamba,
    MLP, SWA, MLP]: 16 Mamba, 8 SWA, 24 MLP) and a GQA Transformer of the
    Llama-3-1.6B shape (24 x [attention over the whole prefix, MLP]), both with a
    32000-token vocabulary.  As in the pages' throughput protocol, every step
    processes 131072 prompt tokens: batch = 131072 / L for L = 4K .. 128K."""
    import dataclasses
    import torch
    from sliding_window_attention_samba_b200 import _lib as L
    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    s = I.WIDE
    vocab, total = 32000, 131072
    kind = {"mamba": L.LAYER_MAMBA, "mlp": L.LAYER_MLP, "swa": L.LAYER_SWA}
    samba_layout = ["mamba", "mlp", "mamba", "mlp", "swa", "mlp"] * 8
    tfm_layout = ["swa", "mlp"] * 24
    bf = torch.bfloat16
    g = torch.Generator(device=dev)
    g.manual_seed(7)
    common = {"emb": torch.randn(vocab, s.d_model, generator=g, device=dev).to(bf),
              "head": (torch.randn(vocab, s.d_model, generator=g, device=dev) * 0.02).to(bf),
              "gfin": torch.ones(s.d_model, device=dev)}
    stacks = {"samba": (samba_layout, make_layers(torch, s, samba_layout, 6, dev)),
              "transformer": (tfm_layout, make_layers(torch, s, tfm_layout, 7, dev))}
    n_params = {k: sum(t.numel() for w in ws for t in w.values()) + 2 * vocab * s.d_model
                for k, (_, ws) in stacks.items()}
    lens = [Ln for Ln in (4096, 16384, 65536, 131072) if Ln <= (args.seq_len or 131072)]
    ws_bytes = max(L.samba_model_workspace_size(
        L.make_model(L.make_config(s), [], [], common["emb"], common["gfin"], common["head"], vocab),
        total // Ln, Ln) for Ln in lens)
    wsp = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    results = []
    clocks = ClockSampler(0)
    clocks.start()
    for Ln in lens:
        Bn = total // Ln
        ids = torch.randint(0, vocab, (Bn, Ln), generator=g, device=dev, dtype=torch.int32)
        logits = torch.empty(Bn, vocab, device=dev, dtype=bf)
        row = {"seq_len": Ln, "batch": Bn}
        for name, (layout, ws_) in stacks.items():
            shape = s if name == "samba" else dataclasses.replace(s, window=Ln)  # full causal attention
            m = L.make_model(L.make_config(shape), [kind[k] for k in layout], ws_, common["emb"], common["gfin"],
                             common["head"], vocab)

            def run(m=m):
                L.samba_model_prefill(m, ids, logits, Bn, Ln, wsp, ws_bytes)

            t = _time(torch, run, 1, max(1, args.steps))
            row[name + "_tokens_per_s"] = Bn * Ln / t
            row[name + "_ms_per_step"] = t * 1e3
        row["ratio"] = row["samba_tokens_per_s"] / row["transformer_tokens_per_s"]
        results.append(row)
        print(json.dumps(dict(workload="prompt_processing", **row)))
    clk = clocks.stop()
    assert L.samba_get_error() == 0
    last = results[-1]
    print(json.dumps({"metric": f"prompt tokens/s, Samba-1.7B layout, L={last['seq_len']}",
                      "value": last["samba_tokens_per_s"], "unit": "tokens/s", "n_gpus": 1, "steps": args.steps,
                      "warmup": 1, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                      "dtype": "bf16", "data": "synthetic",
                      "config": {"workload": "prompt_processing_128K_tokens", "d_model": s.d_model,
                                 "vocab": vocab, "samba_layers": "8 x [Mamba, MLP, Mamba, MLP, SWA, MLP]",
                                 "transformer_layers": "24 x [GQA attention (full causal), MLP]",
                                 "params": n_params, "tokens_per_step": total},
                      "transformer_value": last["transformer_tokens_per_s"], "ratio": last["ratio"],
                      "by_length": results, "clocks": clk}))


def run_model_decode(args):
    """Decode throughput of the two stacks of run_model at batch 16 (the pages'
    generation protocol: 64K generated tokens).  Samba's step cost does not
    depend on the context; the Transformer's attention reads its whole KV cache.
    One step is captured in a CUDA graph and replayed at contexts P = 0, 2K, 8K,
    16K, 32K, 64K (the cache holds P valid entries; its values do not change the
    work), and the time to generate 64K tokens is the trapezoid over P."""
    import dataclasses
    import torch
    from sliding_window_attention_samba_b200 import _lib as L
    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    s = I.WIDE
    vocab, Bn, gen = 32000, 16, 65536
    bf = torch.bfloat16
    kind = {"mamba": L.LAYER_MAMBA, "mlp": L.LAYER_MLP, "swa": L.LAYER_SWA}
    g = torch.Generator(device=dev)
    g.manual_seed(8)
    common = {"emb": torch.randn(vocab, s.d_model, generator=g, device=dev).to(bf),
              "head": (torch.randn(vocab, s.d_model, generator=g, device=dev) * 0.02).to(bf),
              "gfin": torch.ones(s.d_model, device=dev)}
    cache = gen + 256
    setups = {"samba": (["mamba", "mlp", "mamba", "mlp", "swa", "mlp"] * 8, s),
              "transformer": (["swa", "mlp"] * 24, dataclasses.replace(s, window=cache))}
    points = [0, 2048, 8192, 16384, 32768, gen - 1]
    reps = max(10, args.steps)
    out = {}
    clocks = ClockSampler(0)
    clocks.start()
    for name, (layout, shape) in setups.items():
        ws_layers = make_layers(torch, shape, layout, 9 if name == "samba" else 10, dev)
        m = L.make_model(L.make_config(shape), [kind[k] for k in layout], ws_layers, common["emb"], common["gfin"],
                         common["head"], vocab)
        states = []
        for k in layout:
            d = {}
            if k == "mamba":
                d["ssm"] = torch.zeros(Bn, s.d_inner, s.d_state, device=dev)
                d["conv"] = torch.zeros(Bn, s.d_inner, s.d_conv - 1, device=dev, dtype=bf)
            elif k == "swa":
                d["k_ring"] = torch.randn(Bn, shape.window, s.n_kv, s.head_dim, generator=g, device=dev).to(bf)
                d["v_ring"] = torch.randn_like(d["k_ring"].float()).to(bf)
            states.append(d)
        st_arr = L.make_layer_states(states)
        pos = torch.zeros(Bn, dtype=torch.int64, device=dev)
        ids_t = torch.randint(0, vocab, (Bn,), generator=g, device=dev, dtype=torch.int32)
        logits = torch.empty(Bn, vocab, device=dev, dtype=bf)
        n = L.samba_model_step_workspace_size(m, Bn)
        wsp = torch.empty(n, dtype=torch.uint8, device=dev)
        stream = torch.cuda.Stream()
        stream.wait_stream(torch.cuda.current_stream())
        per = {}
        with torch.cuda.stream(stream):
            L.samba_model_step(m, ids_t, logits, st_arr, pos, Bn, wsp, n, stream=stream)
            graph = torch.cuda.CUDAGraph(keep_graph=True)
            with torch.cuda.graph(graph, stream=stream):
                L.samba_model_step(m, ids_t, logits, st_arr, pos, Bn, wsp, n, stream=stream)
            nk = graph_kernel_nodes(graph)
            graph.instantiate()
            for P in points:
                pos.fill_(P)
                for _ in range(3):
                    graph.replay()
                pos.fill_(P)
                e0 = torch.cuda.Event(enable_timing=True)
                e1 = torch.cuda.Event(enable_timing=True)
                e0.record(stream)
                for _ in range(reps):
                    graph.replay()
                e1.record(stream)
                stream.synchronize()
                per[P] = e0.elapsed_time(e1) * 1e-3 / reps
        del graph
        assert L.samba_get_error(stream) == 0
        t_gen = sum((points[i + 1] - points[i]) * (per[points[i]] + per[points[i + 1]]) / 2
                    for i in range(len(points) - 1))
        out[name] = {"step_ms_at_context": {str(P): round(per[P] * 1e3, 4) for P in points},
                     "tokens_per_s_64K_generation": Bn * gen / t_gen, "launches_per_step": nk,
                     "params": sum(t.numel() for w in ws_layers for t in w.values()) + 2 * vocab * s.d_model}
        del states, st_arr, ws_layers, wsp
        torch.cuda.empty_cache()
    clk = clocks.stop()
    sv, tv = out["samba"]["tokens_per_s_64K_generation"], out["transformer"]["tokens_per_s_64K_generation"]
    print(json.dumps({"metric": "decode tokens/s over 64K generated tokens, batch 16, Samba-1.7B layout",
                      "value": sv, "unit": "tokens/s", "n_gpus": 1, "steps": reps, "warmup": 3,
                      "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
                      "data": "synthetic",
                      "config": {"workload": "decode_batch16_64K", "batch": Bn, "generated": gen, "vocab": vocab,
                                 "samba_layers": "8 x [Mamba, MLP, Mamba, MLP, SWA, MLP], 2048-slot rings",
                                 "transformer_layers": f"24 x [GQA attention, MLP], {cache}-slot KV cache",
                                 "graph": "one samba_model_step captured, replayed per step"},
                      "transformer_value": tv, "ratio": sv / tv, "by_model": out, "clocks": clk}))


def measure_sweep(warmup, max_len):
    """Mixer-only length sweep, batch 1, d_model 2048 shapes: the selective scan
    (d_inner 4096, d_state 16; u, dt, z, B, C ~ N(0,1), Delta = softplus(dt + b))
    and SWA (32/4 heads of 64, window 2048, RoPE) timed separately per L.
    Returns one dict per L."""
    import torch
    from sliding_window_attention_samba_b200 import _lib as L
    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    hbm, tf_burst, _, src = load_peaks()
    bf = torch.bfloat16
    D, N, Hq, Hkv, hd, w = 4096, 16, 32, 4, 64, 2048
    A_log = torch.from_numpy(I.a_log_init(D, N)).to(dev)
    dtb = torch.from_numpy(I.dt_bias_init(3, "scan.dt_bias", D)).to(dev)
    Dk = torch.ones(D, device=dev)
    g = torch.Generator(device=dev)
    g.manual_seed(I.tensor_key(I.MIXER_SWEEP_SEED, "sweep") & ((1 << 63) - 1))
    rows = []
    for Ln in I.MIXER_SWEEP_L:
        if Ln > max_len:
            break
        u = torch.randn(1, Ln, D, generator=g, device=dev).to(bf)
        dt = torch.randn(1, Ln, D, generator=g, device=dev).to(bf)
        z = torch.randn(1, Ln, D, generator=g, device=dev).to(bf)
        Bm = torch.randn(1, Ln, N, generator=g, device=dev).to(bf)
        Cm = torch.randn(1, Ln, N, generator=g, device=dev).to(bf)
        y = torch.empty_like(u)
        hT = torch.empty(1, D, N, device=dev)

        def scan():
            L.samba_selective_scan(u, dt, dtb, 1, A_log, Bm, Cm, Dk, z, None, hT, y, 1, Ln, D, N, 1)
        reps = max(3, min(20, (1 << 22) // Ln))
        t_scan = _time(torch, scan, warmup, reps)
        del u, dt, z, y
        q = torch.randn(1, Ln, Hq, hd, generator=g, device=dev).to(bf)
        k = torch.randn(1, Ln, Hkv, hd, generator=g, device=dev).to(bf)
        v = torch.randn(1, Ln, Hkv, hd, generator=g, device=dev).to(bf)
        o = torch.empty_like(q)
        wsn = L.samba_swa_workspace_size(1, Ln, Hq, Hkv, hd, 10000.0, 1)
        ws = torch.empty(wsn, dtype=torch.uint8, device=dev)

        def swa():
            L.samba_swa_fwd(q, k, v, o, 1, Ln, Hq, Hkv, hd, w, 10000.0, 0, 0.0, 1, ws, wsn)
        t_swa = _time(torch, swa, warmup, reps)

        def swa_kernel():  # the attention kernel alone (RoPE off: no table, no rotation pass)
            L.samba_swa_fwd(q, k, v, o, 1, Ln, Hq, Hkv, hd, w, 0.0, 0, 0.0, 1, ws, wsn)
        t_swak = _time(torch, swa_kernel, warmup, reps)
        del q, k, v, o, ws
        torch.cuda.empty_cache()
        assert L.samba_get_error() == 0
        sb = Ln * (8 * D + 4 * N)
        sf = swa_flops(I.WIDE, 1, Ln)
        rows.append({"seq_len": Ln, "reps": reps,
                     "scan": {"ms": t_scan * 1e3, "gbs": sb / t_scan / 1e9,
                              "frac_of_" + src + "_hbm": sb / t_scan / 1e9 / hbm, "tokens_per_s": Ln / t_scan,
                              "includes": "softplus(dt + bias) in the kernel"},
                     "swa": {"ms": t_swa * 1e3, "tflops": sf / t_swa / 1e12,
                             "frac_of_" + src + "_bf16_burst": sf / t_swa / 1e12 / tf_burst,
                             "tokens_per_s": Ln / t_swa, "includes": "RoPE of q and k (standalone entry)",
                             "kernel_ms": t_swak * 1e3, "kernel_tflops": sf / t_swak / 1e12,
                             "kernel_frac_of_" + src + "_bf16_burst": sf / t_swak / 1e12 / tf_burst}})
    return rows


def run_sweep(args):
    for r in measure_sweep(args.warmup, args.max_len):
        print(json.dumps({"workload": "mixer_sweep", "dtype": "bf16", **r}))


def _time(torch, fn, warmup, reps):
    for _ in range(max(1, warmup)):
        fn()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(reps):
        fn()
    e1.record()
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) * 1e-3 / reps


def main():
    args = parse()
    if args.workload == "decode":
        return run_decode(args)
    if args.workload == "sweep":
        return run_sweep(args)
    if args.workload == "chunked":
        return run_chunked(args)
    if args.workload == "model":
        return run_model(args)
    if args.workload == "model_decode":
        return run_model_decode(args)
    rank = int(os.environ.get("RANK", 0))
    world = int(os.environ.get("WORLD_SIZE", 1))
    local_rank = int(os.environ.get("LOCAL_RANK", 0))
    shape, Bn, Ln, n_blocks, _ = I.WORKLOADS[workload_of(args)]
    if args.seq_len:
        Ln = args.seq_len
    cfgd = {"workload": workload_of(args), "weights": "random init", "global_batch": Bn * max(world, 1),
            "seq_len": Ln, "n_blocks": n_blocks, "d_model": shape.d_model, "window": shape.window,
            "parallelism": f"replicas{max(world, 1)}", "l2": "activations per block >> 126 MB L2; no flush needed"}

    if args.impl == "reference":
        if rank != 0:
            return
        vals = []
        for i in range(args.warmup + args.steps):
            v, desc = oracle_sample()
            if i >= args.warmup:
                vals.append(v)
        v = statistics.mean(vals)
        print(json.dumps({"impl": "reference", "metric": METRIC, "value": v, "unit": UNIT, "n_gpus": args.gpus,
                          "steps": args.steps, "warmup": args.warmup, "higher_is_better": True, "scaling": "weak",
                          "vs_baseline": None, "dtype": "f64", "data": "synthetic", "config": cfgd,
                          "cpu_baseline": {"value": v, "unit": UNIT, "cores": cpu_threads(), "kind": "oracle",
                                           "sample": desc},
                          "e2e": {"value": v, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}))
        return

    if world > 1:
        import torch
        import torch.distributed as dist
        import datetime
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    r = run_cuda(args, rank, world, local_rank)
    peaks = load_peaks()
    if rank == 0:
        value = replica_throughput(Bn * Ln, world, r["t_dev"], args.steps, n_blocks)
        e2e = replica_throughput(Bn * Ln, world, r["t_e2e"], args.steps, n_blocks)
        roof, rep = kernel_report(r["kt"], r["s"], Bn * Ln, Bn, Ln, peaks, r.get("t_up_live"), r["clocks"])
        cpu = None
        if not args.no_cpu_baseline:
            v, desc = oracle_sample()
            cpu = {"value": v, "unit": UNIT, "cores": cpu_threads(), "kind": "oracle", "sample": desc}
        extra = {}
        if world == 1 and not args.no_extras:
            # the other single-GPU figures of the metric: decode at batch 32
            # (65 536 graph-replayed steps) and the mixer sweep L = 4K .. 1M
            import torch
            torch.cuda.empty_cache()
            extra["decode"] = measure_decode(DECODE_STEPS, args.warmup)
            torch.cuda.empty_cache()
            extra["sweep"] = measure_sweep(args.warmup, args.max_len)
        # norms, projections (the dt projection inside the scan when folded), conv, scan, rope table, swa
        launches_per_block = 4 + (9 if dt_folded(shape) else 10) + 1 + 1 + 1 + 1
        metric = {"prefill": METRIC, "block": "prefill tokens/s per Samba block (B=4, L=4096)",
                  "block38": "prefill tokens/s per Samba block at the 3.8B widths (L=128K)"}[args.workload]
        line = {"metric": metric,
                "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": r["t_dev"] / args.steps * 1e3, "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic", "config": cfgd,
                "e2e": {"value": e2e, "unit": UNIT, "h2d_bytes_per_step": r["h2d"], "d2h_bytes_per_step": r["d2h"],
                        "mode": "pinned host input in and output out every step, on a copy stream overlapping "
                                "the previous/next step's compute (double-buffered)"},
                "roofline": roof, "kernels": rep, "cpu_baseline": cpu, "clocks": r["clocks"],
                "gpu_launches": launches_per_block * n_blocks * args.steps, **extra}
        print(json.dumps(line))
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
