"""The bench's algorithmic work figures (the roofline numerators), checked on
CPU against independent counts: a projection's FLOPs per token are twice its
weight parameters; the banded attention's score count is a direct sum over
queries; the decode step's bytes are the byte sizes of the tensors it streams."""
import numpy as np
import pytest

import bench
from sliding_window_attention_samba_b200 import inputs as I


def block_projection_params(s):
    """Weight parameters of every projection of one block, from the layer list."""
    mats = {
        "in_proj (W_in | W_g)": (2 * s.d_inner, s.d_model),
        "x_proj": (s.dt_rank + 2 * s.d_state, s.d_inner),
        "dt_proj": (s.d_inner, s.dt_rank),
        "out_proj": (s.d_model, s.d_inner),
        "mlp1 W1, W2": (2 * s.d_ff, s.d_model),
        "mlp1 W3": (s.d_model, s.d_ff),
        "Wq": (s.n_q * s.head_dim, s.d_model),
        "Wk": (s.n_kv * s.head_dim, s.d_model),
        "Wv": (s.n_kv * s.head_dim, s.d_model),
        "Wo": (s.d_model, s.n_q * s.head_dim),
        "mlp2 W1, W2": (2 * s.d_ff, s.d_model),
        "mlp2 W3": (s.d_model, s.d_ff),
    }
    return sum(a * b for a, b in mats.values())


@pytest.mark.parametrize("shape", [I.WIDE, I.WIDE38, I.TINY])
def test_gemm_flops_are_twice_the_parameters_per_token(shape):
    T = 4096
    total = sum(fl for (*_r, fl) in bench.gemm_list(shape, T))
    assert total == 2 * block_projection_params(shape) * T


def test_block_flops_per_token_at_2048_wide():
    # 136.4 M projection parameters: 272.9 MFLOP per token
    per_token = sum(fl for (*_r, fl) in bench.gemm_list(I.WIDE, 1))
    assert per_token == pytest.approx(272.9e6, rel=1e-3)


@pytest.mark.parametrize("L", [1, 5, 64, 300])
def test_swa_flops_brute_force_band(L):
    s = I.TINY  # window 64
    pairs = sum(min(t + 1, s.window) for t in range(L))  # keys each query sees
    assert bench.swa_flops(s, 2, L) == 4.0 * s.head_dim * s.n_q * pairs * 2


def test_swa_flops_headline():
    assert bench.swa_flops(I.WIDE, 1, 131072) == pytest.approx(2.18e12, rel=2e-3)


def test_decode_bytes_per_step_from_tensor_sizes():
    s, B = I.WIDE, 32
    bf16, f32 = 2, 4
    weights = block_projection_params(s) * bf16
    ring = 2 * B * s.window * s.n_kv * s.head_dim * bf16           # K and V, whole window read
    ssm = 2 * B * s.d_inner * s.d_state * f32                       # read and written
    conv = 2 * B * s.d_inner * (s.d_conv - 1) * bf16               # read and written
    assert bench.decode_bytes_per_step(s, B) == weights + ring + ssm + conv
    assert bench.decode_bytes_per_step(s, B) == pytest.approx(358e6, rel=5e-3)


def test_scan_bytes_per_token():
    # u, Delta, z in and y out (bf16, d_inner each) plus B and C (bf16, d_state each)
    s = I.WIDE
    assert 4 * s.d_inner * 2 + 2 * s.d_state * 2 == 32832


def test_replica_throughput_counts_all_ranks():
    assert bench.replica_throughput(131072, 4, 2.0, 10, 4) == pytest.approx(4 * 131072 * 10 * 4 / 2.0)
    assert np.isclose(bench.replica_throughput(1, 1, 1.0, 1, 1), 1.0)


def test_graph_kernel_nodes_without_a_graph_is_unknown():
    """The decode lines' launch count comes from the captured graph's kernel
    nodes; where the handle cannot be read (no GPU, no graph kept) the helper
    reports None and the line falls back to its stated count instead of
    inventing one."""
    class NoGraph:
        def raw_cuda_graph(self):
            raise RuntimeError("keep_graph was not set")
    assert bench.graph_kernel_nodes(NoGraph()) is None
