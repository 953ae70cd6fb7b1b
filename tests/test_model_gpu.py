"""Language-model stack (samba_model_prefill): token embedding, a layout of
Mamba / MLP / SWA sub-layers, final RMSNorm and the vocabulary projection of
the last position, against the fp64 oracle.  Layouts: the paper's 2:1 pattern
(Mamba, MLP, Mamba, MLP, SWA, MLP), and a GQA Transformer as (attention with a
window >= L, MLP) pairs."""
import dataclasses

import numpy as np
import pytest

from oracle import samba_oracle as O
from sliding_window_attention_samba_b200 import inputs as I
from tests.helpers import TOL, block_weights_dev, dev, host, path_err, rel_err

pytestmark = pytest.mark.gpu

KIND = {"mamba": 0, "mlp": 1, "swa": 2}
SAMBA_2_1 = ["mamba", "mlp", "mamba", "mlp", "swa", "mlp"]


@pytest.fixture(scope="module")
def L():
    import torch
    from sliding_window_attention_samba_b200 import _lib
    torch.cuda.init()
    return _lib


def _run(L, shape, layout, Bn, Ln, vocab, seed):
    import torch
    layers = [I.block_weights(shape, seed, layer=i) for i in range(len(layout))]
    emb = I.draw_normal(seed, "model.emb", (vocab, shape.d_model), 1.0, shape.dtype)
    head = I.draw_normal(seed, "model.head", (vocab, shape.d_model), 0.02, shape.dtype)
    gfin = I.draw_normal(seed, "model.gfin", (shape.d_model,), 1.0, "f32")
    ids = (I.uniforms(I.tensor_key(seed, "model.ids"), 0, Bn * Ln) * vocab).astype(np.int64).reshape(Bn, Ln)
    ids = np.minimum(ids, vocab - 1)
    ref = O.model_prefill(ids, list(zip(layout, layers)), emb, gfin, head, shape)
    dt = shape.dtype
    keep = [block_weights_dev(W, dt) for W in layers]  # the structs hold raw pointers: keep every tensor alive
    emb_d, gfin_d, head_d = dev(emb, dt), dev(gfin), dev(head, dt)
    m = L.make_model(L.make_config(shape), [KIND[k] for k in layout], keep, emb_d, gfin_d, head_d, vocab)
    n = L.samba_model_workspace_size(m, Bn, Ln)
    ws = torch.empty(n, dtype=torch.uint8, device="cuda")
    ids_d = torch.from_numpy(ids.astype(np.int32)).cuda()
    logits = torch.empty(Bn, vocab, device="cuda", dtype=torch.bfloat16 if dt == "bf16" else torch.float32)
    L.samba_model_prefill(m, ids_d, logits, Bn, Ln, ws, n)
    torch.cuda.synchronize()
    assert L.samba_get_error() == 0
    return host(logits), ref


def test_samba_2to1_stack_tiny_f32(L):
    got, ref = _run(L, I.TINY, SAMBA_2_1 * 2, 2, 150, 97, 21)  # past the 64-token window
    assert rel_err(got, ref) <= TOL["f32"]


def test_transformer_layout_full_attention_tiny_f32(L):
    Ln = 150
    shape = dataclasses.replace(I.TINY, window=Ln)  # window >= L: full causal attention
    got, ref = _run(L, shape, ["swa", "mlp"] * 3, 2, Ln, 64, 22)
    assert rel_err(got, ref) <= TOL["f32"]


def test_samba_2to1_stack_wide_bf16(L):
    got, ref = _run(L, I.WIDE, SAMBA_2_1, 1, 2304, 512, 23)
    assert path_err(got, ref, "bf16") <= TOL["bf16"]
    assert int(np.argmax(got[0])) == int(np.argmax(ref[0]))


def test_out_of_range_token_id_sets_device_error(L):
    import torch
    shape = I.TINY
    W = I.block_weights(shape, 24)
    Wd = block_weights_dev(W, "f32")
    emb, head = dev(np.ones((10, shape.d_model), np.float32)), dev(np.ones((10, shape.d_model), np.float32))
    g = dev(np.ones(shape.d_model, np.float32))
    m = L.make_model(L.make_config(shape), [1], [Wd], emb, g, head, 10)
    n = L.samba_model_workspace_size(m, 1, 4)
    ws = torch.empty(n, dtype=torch.uint8, device="cuda")
    ids = torch.tensor([[1, 2, 10, 3]], dtype=torch.int32, device="cuda")
    logits = torch.empty(1, 10, device="cuda")
    L.samba_model_prefill(m, ids, logits, 1, 4, ws, n)
    torch.cuda.synchronize()
    assert L.samba_get_error() == L.SAMBA_ERR_DEVICE
    assert L.samba_get_error() == 0


class GpuModel:
    """Device weights, model struct and per-layer decode states of a layout."""

    def __init__(self, L_, shape, layout, vocab, seed, Bn):
        import torch
        self.L, self.shape, self.layout, self.vocab, self.Bn = L_, shape, layout, vocab, Bn
        dt = shape.dtype
        self.tdt = torch.bfloat16 if dt == "bf16" else torch.float32
        self.W = [I.block_weights(shape, seed, layer=i) for i in range(len(layout))]
        self.emb = I.draw_normal(seed, "model.emb", (vocab, shape.d_model), 1.0, dt)
        self.head = I.draw_normal(seed, "model.head", (vocab, shape.d_model), 0.02, dt)
        self.gfin = I.draw_normal(seed, "model.gfin", (shape.d_model,), 1.0, "f32")
        self.keep = [block_weights_dev(W, dt) for W in self.W]
        self.emb_d, self.gfin_d, self.head_d = dev(self.emb, dt), dev(self.gfin), dev(self.head, dt)
        self.m = L_.make_model(L_.make_config(shape), [KIND[k] for k in layout], self.keep, self.emb_d, self.gfin_d,
                               self.head_d, vocab)
        s = shape
        self.states = []
        for k in layout:
            d = {}
            if k == "mamba":
                d["ssm"] = torch.zeros(Bn, s.d_inner, s.d_state, device="cuda")
                d["conv"] = torch.zeros(Bn, s.d_inner, s.d_conv - 1, device="cuda", dtype=self.tdt)
            elif k == "swa":
                d["k_ring"] = torch.zeros(Bn, s.window, s.n_kv, s.head_dim, device="cuda", dtype=self.tdt)
                d["v_ring"] = torch.zeros_like(d["k_ring"])
            self.states.append(d)
        self.st = L_.make_layer_states(self.states)
        self.pos = torch.zeros(Bn, dtype=torch.int64, device="cuda")
        n = L_.samba_model_step_workspace_size(self.m, Bn)
        self.ws = torch.empty(n, dtype=torch.uint8, device="cuda")
        self.ids_t = torch.zeros(Bn, dtype=torch.int32, device="cuda")
        self.logits = torch.empty(Bn, vocab, device="cuda", dtype=self.tdt)

    def step(self, ids_col, stream=None):
        import torch
        self.ids_t.copy_(torch.from_numpy(ids_col.astype(np.int32)))
        self.L.samba_model_step(self.m, self.ids_t, self.logits, self.st, self.pos, self.Bn, self.ws,
                                self.ws.numel(), stream=stream)

    def oracle(self, ids):
        return O.model_prefill(ids, list(zip(self.layout, self.W)), self.emb, self.gfin, self.head, self.shape)


def _ids(seed, Bn, Ln, vocab):
    ids = (I.uniforms(I.tensor_key(seed, "model.ids"), 0, Bn * Ln) * vocab).astype(np.int64).reshape(Bn, Ln)
    return np.minimum(ids, vocab - 1)


def test_model_step_equals_prefill_tiny_f32(L):
    """Decoding token by token from empty states gives, at every step, the
    prefill logits of the prefix (2:1 stack, past the 64-slot ring)."""
    Bn, S, vocab = 2, 80, 97
    g = GpuModel(L, I.TINY, SAMBA_2_1, vocab, 31, Bn)
    ids = _ids(31, Bn, S, vocab)
    check = {0, 1, 5, 63, 64, 79}
    for t in range(S):
        g.step(ids[:, t])
        if t in check:
            assert rel_err(host(g.logits), g.oracle(ids[:, :t + 1])) <= TOL["f32"], t
    assert np.array_equal(host(g.pos), np.full(Bn, S))


def test_model_step_full_cache_split_attention_bf16(L):
    """A Transformer layout with a 4096-slot full KV cache (the split decode
    attention over 256-slot slices, merged from the workspace) against prefill."""
    import dataclasses
    shape = dataclasses.replace(I.WIDE, window=4096)
    Bn, S, vocab = 2, 700, 256
    g = GpuModel(L, shape, ["swa", "mlp"], vocab, 32, Bn)
    ids = _ids(32, Bn, S, vocab)
    for t in range(S):
        g.step(ids[:, t])
        if t in (0, 255, 256, 511, 699):
            assert path_err(host(g.logits), g.oracle(ids[:, :t + 1]), "bf16") <= TOL["bf16"], t


def test_model_step_norm_fold_on_off_wide_bf16(L, monkeypatch):
    """The decode norm fold over a whole 2:1 stack (every norm after the first
    sub-layer's, the final one included, completed by the projections around
    it) against the plain norm launches (SAMBA_NORM_FOLD=0): both against the
    oracle's prefill of every prefix, close to each other, and the folded steps
    bit-reproducible from the same states."""
    import torch
    Bn, S, vocab = 3, 6, 264
    g = GpuModel(L, I.WIDE, SAMBA_2_1, vocab, 34, Bn)
    ids = _ids(34, Bn, S, vocab)
    tensors = [t for d in g.states for t in d.values()] + [g.pos]
    s0 = [t.clone() for t in tensors]

    def run():
        for t_, s_ in zip(tensors, s0):
            t_.copy_(s_)
        out = []
        for t in range(S):
            g.step(ids[:, t])
            out.append(g.logits.clone())
        torch.cuda.synchronize()
        assert L.samba_get_error() == 0
        return out
    folded, again = run(), run()
    monkeypatch.setenv("SAMBA_NORM_FOLD", "0")
    plain = run()
    for t in range(S):
        assert torch.equal(folded[t], again[t]), t
        if t in (0, 2, S - 1):
            ref = g.oracle(ids[:, :t + 1])
            for y in (folded[t], plain[t]):
                assert path_err(host(y), ref, "bf16") <= TOL["bf16"], t
        d = float((folded[t].float() - plain[t].float()).norm() / plain[t].float().norm())
        assert d <= 1e-2, (t, d)


def test_model_step_graph_replay_bit_exact(L):
    import torch
    Bn, vocab = 3, 50
    g = GpuModel(L, I.TINY, SAMBA_2_1, vocab, 33, Bn)
    ids = _ids(33, Bn, 12, vocab)
    snap = lambda: [t.clone() for d in g.states for t in d.values()] + [g.pos.clone()]
    tensors = [t for d in g.states for t in d.values()] + [g.pos]
    g.step(ids[:, 0])  # first call outside capture
    torch.cuda.synchronize()
    s0 = snap()
    eager = []
    for t in range(1, 12):
        g.step(ids[:, t])
        eager.append(g.logits.clone())
    for t_, s_ in zip(tensors, s0):
        t_.copy_(s_)
    st = torch.cuda.Stream()
    st.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(st):
        gr = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gr, stream=st):
            g.L.samba_model_step(g.m, g.ids_t, g.logits, g.st, g.pos, Bn, g.ws, g.ws.numel(), stream=st)
    torch.cuda.current_stream().wait_stream(st)
    for t_, s_ in zip(tensors, s0):
        t_.copy_(s_)
    for t in range(1, 12):
        g.ids_t.copy_(torch.from_numpy(ids[:, t].astype(np.int32)))
        gr.replay()
        torch.cuda.synchronize()
        assert torch.equal(g.logits, eager[t - 1]), t
