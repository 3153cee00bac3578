"""The seeded synthetic inputs follow their stated recipe: shapes, dtypes, draw
order, spreads and determinism; the latency models give each workload its
stated item weights and budget grid.  CPU only (the large shapes are checked
through their latency side; their draw uses the same code as the small shapes)."""
import math

import pytest
import torch

from knapsack_layer_selection_b200 import workloads as W
from oracle import ks_oracle as O


@pytest.mark.parametrize("name,ctx,w_attn,w_mlp,K", [
    ("tiny", None, 4, 3, 28),
    ("small", None, 11, 5, 256),
    ("llama3_8b_8k", None, 14, 2, 512),
    ("llama3_8b_32k", 4096, 26, 6, 1024),
    ("llama3_8b_32k", 16384, 30, 2, 1024),
    ("llama3_8b_32k", 32768, 31, 1, 1024),
    ("qwen3_32b_16k", None, 15, 1, 1024),
])
def test_item_weights_and_grid_per_workload(name, ctx, w_attn, w_mlp, K):
    wl = W.WORKLOADS[name]
    w = O.quantize_weights(wl.latencies(ctx), wl.n_bins)
    assert w == [w_attn, w_mlp] * wl.n_layers
    assert sum(w) == K


def test_every_workload_is_listed_once_and_runs_on_the_tensor_core_tiles():
    assert sorted(W.WORKLOAD_ORDER) == sorted(W.WORKLOADS)
    for wl in W.WORKLOADS.values():
        assert wl.n_q_heads % wl.n_kv_heads == 0 and wl.head_dim in (64, 128)
        if wl.wdtype == "bf16":
            assert wl.d_model % 256 == 0 and wl.q_dim % 256 == 0 and wl.ffn % 128 == 0


@pytest.mark.parametrize("name", ["tiny", "small"])
def test_inputs_follow_the_recipe(name):
    wl = W.WORKLOADS[name]
    inp = W.make_inputs(wl)
    dt = W.torch_dtype(wl)
    d, qd, F = wl.d_model, wl.q_dim, wl.ffn
    shapes = {"wq": (qd, d), "wo": (d, qd), "w_gate": (F, d), "w_up": (F, d), "w_down": (d, F),
              "attn_norm": (d,), "mlp_norm": (d,)}
    assert len(inp.layers) == wl.n_layers
    for L in inp.layers:
        assert {k: tuple(v.shape) for k, v in L.items()} == shapes
        assert all(v.dtype == dt for v in L.values())
        assert torch.equal(L["attn_norm"], torch.ones(d, dtype=dt))
        assert torch.equal(L["mlp_norm"], torch.ones(d, dtype=dt))
    kv = (wl.n_layers, wl.ctx + wl.T, wl.n_kv_heads, wl.head_dim)
    assert tuple(inp.k_cache.shape) == kv and tuple(inp.v_cache.shape) == kv
    assert inp.k_cache.dtype == dt and inp.x0.dtype == torch.float32
    assert tuple(inp.x0.shape) == (wl.T, d)
    # spreads: linear weights 0.02, cache 0.02 sqrt(d), x0 1 (within sampling error)
    wq = inp.layers[0]["wq"].float()
    assert abs(wq.std().item() / 0.02 - 1) < 0.02 and abs(wq.mean().item()) < 1e-3
    assert abs(inp.k_cache.float().std().item() / (0.02 * math.sqrt(d)) - 1) < 0.02
    assert abs(inp.x0.std().item() - 1) < 0.15


def test_draw_order_and_determinism():
    wl = W.WORKLOADS["tiny"]
    a, b = W.make_inputs(wl), W.make_inputs(wl)
    for La, Lb in zip(a.layers, b.layers):
        assert all(torch.equal(La[k], Lb[k]) for k in La)
    assert torch.equal(a.k_cache, b.k_cache) and torch.equal(a.x0, b.x0)
    c = W.make_inputs(wl, seed=1)
    assert not torch.equal(a.x0, c.x0)
    # one generator, drawn in the stated order: layer 0's Wq comes first, x0 last
    g = torch.Generator().manual_seed(0)
    first = torch.randn(wl.q_dim, wl.d_model, generator=g) * 0.02
    assert torch.equal(a.layers[0]["wq"], first)
    g = torch.Generator().manual_seed(0)
    for _ in range(wl.n_layers):
        for shape in ((wl.q_dim, wl.d_model), (wl.d_model, wl.q_dim), (wl.ffn, wl.d_model),
                      (wl.ffn, wl.d_model), (wl.d_model, wl.ffn)):
            torch.randn(*shape, generator=g)
    kv = (wl.n_layers, wl.ctx + wl.T, wl.n_kv_heads, wl.head_dim)
    torch.randn(*kv, generator=g)
    torch.randn(*kv, generator=g)
    assert torch.equal(a.x0, torch.randn(wl.T, wl.d_model, generator=g))


def test_lm_head_and_random_states():
    wl = W.WORKLOADS["tiny"]
    h = W.lm_head(wl)
    assert tuple(h.shape) == (W.VOCAB["tiny"], wl.d_model) and h.dtype == torch.bfloat16
    assert torch.equal(h, W.lm_head(wl)) and not torch.equal(h, W.lm_head(wl, seed=2))
    s = W.random_states((3, 4, 8), 5)
    assert torch.equal(s, W.random_states((3, 4, 8), 5)) and s.dtype == torch.float32


@pytest.mark.parametrize("name", ["tiny", "small"])
def test_streamed_inputs_equal_the_full_draw(name):
    """StreamedInputs (one layer held at a time, each redrawn from its recorded
    generator state) gives the same values and the same digest as make_inputs."""
    wl = W.WORKLOADS[name]
    full = W.make_inputs(wl)
    st = W.StreamedInputs(wl)
    assert st.digest == W.input_digest(full)
    for l in (wl.n_layers - 1, 0, 1):               # any order: each layer from its own state
        for k in W.LAYER_KEYS:
            assert torch.equal(st.layers[l][k], full.layers[l][k]), (l, k)
    assert torch.equal(st.k_cache, full.k_cache) and torch.equal(st.v_cache, full.v_cache)
    assert torch.equal(st.x0, full.x0)
    # a different seed changes the digest
    assert W.StreamedInputs(wl, seed=1).digest != st.digest


def test_streamed_inputs_kept_on_a_device_need_no_second_draw(monkeypatch):
    """With a device given, the layers are copied there while the digest is taken,
    and to(device) hands those copies back without drawing again."""
    wl = W.WORKLOADS["tiny"]
    full = W.make_inputs(wl)
    st = W.StreamedInputs(wl, device="cpu")
    assert st.digest == W.input_digest(full)
    monkeypatch.setattr(W, "_draw_layer", lambda *a, **k: pytest.fail("layer drawn again"))
    on = st.to("cpu")
    for l in range(wl.n_layers):
        for k in W.LAYER_KEYS:
            assert torch.equal(on.layers[l][k], full.layers[l][k]), (l, k)
    assert torch.equal(on.k_cache, full.k_cache) and torch.equal(on.x0, full.x0)


def test_every_workload_is_drawn_on_the_cpu_generator():
    assert all(wl.gen_device == "cpu" for wl in W.WORKLOADS.values())
