"""Pins of the oracle's alternative attention reading R7w (keys/values of the T
window positions recomputed from the candidate's own state through Wk/Wv,
the earlier positions from the full model's cache) -- the variant the review's
description leaves open next to R7, where every key/value comes from the cache.

* torch fp64 library ops (RMSNorm, linear maps, complex-number RoPE, SDPA with
  an explicit mask and GQA) compute the same sublayer independently;
* when the cache's window rows hold a state's own keys/values (built by the
  torch path), R7w and R7 agree on that state, and not on another one;
* within the window attention is causal: token t never sees a later token of
  its own state, while under R7 tokens do not see each other at all;
* the DP invariants hold with R7w items (all-execute cell, re-run of each set,
  exhaustive bound), and planted mistakes in the window keys are caught.
No GPU involved: R7w has no kernel; these pins fix the oracle a kernel for it
would be compared with.
"""
import dataclasses

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from knapsack_layer_selection_b200 import workloads as W
from oracle import ks_oracle as O
from tests._util import oracle_model, x0_np


def _with_window_weights(m: O.Model, seed: int) -> O.Model:
    """A copy of m whose layers also carry Wk, Wv [Hkv*hd][d] ~ N(0, 1/d)."""
    rng = np.random.default_rng(seed)
    layers = []
    for i in range(len(m.layers)):
        L = dict(m.layers[i])
        d = L["wq"].shape[1]
        kvd = m.n_kv_heads * m.head_dim
        L["wk"] = rng.normal(0.0, d ** -0.5, (kvd, d))
        L["wv"] = rng.normal(0.0, d ** -0.5, (kvd, d))
        layers.append(L)
    kc = [np.asarray(m.k_cache[i], np.float64) for i in range(len(m.layers))]
    vc = [np.asarray(m.v_cache[i], np.float64) for i in range(len(m.layers))]
    return dataclasses.replace(m, layers=layers, k_cache=kc, v_cache=vc)


def _gqa_model(seed=3, L=2, d=64, Hq=4, Hkv=2, hd=16, F_=96, n_pos=14) -> O.Model:
    rng = np.random.default_rng(seed)
    s = d ** -0.5
    layers = [{"attn_norm": rng.uniform(0.5, 1.5, d), "wq": rng.normal(0, s, (Hq * hd, d)),
               "wo": rng.normal(0, s, (d, Hq * hd)), "mlp_norm": rng.uniform(0.5, 1.5, d),
               "w_gate": rng.normal(0, s, (F_, d)), "w_up": rng.normal(0, s, (F_, d)),
               "w_down": rng.normal(0, F_ ** -0.5, (d, F_)),
               "wk": rng.normal(0, s, (Hkv * hd, d)), "wv": rng.normal(0, s, (Hkv * hd, d))}
              for _ in range(L)]
    kc = [rng.normal(0, 1, (n_pos, Hkv, hd)) for _ in range(L)]
    vc = [rng.normal(0, 1, (n_pos, Hkv, hd)) for _ in range(L)]
    return O.Model(Hq, Hkv, hd, 1e-6, 1e4, layers, kc, vc)


def _rope_complex(x, ctx, base):
    """RoPE of x [M, T, H, hd] at positions ctx + t as a complex multiplication
    of the pairs (j, j + hd/2)."""
    M, T, H, hd = x.shape
    half = hd // 2
    z = torch.complex(x[..., :half], x[..., half:])
    pos = torch.arange(ctx, ctx + T, dtype=torch.float64)
    inv = torch.tensor([base ** (-2.0 * j / hd) for j in range(half)], dtype=torch.float64)
    rot = torch.polar(torch.ones(T, half, dtype=torch.float64), pos[:, None] * inv[None, :])
    z = z * rot[None, :, None, :]
    return torch.cat([z.real, z.imag], dim=-1)


def _torch_window_kv(m, layer, H, ctx):
    Lw = {k: torch.tensor(np.asarray(v), dtype=torch.float64) for k, v in m.layers[layer].items()}
    H = torch.tensor(H, dtype=torch.float64)
    M, T, d = H.shape
    xh = F.rms_norm(H, (d,), weight=Lw["attn_norm"], eps=m.rms_eps)
    kw = _rope_complex(F.linear(xh, Lw["wk"]).reshape(M, T, m.n_kv_heads, m.head_dim), ctx,
                       m.rope_base)
    vw = F.linear(xh, Lw["wv"]).reshape(M, T, m.n_kv_heads, m.head_dim)
    return xh, kw, vw


def _torch_window_item(m, layer, H, ctx):
    """Attention sublayer under R7w with torch fp64 library ops (independent path)."""
    Lw = {k: torch.tensor(np.asarray(v), dtype=torch.float64) for k, v in m.layers[layer].items()}
    xh, kw, vw = _torch_window_kv(m, layer, H, ctx)
    Ht = torch.tensor(H, dtype=torch.float64)
    M, T, d = Ht.shape
    Hq, hd = m.n_q_heads, m.head_dim
    q = _rope_complex(F.linear(xh, Lw["wq"]).reshape(M, T, Hq, hd), ctx, m.rope_base)
    kc = torch.tensor(np.asarray(m.k_cache[layer][:ctx]), dtype=torch.float64)
    vc = torch.tensor(np.asarray(m.v_cache[layer][:ctx]), dtype=torch.float64)
    k = torch.cat([kc[None].expand(M, -1, -1, -1), kw], dim=1)          # [M, ctx+T, Hkv, hd]
    v = torch.cat([vc[None].expand(M, -1, -1, -1), vw], dim=1)
    n = ctx + T
    mask = torch.arange(n)[None, :] <= (ctx + torch.arange(T))[:, None]
    o = F.scaled_dot_product_attention(q.permute(0, 2, 1, 3), k.permute(0, 2, 1, 3),
                                       v.permute(0, 2, 1, 3), attn_mask=mask, enable_gqa=True)
    o = o.permute(0, 2, 1, 3).reshape(M, T, Hq * hd)
    return (Ht + F.linear(o, Lw["wo"])).numpy()


def _rel(a, b):
    return float(np.max(np.abs(a - b)) / np.max(np.abs(b)))


@pytest.fixture(scope="module")
def tiny_w():
    wl = W.WORKLOADS["tiny"]
    inp = W.make_inputs(wl)
    return wl, inp, _with_window_weights(oracle_model(inp), seed=11)


def test_window_item_matches_torch_library():
    m = _gqa_model()
    ctx, T = 9, 5
    H = np.random.default_rng(0).normal(0, 1, (3, T, 64))
    for layer in range(2):
        got = O.attn_item(m, layer, H, ctx, kv="window")
        assert _rel(got, _torch_window_item(m, layer, H, ctx)) < 1e-12


def test_window_item_matches_torch_library_on_tiny(tiny_w):
    wl, inp, m = tiny_w
    H = np.random.default_rng(1).normal(0, 1, (2, wl.T, wl.d_model))
    got = O.apply_item(m, 2, H, wl.ctx, kv="window")
    assert _rel(got, _torch_window_item(m, 1, H, wl.ctx)) < 1e-12


def test_window_equals_cache_when_the_cache_holds_the_states_own_kv():
    m = _gqa_model(n_pos=14)
    ctx, T, layer = 9, 5, 1
    rng = np.random.default_rng(5)
    H = rng.normal(0, 1, (1, T, 64))
    _, kw, vw = _torch_window_kv(m, layer, H, ctx)
    kc = [c.copy() for c in m.k_cache]
    vc = [c.copy() for c in m.v_cache]
    kc[layer][ctx:ctx + T] = kw[0].numpy()
    vc[layer][ctx:ctx + T] = vw[0].numpy()
    m2 = dataclasses.replace(m, k_cache=kc, v_cache=vc)
    a = O.attn_item(m2, layer, H, ctx, kv="window")
    b = O.attn_item(m2, layer, H, ctx, kv="cache")
    assert _rel(a - H, b - H) < 1e-12
    # another state keeps its own window keys: the two readings now differ
    H2 = rng.normal(0, 1, (1, T, 64))
    a2 = O.attn_item(m2, layer, H2, ctx, kv="window")
    b2 = O.attn_item(m2, layer, H2, ctx, kv="cache")
    assert _rel(a2 - H2, b2 - H2) > 1e-3


def test_window_is_causal_and_cache_reading_is_per_token():
    m = _gqa_model()
    ctx, T = 9, 5
    rng = np.random.default_rng(7)
    H = rng.normal(0, 1, (1, T, 64))
    for j in range(T):
        Hp = H.copy()
        Hp[0, j] += rng.normal(0, 1, 64)
        a = O.attn_item(m, 0, H, ctx, kv="window")
        ap = O.attn_item(m, 0, Hp, ctx, kv="window")
        # tokens before j never see token j (its key is masked), bit for bit
        assert np.array_equal(a[0, :j], ap[0, :j]), j
        # every later token does see it
        for t in range(j + 1, T):
            assert not np.allclose(a[0, t], ap[0, t], rtol=0, atol=1e-9), (j, t)
        # under R7 the tokens do not see each other: only token j moves
        c = O.attn_item(m, 0, H, ctx, kv="cache")
        cp = O.attn_item(m, 0, Hp, ctx, kv="cache")
        others = [t for t in range(T) if t != j]
        assert np.array_equal(c[0, others], cp[0, others]), j


def test_window_dp_invariants_on_tiny(tiny_w):
    wl, inp, m = tiny_w
    t = wl.latencies()
    w = O.quantize_weights(t, wl.n_bins)
    x0 = x0_np(inp)
    s = O.dp_solve(m, x0, wl.ctx, w, t, wl.gamma_max, per_cell=True, kv="window")
    K = sum(w)
    # the reference chain is the all-execute chain, and it scores exactly 1
    assert s.values[K] == 1.0 and s.sets[K] == list(range(wl.n_items))
    assert np.array_equal(O.chain(m, x0, wl.ctx, range(wl.n_items), kv="window"), s.ref[-1])
    # every cell's set re-run from scratch reproduces its value bit for bit
    for b in range(K + 1):
        assert O.eval_set(m, x0, wl.ctx, s.sets[b], s.ref, kv="window") == s.values[b], b
        assert s.used_w[b] <= b
    # exhaustive search over all 2^8 subsets bounds every value
    best, _ = O.brute_force(m, x0, wl.ctx, w, s.ref, kv="window")
    assert np.all(s.values <= best + 1e-12)
    # the reading matters: R7 gives different reference states on the same inputs
    r7 = O.reference_states(m, x0, wl.ctx)
    assert not np.allclose(r7[2], s.ref[2])


def test_planted_window_key_mistakes_are_caught(monkeypatch):
    m = _gqa_model()
    ctx, T = 9, 5
    H = np.random.default_rng(0).normal(0, 1, (2, T, 64))
    want = _torch_window_item(m, 0, H, ctx)

    def unrotated(model, layer, xh, ctx_):                       # keys left without RoPE
        Lw = model.layers[layer]
        M, T_, d = xh.shape
        shape = (M, T_, model.n_kv_heads, model.head_dim)
        k = (xh.reshape(M * T_, d) @ np.asarray(Lw["wk"]).T).reshape(shape)
        v = (xh.reshape(M * T_, d) @ np.asarray(Lw["wv"]).T).reshape(shape)
        return k, v

    def shifted(model, layer, xh, ctx_):                         # keys rotated one position late
        Lw = model.layers[layer]
        M, T_, d = xh.shape
        shape = (M, T_, model.n_kv_heads, model.head_dim)
        k = (xh.reshape(M * T_, d) @ np.asarray(Lw["wk"]).T).reshape(shape)
        k = O.rope_rotate_half(k, ctx_ + 1 + np.arange(T_), model.rope_base)
        v = (xh.reshape(M * T_, d) @ np.asarray(Lw["wv"]).T).reshape(shape)
        return k, v

    for bad in (unrotated, shifted):
        with monkeypatch.context() as mp:
            mp.setattr(O, "window_kv", bad)
            assert _rel(O.attn_item(m, 0, H, ctx, kv="window"), want) > 1e-6, bad.__name__
    assert _rel(O.attn_item(m, 0, H, ctx, kv="window"), want) < 1e-12
