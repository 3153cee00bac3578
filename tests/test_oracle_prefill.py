"""Pins of the oracle's full-model prefill (the workloads' "KV cache from the
full model" for the tiny and small configurations):

* against torch fp64 library ops (RMSNorm, linear maps, RoPE as a complex
  multiplication, causal SDPA with GQA, SiLU) on a small GQA model;
* a fixed point that ties it to the DP's own sublayers: with the prefilled
  cache, the reference chain of the last T tokens (attn_item / mlp_item over the
  cache, reading R7) reproduces the prefill's hidden states of those tokens at
  every depth, and so does the window reading R7w (the cache then holds each
  reference state's own keys and values);
* a planted mistake (one future position visible) breaks the fixed point.
No GPU involved.
"""
import dataclasses
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from knapsack_layer_selection_b200 import workloads as W
from oracle import ks_oracle as O
from tests._util import oracle_model


def _model(seed=5, L=2, d=64, Hq=4, Hkv=2, hd=16, F_=96) -> O.Model:
    rng = np.random.default_rng(seed)
    s = d ** -0.5
    layers = [{"attn_norm": rng.uniform(0.5, 1.5, d), "wq": rng.normal(0, s, (Hq * hd, d)),
               "wo": rng.normal(0, s, (d, Hq * hd)), "mlp_norm": rng.uniform(0.5, 1.5, d),
               "w_gate": rng.normal(0, s, (F_, d)), "w_up": rng.normal(0, s, (F_, d)),
               "w_down": rng.normal(0, F_ ** -0.5, (d, F_)),
               "wk": rng.normal(0, s, (Hkv * hd, d)), "wv": rng.normal(0, s, (Hkv * hd, d))}
              for _ in range(L)]
    return O.Model(Hq, Hkv, hd, 1e-6, 1e4, layers, [], [])


def _rope(x, base):
    """RoPE of x [n, H, hd] at positions 0 .. n-1 as a complex multiplication."""
    n, H, hd = x.shape
    half = hd // 2
    z = torch.complex(x[..., :half], x[..., half:])
    inv = torch.tensor([base ** (-2.0 * j / hd) for j in range(half)], dtype=torch.float64)
    rot = torch.polar(torch.ones(n, half, dtype=torch.float64),
                      torch.arange(n, dtype=torch.float64)[:, None] * inv[None, :])
    z = z * rot[:, None, :]
    return torch.cat([z.real, z.imag], dim=-1)


def _torch_prefill(m, emb):
    h = torch.tensor(emb, dtype=torch.float64)
    n, d = h.shape
    ks, vs, hid = [], [], [h]
    for Lw in m.layers:
        Lw = {k: torch.tensor(np.asarray(v), dtype=torch.float64) for k, v in Lw.items()}
        xh = F.rms_norm(h, (d,), weight=Lw["attn_norm"], eps=m.rms_eps)
        q = _rope(F.linear(xh, Lw["wq"]).reshape(n, m.n_q_heads, m.head_dim), m.rope_base)
        k = _rope(F.linear(xh, Lw["wk"]).reshape(n, m.n_kv_heads, m.head_dim), m.rope_base)
        v = F.linear(xh, Lw["wv"]).reshape(n, m.n_kv_heads, m.head_dim)
        ks.append(k)
        vs.append(v)
        o = F.scaled_dot_product_attention(q.transpose(0, 1), k.transpose(0, 1), v.transpose(0, 1),
                                           is_causal=True, enable_gqa=True)
        h = h + F.linear(o.transpose(0, 1).reshape(n, -1), Lw["wo"])
        hid.append(h)
        xm = F.rms_norm(h, (d,), weight=Lw["mlp_norm"], eps=m.rms_eps)
        h = h + F.linear(F.silu(F.linear(xm, Lw["w_gate"])) * F.linear(xm, Lw["w_up"]), Lw["w_down"])
        hid.append(h)
    return torch.stack(ks).numpy(), torch.stack(vs).numpy(), torch.stack(hid).numpy()


def _rel(a, b):
    return float(np.max(np.abs(a - b)) / np.max(np.abs(b)))


def test_prefill_matches_torch_library():
    m = _model()
    emb = np.random.default_rng(0).normal(0, 1, (13, 64))
    pf = O.prefill(m, emb)
    k, v, hid = _torch_prefill(m, emb)
    assert _rel(pf.k_cache, k) < 1e-12 and _rel(pf.v_cache, v) < 1e-12
    assert _rel(pf.hidden, hid) < 1e-12


def _chain_matches_prefill(m, emb, T, kv):
    pf = O.prefill(m, emb)
    n = emb.shape[0]
    mc = dataclasses.replace(m, k_cache=list(pf.k_cache), v_cache=list(pf.v_cache))
    ref = O.reference_states(mc, emb[n - T:], n - T, kv=kv)
    return max(_rel(ref[i], pf.hidden[i][n - T:]) for i in range(ref.shape[0]))


@pytest.mark.parametrize("kv", ["cache", "window"])
def test_reference_chain_over_the_prefilled_cache_is_the_prefill(kv):
    m = _model(seed=7)
    emb = np.random.default_rng(1).normal(0, 1, (17, 64))
    assert _chain_matches_prefill(m, emb, 4, kv) < 1e-12


def test_prefill_on_the_tiny_workload_is_a_fixed_point():
    wl = W.WORKLOADS["tiny"]
    inp = W.make_inputs(wl)
    ww = W.window_weights(wl)
    inp = dataclasses.replace(inp, layers=[{**L, **w} for L, w in zip(inp.layers, ww)])
    m = oracle_model(inp)
    m = dataclasses.replace(m, layers=[m.layers[i] for i in range(len(m.layers))])
    emb = W.sequence_embeddings(wl).double().numpy()
    assert emb.shape == (wl.ctx + wl.T, wl.d_model)
    assert _chain_matches_prefill(m, emb, wl.T, "cache") < 1e-11


def test_planted_future_position_breaks_the_fixed_point(monkeypatch):
    """A prefill that lets each position see one position ahead no longer
    agrees with the chain over its own cache (the chain's mask is causal)."""
    m = _model(seed=9)
    emb = np.random.default_rng(2).normal(0, 1, (15, 64))
    good = _chain_matches_prefill(m, emb, 5, "cache")
    orig = O.prefill

    def leaky_prefill(model, e):
        # the same as O.prefill with the causal mask widened by one position
        h = np.asarray(e, np.float64)
        n, d = h.shape
        Hq, Hkv, hd = model.n_q_heads, model.n_kv_heads, model.head_dim
        grp = Hq // Hkv
        pos = np.arange(n)
        mask = pos[None, :] <= pos[:, None] + 1
        kc, vc, hid = [], [], [h]
        for l, Lw in enumerate(model.layers):
            xh = O.rms_norm(h, Lw["attn_norm"], model.rms_eps)
            q = O.rope_rotate_half((xh @ Lw["wq"].T).reshape(1, n, Hq, hd), pos, model.rope_base)[0]
            k = O.rope_rotate_half((xh @ Lw["wk"].T).reshape(1, n, Hkv, hd), pos, model.rope_base)[0]
            v = (xh @ Lw["wv"].T).reshape(n, Hkv, hd)
            kc.append(k)
            vc.append(v)
            o = np.empty((n, Hq, hd))
            for hq in range(Hq):
                s = np.where(mask, q[:, hq] @ k[:, hq // grp].T / math.sqrt(hd), -np.inf)
                p = np.exp(s - s.max(-1, keepdims=True))
                o[:, hq] = (p / p.sum(-1, keepdims=True)) @ v[:, hq // grp]
            h = h + o.reshape(n, -1) @ Lw["wo"].T
            hid.append(h)
            h = O.mlp_item(model, l, h[None])[0]
            hid.append(h)
        return O.Prefill(np.stack(kc), np.stack(vc), np.stack(hid))

    monkeypatch.setattr(O, "prefill", leaky_prefill)
    bad = _chain_matches_prefill(m, emb, 5, "cache")
    monkeypatch.setattr(O, "prefill", orig)
    assert good < 1e-12 and bad > 1e-3, (good, bad)
