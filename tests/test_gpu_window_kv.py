"""GPU parity of the window key/value reading (ks_cache_desc.kv_mode =
KS_KV_WINDOW) against the oracle's kv="window" (reading R7w): the T window
positions' keys and values are recomputed from each candidate state through
Wk / Wv (keys rotated at ctx + t), the context positions come from the cache,
and token t sees the window tokens 0 .. t of its own state.

* one Attention sublayer on a batch of states that spans several 128-row tiles
  with a ragged tail, at context lengths 0, one short of a key block, and the
  workload's own -- fp32 (CUDA-core kernels) and bf16 (tensor-core kernels);
* whole DP solves on the tiny and small workloads (and small's first four
  layers) under the near-tie / taint rule, dense and with distinct-state
  execution; the reference states the solve carries match the oracle's chain;
* host checks: Wk / Wv are required, T must divide 128 on the tensor cores.
"""
import dataclasses

import numpy as np
import pytest
import torch

from knapsack_layer_selection_b200 import binding as B
from knapsack_layer_selection_b200 import build as BUILD
from knapsack_layer_selection_b200 import workloads as W
from oracle import ks_oracle as O
from tests._parity import compare_solve
from tests._util import oracle_model, x0_np

pytestmark = pytest.mark.gpu

VAL_TOL = {"f32": 1e-5, "bf16": 2e-3}
SUBLAYER_TOL = {"f32": 1e-5, "bf16": 1e-2}


@pytest.fixture(scope="module", autouse=True)
def lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    BUILD.build()
    return B.load()


def window_inputs(name, n_layers=None):
    """The workload's seeded inputs with each layer's Wk / Wv added."""
    wl = W.WORKLOADS[name]
    inp = W.make_inputs(wl)
    ww = W.window_weights(wl)
    inp = dataclasses.replace(inp, layers=[{**L, **w} for L, w in zip(inp.layers, ww)])
    return inp.first_layers(n_layers) if n_layers is not None else inp


def model_of(wl):
    return B.model_desc(wl.n_layers, wl.d_model, wl.n_q_heads, wl.n_kv_heads, wl.head_dim, wl.ffn,
                        wl.rms_eps, wl.rope_base, wl.wdtype)


def _branch_rel_err(out_g, out_o, H):
    return float(np.linalg.norm((out_g - H) - (out_o - H)) / np.linalg.norm(out_o - H))


@pytest.mark.parametrize("name,E,ctx", [("tiny", 9, 128), ("tiny", 5, 0), ("small", 37, 2048),
                                        ("small", 37, 127), ("small", 20, 0)])
def test_window_attention_sublayer_matches_oracle(name, E, ctx):
    inp = window_inputs(name)
    wl = inp.wl
    g = inp.to("cuda")
    m = model_of(wl)
    layers = B.layer_array(g.layers, W.torch_dtype(wl), m)
    cache = B.cache_desc(g.k_cache, g.v_cache, ctx, m, kv="window")
    om = oracle_model(inp)
    H = W.random_states((E, wl.T, wl.d_model), 21)
    H[2] = H[1]                                   # two identical states
    Hd = H.cuda()
    ws = B.workspace(m, E, wl.T)
    for k in (0, 2 * (wl.n_layers - 1)):          # the first and the last Attention item
        out = torch.empty_like(Hd)
        B.sublayer_forward(m, layers, cache, wl.T, k, Hd, out, ws)
        one = torch.empty_like(Hd[:1])
        B.sublayer_forward(m, layers, cache, wl.T, k, Hd[1:2].contiguous(), one, ws)
        torch.cuda.synchronize()
        assert B.workspace_status(ws) == 0
        og = O.apply_item(om, k, H.double().numpy(), ctx, kv="window")
        err = _branch_rel_err(out.double().cpu().numpy(), og, H.double().numpy())
        assert err < SUBLAYER_TOL[wl.wdtype], (k, err)
        # the window reading differs from the cache reading well beyond the
        # tolerance (else nothing is tested); at long contexts the T window keys
        # are a small share of the attention, so the gap is a few per cent
        oc = O.apply_item(om, k, H.double().numpy(), ctx, kv="cache")
        assert _branch_rel_err(oc, og, H.double().numpy()) > 3 * SUBLAYER_TOL[wl.wdtype]
        # a state's result depends only on its own rows
        assert torch.equal(out[1], out[2])
        assert torch.equal(out[1], one[0])


_cache = {}


def solved_oracle(name, n_layers, mode):
    key = (name, n_layers, mode)
    if key not in _cache:
        inp = window_inputs(name, n_layers)
        wl = inp.wl
        base = W.WORKLOADS[name]
        t = base.latencies()[:wl.n_items]
        w = O.quantize_weights(base.latencies(), base.n_bins)[:wl.n_items]
        orc = O.dp_solve(oracle_model(inp), x0_np(inp), wl.ctx, w, t, wl.gamma_max,
                         per_cell=(wl.wdtype == "f32"), mode=mode, kv="window")
        _cache[key] = (inp, w, t, orc)
    return _cache[key]


@pytest.mark.parametrize("name,n_layers,mode,dedup", [
    ("tiny", None, "at_most", False), ("tiny", None, "exact", False),
    ("small", 4, "at_most", False), ("small", None, "at_most", False),
    ("small", None, "at_most", True), ("small", None, "exact", True)])
def test_window_solve_matches_oracle(name, n_layers, mode, dedup):
    inp, w, t, orc = solved_oracle(name, n_layers, mode)
    wl = inp.wl
    g = inp.to("cuda")
    s = B.Solver(model_of(wl), g.layers, g.k_cache, g.v_cache, wl.ctx, wl.T, t,
                 B.params(wl.gamma_max, wl.n_bins, budget_mode=mode, dedup=dedup), w=w,
                 keep_cos=True, kv="window")
    s.solve(g.x0)
    torch.cuda.synchronize()
    s.check_status()
    o = s.out
    bp = o.bp.cpu().numpy()
    res = {"bp": bp, "values": o.values.cpu().numpy(), "sets": B.sets_to_lists(o.sets, wl.n_items),
           "best": o.best.cpu().numpy()}
    rows = np.where(bp == 1, o.cos_exec.cpu().numpy(), o.cos_skip.cpu().numpy())
    rep = compare_solve(orc, res, w, VAL_TOL[wl.wdtype], wl.n_items, rows_val_gpu=rows)
    ref = o.ref_states.double().cpu().numpy()
    tol = 1e-5 if wl.wdtype == "f32" else 2e-2
    for k in range(1, wl.n_items + 1):
        assert np.linalg.norm(ref[k] - orc.ref[k]) / np.linalg.norm(orc.ref[k]) < tol, k
    print(f"\nwindow K/V {name}/{n_layers} {mode} dedup={dedup}: {rep}")
    rep.assert_ok()
    if mode == "at_most":
        assert abs(res["values"][-1] - 1.0) <= 1e-6


def test_window_reading_host_checks():
    inp = W.make_inputs(W.WORKLOADS["small"]).first_layers(1)
    wl = inp.wl
    g = inp.to("cuda")
    m = model_of(wl)
    # no Wk / Wv
    with pytest.raises(B.KnapSpecError, match="wk and wv"):
        s = B.Solver(m, g.layers, g.k_cache, g.v_cache, wl.ctx, wl.T, wl.latencies()[:2],
                     B.params(wl.gamma_max, 16), kv="window")
        s.solve(g.x0)
    # T must divide 128 on the tensor-core path
    ww = W.window_weights(wl, device="cpu")
    layers = [{**L, **{k: v.cuda() for k, v in w_.items()}} for L, w_ in zip(g.layers, ww)]
    with pytest.raises(B.KnapSpecError, match="divide 128"):
        s = B.Solver(m, layers, g.k_cache, g.v_cache, wl.ctx, 6, wl.latencies()[:2],
                     B.params(wl.gamma_max, 16), kv="window")
        s.solve(torch.zeros(6, wl.d_model, device="cuda"))
