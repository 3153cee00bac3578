"""Distinct-state execution (ks_params.dedup) reproduces the dense solve bit for
bit: every row of every kernel is computed independently of the rows around
it, so running an item once per distinct source state and reading the result
back for every cell that holds that state changes nothing but the work."""
import numpy as np
import pytest
import torch

from knapsack_layer_selection_b200 import binding as B
from knapsack_layer_selection_b200 import build as BUILD
from knapsack_layer_selection_b200 import workloads as W

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    BUILD.build()
    return B.load()


def run(wl, g, **kw):
    m = B.model_desc(wl.n_layers, wl.d_model, wl.n_q_heads, wl.n_kv_heads, wl.head_dim, wl.ffn,
                     wl.rms_eps, wl.rope_base, wl.wdtype)
    s = B.Solver(m, g.layers, g.k_cache, g.v_cache, wl.ctx, wl.T, wl.latencies(),
                 B.params(wl.gamma_max, wl.n_bins, **kw), keep_cos=True)
    s.solve(g.x0)
    torch.cuda.synchronize()
    s.check_status()
    o = s.out
    return s, {k: getattr(o, k).cpu().numpy() for k in
               ("bp", "values", "sets", "used_w", "t_draft", "best", "best_tpt", "ref_states",
                "cos_skip", "cos_exec", "exec_counts")}


CASES = [("tiny", {}), ("small", {}), ("small", {"budget_mode": "exact"}),
         ("small", {"prune_tau": 0.85, "skip_cap": 128}), ("tiny", {"budget_mode": "exact"})]


@pytest.mark.parametrize("name,kw", CASES)
def test_dedup_is_bit_identical_to_dense(name, kw):
    wl = W.WORKLOADS[name]
    g = W.make_inputs(wl).to("cuda")
    s_dense, dense = run(wl, g, **kw)
    s_dd, dd = run(wl, g, dedup=True, **kw)
    for k in ("bp", "values", "sets", "used_w", "t_draft", "best", "best_tpt", "ref_states",
              "cos_skip", "cos_exec"):
        assert np.array_equal(dense[k], dd[k], equal_nan=True), k
    E1 = np.array([s_dense.C - w + 1 for w in s_dense.w])     # dense batch: cells + reference
    assert np.array_equal(dense["exec_counts"], E1)
    assert np.all(dd["exec_counts"] >= 1) and np.all(dd["exec_counts"] <= E1)
    print(f"\n{name} {kw}: distinct states executed {int(dd['exec_counts'].sum())} of "
          f"{int(E1.sum())} ({dd['exec_counts'].sum() / E1.sum():.1%})")


def test_dedup_rejects_grids_beyond_its_table():
    wl = W.WORKLOADS["tiny"]
    g = W.make_inputs(wl).to("cuda")
    m = B.model_desc(wl.n_layers, wl.d_model, wl.n_q_heads, wl.n_kv_heads, wl.head_dim, wl.ffn,
                     wl.rms_eps, wl.rope_base, wl.wdtype)
    t = wl.latencies()
    with pytest.raises(B.KnapSpecError, match="3071"):
        s = B.Solver(m, g.layers, g.k_cache, g.v_cache, wl.ctx, wl.T, t,
                     B.params(wl.gamma_max, 4000, dedup=True))
        s.solve(g.x0)


@pytest.mark.parametrize("name,kw", [("small", {}), ("small", {"budget_mode": "exact"}),
                                     ("tiny", {})])
def test_byte_check_separates_colliding_fingerprints(name, kw):
    """With fingerprints cut to 8 bits, unequal states share fingerprints often;
    every such fold must be rejected by the byte comparison, leaving the result
    bit-identical to the dense solve."""
    wl = W.WORKLOADS[name]
    g = W.make_inputs(wl).to("cuda")
    s_dense, dense = run(wl, g, **kw)
    s_weak, weak = run(wl, g, dedup="weak", **kw)
    s_full, full = run(wl, g, dedup=True, **kw)
    for k in ("bp", "values", "sets", "used_w", "t_draft", "best", "best_tpt", "ref_states",
              "cos_skip", "cos_exec"):
        assert np.array_equal(dense[k], weak[k], equal_nan=True), k
    rejected_weak = int(s_weak.out.dedup_rejected.sum())
    rejected_full = int(s_full.out.dedup_rejected.sum())
    assert rejected_full == 0          # no 64-bit collision expected on these inputs
    if name == "small":
        assert rejected_weak > 0       # 8-bit fingerprints: collisions did happen
    # a rejected fold runs its state on its own, never fewer states than the full check
    assert np.all(weak["exec_counts"] >= full["exec_counts"])
    print(f"\n{name} {kw}: 8-bit fingerprints: byte check rejected {rejected_weak} folds; "
          f"states executed {int(weak['exec_counts'].sum())} (64-bit: {int(full['exec_counts'].sum())})")
