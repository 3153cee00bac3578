"""GPU ks_solve against the oracle on whole DPs, with the near-tie/taint rule.

tiny (fp32, all 29 budgets), small (bf16, all 257 budgets) and small's first
four layers (8 items), whose exhaustive subset search also bounds the GPU's
values.  Determinism and the given-reference path are checked bit for bit.
"""
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


@pytest.fixture(scope="module", autouse=True)
def lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    BUILD.build()
    return B.load()


def make_solver(wl, inp_gpu, w=None, t=None, keep_cos=True, mode="at_most", tau=None, cap=None):
    m = B.model_desc(wl.n_layers, wl.d_model, wl.n_q_heads, wl.n_kv_heads, wl.head_dim, wl.ffn,
                     wl.rms_eps, wl.rope_base, wl.wdtype)
    t = wl.latencies() if t is None else t
    prm = B.params(wl.gamma_max, wl.n_bins, budget_mode=mode, prune_tau=tau, skip_cap=cap)
    return B.Solver(m, inp_gpu.layers, inp_gpu.k_cache, inp_gpu.v_cache, wl.ctx, wl.T, t, prm,
                    w=w, keep_cos=keep_cos)


def gpu_result(solver):
    torch.cuda.synchronize()
    solver.check_status()
    o = solver.out
    bp = o.bp.cpu().numpy()
    rows = np.where(bp == 1, o.cos_exec.cpu().numpy(), o.cos_skip.cpu().numpy())
    return {"bp": bp, "values": o.values.cpu().numpy(),
            "sets": B.sets_to_lists(o.sets, solver.n_items),
            "used_w": o.used_w.cpu().numpy(), "t_draft": o.t_draft.cpu().numpy(),
            "best": o.best.cpu().numpy(), "rows": rows,
            "ref": o.ref_states.cpu().numpy()}


_cache = {}


def solved(name, n_layers=None, mode="at_most", tau=None, cap=None):
    key = (name, n_layers, mode, tau, cap)
    if key in _cache:
        return _cache[key]
    wl = W.WORKLOADS[name]
    inp = W.make_inputs(wl)
    t = wl.latencies()
    w = O.quantize_weights(t, wl.n_bins)
    if n_layers is not None:
        inp = inp.first_layers(n_layers)
        wl = inp.wl
        t, w = t[:2 * n_layers], w[:2 * n_layers]
    g = inp.to("cuda")
    solver = make_solver(wl, g, w=w, t=t, mode=mode, tau=tau, cap=cap)
    solver.solve(g.x0)
    res = gpu_result(solver)
    orc = O.dp_solve(oracle_model(inp), x0_np(inp), wl.ctx, w, t, wl.gamma_max,
                     per_cell=(wl.wdtype == "f32"), mode=mode, prune_tau=tau, skip_cap=cap)
    _cache[key] = (wl, inp, g, solver, res, orc, w, t)
    return _cache[key]


@pytest.mark.parametrize("name,n_layers", [("tiny", None), ("small", 4), ("small", None)])
def test_solve_matches_oracle(name, n_layers):
    wl, inp, g, solver, res, orc, w, t = solved(name, n_layers)
    rep = compare_solve(orc, res, w, VAL_TOL[wl.wdtype], wl.n_items, rows_val_gpu=res["rows"])
    print(f"\n{name}/{n_layers}: {rep}")
    rep.assert_ok()
    C = len(orc.values)
    assert len(res["values"]) == C
    # all-execute cell: exactly the reference chain
    assert abs(res["values"][-1] - 1.0) <= 1e-6
    assert res["sets"][-1] == list(range(wl.n_items))
    # used weight never exceeds the budget and matches the set
    for b in range(C):
        assert res["used_w"][b] <= b
        assert res["used_w"][b] == sum(w[k] for k in res["sets"][b])


@pytest.mark.parametrize("name,n_layers", [("tiny", None), ("small", 4), ("small", None)])
def test_exact_budget_mode_matches_oracle(name, n_layers):
    """The paper's exact-budget table (only g[0,0] starts valid): validity is
    integer logic and must match exactly; values and choices under the same
    near-tie/taint rule as the at-most mode."""
    wl, inp, g, solver, res, orc, w, t = solved(name, n_layers, "exact")
    rep = compare_solve(orc, res, w, VAL_TOL[wl.wdtype], wl.n_items, rows_val_gpu=res["rows"])
    print(f"\n{name}/{n_layers} exact: {rep}")
    rep.assert_ok()
    valid_o = orc.dp.valid[-1]
    assert np.array_equal(np.isfinite(res["values"]), valid_o)
    for b in range(len(valid_o)):
        if valid_o[b]:
            assert res["used_w"][b] == b
        else:
            assert res["used_w"][b] == -1 and res["sets"][b] == []
    # reachable budgets are exactly the subset sums
    assert abs(res["values"][-1] - 1.0) <= 1e-6


PRUNE_CASES = [("tiny", None, "at_most", 0.9992, None), ("tiny", None, "exact", None, 14),
               ("small", 4, "at_most", 0.8, 32), ("small", None, "at_most", 0.85, 128),
               ("small", None, "exact", 0.85, 128)]


@pytest.mark.parametrize("name,n_layers,mode,tau,cap", PRUNE_CASES)
def test_pruning_rules_match_oracle(name, n_layers, mode, tau, cap):
    """Cosine threshold and skip cap (the review's tau and K/2): the cells each
    rule drops must be the oracle's, up to cells whose value is within the
    near-tie distance of tau (treated like near-ties)."""
    wl, inp, g, solver, res, orc, w, t = solved(name, n_layers, mode, tau, cap)
    rep = compare_solve(orc, res, w, VAL_TOL[wl.wdtype], wl.n_items, rows_val_gpu=res["rows"],
                        prune_tau=tau)
    valid_o = orc.dp.valid[-1]
    dropped = int((~valid_o).sum())
    print(f"\n{name}/{n_layers} {mode} tau={tau} cap={cap}: {dropped} of {len(valid_o)} final "
          f"cells dropped; {rep}")
    rep.assert_ok()
    ok = ~np.isnan(orc.values) | ~np.isnan(res["values"])
    kept = np.where(orc.dp.bp == 1, orc.dp.cos_e, orc.dp.cos_s)
    near = (np.abs(np.nan_to_num(kept, nan=np.inf) - (tau if tau is not None else -9)) < 1e-4).any(0)
    # validity agrees wherever no near-threshold cell could have flipped it
    if not near.any():
        assert np.array_equal(np.isnan(res["values"]), np.isnan(orc.values))
    if cap is not None:
        K = sum(w)
        assert np.all(np.isnan(res["values"][:max(0, K - cap)]))


def test_small_first_8_items_bounded_by_exhaustive_search():
    wl, inp, g, solver, res, orc, w, t = solved("small", 4)
    best, _ = O.brute_force(oracle_model(inp), x0_np(inp), wl.ctx, w, orc.ref)
    assert np.all(res["values"] <= best + VAL_TOL["bf16"])
    gaps = int(np.sum(res["values"] < best - VAL_TOL["bf16"]))
    print(f"\nsmall/8 items: GPU DP below the exhaustive optimum at {gaps} of {len(best)} budgets")


def test_solve_is_deterministic_and_given_ref_path_agrees():
    wl, inp, g, solver, res, orc, w, t = solved("small", 4)
    solver.solve(g.x0)
    again = gpu_result(solver)
    for k in ("bp", "values", "used_w", "t_draft", "best", "ref"):
        assert np.array_equal(res[k], again[k]), k
    ref = solver.out.ref_states.clone()
    solver.solve(g.x0, ref=ref)
    given = gpu_result(solver)
    for k in ("bp", "values", "best"):
        assert np.array_equal(res[k], given[k]), k


def test_tiny_tpt_and_latency_outputs():
    wl, inp, g, solver, res, orc, w, t = solved("tiny")
    # the draft latencies are sums of the raw latencies over each set
    for b, items in enumerate(res["sets"]):
        acc = 0.0
        for k in items:
            acc += t[k]
        assert res["t_draft"][b] == acc
    grid = solver.out.tpt.cpu().numpy()
    b, gm = res["best"]
    assert grid[b, gm - 1] == np.nanmax(grid)


@pytest.mark.parametrize("name,mode,dedup", [("tiny", "at_most", True), ("small", "at_most", True),
                                             ("small", "at_most", "weak"), ("small", "exact", True)])
def test_distinct_state_solve_matches_oracle(name, mode, dedup):
    """Distinct-state execution compared with the oracle directly (not only with
    the dense GPU solve): same rule, same tolerances."""
    wl, inp, g, solver, res, orc, w, t = solved(name, None, mode)
    m = B.model_desc(wl.n_layers, wl.d_model, wl.n_q_heads, wl.n_kv_heads, wl.head_dim, wl.ffn,
                     wl.rms_eps, wl.rope_base, wl.wdtype)
    s = B.Solver(m, g.layers, g.k_cache, g.v_cache, wl.ctx, wl.T, t,
                 B.params(wl.gamma_max, wl.n_bins, budget_mode=mode, dedup=dedup), w=w,
                 keep_cos=True)
    s.solve(g.x0)
    dd = gpu_result(s)
    rep = compare_solve(orc, dd, w, VAL_TOL[wl.wdtype], wl.n_items, rows_val_gpu=dd["rows"])
    print(f"\n{name} {mode} dedup={dedup}: executed {int(s.out.exec_counts.sum())} states, "
          f"byte check rejected {int(s.out.dedup_rejected.sum())} fingerprint matches; {rep}")
    rep.assert_ok()


@pytest.mark.parametrize("name", ["tiny", "small"])
def test_solve_on_the_full_model_cache_matches_oracle(name):
    """The configurations' "KV cache from the full model": the cache is the
    full model's own prefill over ctx + T tokens (oracle fp64, stored in the
    workload's dtype), x0 the last T tokens' embeddings; full grid, taint rule."""
    from tests._util import prefilled_inputs
    inp = prefilled_inputs(name)
    wl = inp.wl
    t = wl.latencies()
    w = O.quantize_weights(t, wl.n_bins)
    g = inp.to("cuda")
    solver = make_solver(wl, g, w=w, t=t)
    solver.solve(g.x0)
    res = gpu_result(solver)
    orc = O.dp_solve(oracle_model(inp), x0_np(inp), wl.ctx, w, t, wl.gamma_max,
                     per_cell=(wl.wdtype == "f32"))
    rep = compare_solve(orc, res, w, VAL_TOL[wl.wdtype], wl.n_items, rows_val_gpu=res["rows"])
    print(f"\n{name} on the full model's cache: best (b={orc.best_b}, gamma={orc.best_gamma}), "
          f"min final value {np.nanmin(orc.values):.4f}; {rep}")
    rep.assert_ok()
