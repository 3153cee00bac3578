"""GPU parity of each step of the hot path against the oracle, through the C ABI.

select (a4), reconstruct (a5), TPT (a6), each sublayer (a2/a3) and the
reference chain (a1) on seeded inputs that span several tiles, ragged tails and
the degenerate cases (no cell can execute, exact ties, C = 1).
"""
import numpy as np
import pytest
import torch

from knapsack_layer_selection_b200 import binding as B
from knapsack_layer_selection_b200 import build as BUILD
from knapsack_layer_selection_b200 import workloads as W
from oracle import ks_oracle as O
from tests._util import oracle_model, x0_np

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    BUILD.build()
    return B.load()


def _states(shape, seed):
    return W.random_states(shape, seed)


# ---------------------------------------------------------------- a4 select
SELECT_CASES = [(1, 1, 4, 1), (7, 3, 64, 2), (37, 4, 256, 5), (129, 16, 4096, 14),
                (5, 2, 132, 9), (300, 8, 1024, 1)]


@pytest.mark.parametrize("C,T,d,w", SELECT_CASES)
def test_select_step_matches_oracle(C, T, d, w):
    g = torch.Generator().manual_seed(C * 131 + d)
    target = _states((T, d), 1)
    # candidates scattered around the target at different distances, so both
    # choices occur; a few execute candidates tie the skip candidate exactly
    prev = target + torch.randn(C, T, d, generator=g) * torch.rand(C, 1, 1, generator=g) * 2
    E = max(C - w, 0)
    exe = target + torch.randn(max(E, 1), T, d, generator=g) * torch.rand(max(E, 1), 1, 1, generator=g) * 2
    for e in range(0, E, 5):
        exe[e] = prev[e + w]
    if E > 3:
        exe[3] = target
    dev = "cuda"
    prev_d, exe_d, tgt_d = prev.to(dev), exe.to(dev), target.to(dev)
    cur = torch.empty_like(prev_d)
    val = torch.empty(C, device=dev)
    bp = torch.empty(C, dtype=torch.uint8, device=dev)
    cs = torch.empty(C, device=dev)
    ce = torch.empty(C, device=dev)
    B.select_step(prev_d, exe_d, tgt_d, w, cur, val, bp, cs, ce)
    torch.cuda.synchronize()

    tnp = target.double().numpy()
    res = O.knapsack_dp([w], C, prev.double().numpy(), np.ones(C, bool),
                        lambda k, H: exe[:E].double().numpy()[:len(H)],
                        lambda r, H: O.meancos(H, tnp))
    bp_o = res.bp[0]
    near = np.abs(np.nan_to_num(res.cos_e[0], nan=9) - res.cos_s[0]) < 1e-12
    bp_g = bp.cpu().numpy()
    assert np.all((bp_g == bp_o) | near)
    assert np.allclose(cs.cpu().numpy(), res.cos_s[0], rtol=0, atol=1e-6)
    ce_g = ce.cpu().numpy()
    assert np.all(np.isnan(ce_g[:w]))
    assert np.allclose(ce_g[w:], res.cos_e[0][w:], rtol=0, atol=1e-6)
    assert np.allclose(val.cpu().numpy(), res.val[1], rtol=0, atol=1e-6)
    # exact ties keep the skip state; the target itself scores exactly 1
    for e in range(0, E, 5):
        if e != 3:
            assert bp_g[e + w] == 0
    if E > 3:
        assert val[3 + w].item() == 1.0 and bp_g[3 + w] == 1
    # the winner is copied bit for bit
    cur_c = cur.cpu()
    for b in range(C):
        src = exe[b - w] if bp_g[b] else prev[b]
        assert torch.equal(cur_c[b], src)


# ---------------------------------------------------------------- a5 reconstruct
@pytest.mark.parametrize("n,C", [(1, 1), (8, 29), (32, 257), (64, 513), (128, 1025), (130, 700)])
def test_reconstruct_matches_oracle(n, C):
    rng = np.random.default_rng(n * 7 + C)
    w = rng.integers(1, 9, size=n).astype(np.int32)
    t = rng.uniform(0.5, 40.0, size=n)
    bp = (rng.random((n, C)) < 0.5).astype(np.uint8)
    for k in range(n):
        bp[k, :min(C, w[k])] = 0           # no execute below the item's weight
    dev = "cuda"
    words = (n + 63) // 64
    sets = torch.zeros(C, words, dtype=torch.int64, device=dev)
    used = torch.zeros(C, dtype=torch.int32, device=dev)
    td = torch.zeros(C, dtype=torch.float64, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    B.reconstruct(torch.from_numpy(bp).to(dev), torch.from_numpy(w).to(dev),
                  torch.from_numpy(t).to(dev), sets, used, td, status)
    torch.cuda.synchronize()
    assert status.item() == 0
    got = B.sets_to_lists(sets, n)
    used_g, td_g = used.cpu().numpy(), td.cpu().numpy()
    for b in range(C):
        items, u = O.reconstruct(bp, w, b)
        assert got[b] == items
        assert used_g[b] == u
        acc = 0.0
        for k in items:
            acc += float(t[k])
        assert td_g[b] == acc


def test_reconstruct_flags_a_walk_that_leaves_the_grid():
    # bp says "execute" at a cell below the item's weight: the walk would go
    # negative; the kernel reports KS_ERR_INTERNAL instead of reading out of range
    dev = "cuda"
    bp = torch.ones(2, 3, dtype=torch.uint8, device=dev)
    w = torch.tensor([2, 2], dtype=torch.int32, device=dev)
    t = torch.tensor([1.0, 1.0], dtype=torch.float64, device=dev)
    sets = torch.zeros(3, 1, dtype=torch.int64, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    B.reconstruct(bp, w, t, sets, None, None, status)
    torch.cuda.synchronize()
    assert status.item() == 6


# ---------------------------------------------------------------- a6 TPT
@pytest.mark.parametrize("C,G", [(1, 1), (29, 8), (513, 10), (1025, 10), (3000, 7)])
def test_tpt_matches_oracle(C, G):
    rng = np.random.default_rng(C + G)
    vals = rng.uniform(0.3, 1.0, C).astype(np.float32)
    td = rng.uniform(0.0, 300.0, C)
    # duplicated cells (a skip-only carry repeats a set): exact TPT ties
    for b in range(1, C, 7):
        vals[b] = vals[b - 1]
        td[b] = td[b - 1]
    vals[C // 2] = 1.0
    td[0] = 0.0
    t_target = 512.0
    dev = "cuda"
    prm = B.params(G)
    grid = torch.zeros(C, G, dtype=torch.float64, device=dev)
    best = torch.zeros(2, dtype=torch.int32, device=dev)
    bt = torch.zeros(1, dtype=torch.float64, device=dev)
    B.tpt_argmax(torch.from_numpy(vals).to(dev), torch.from_numpy(td).to(dev), t_target, prm,
                 grid, best, bt)
    torch.cuda.synchronize()
    og = O.tpt_grid(vals.astype(np.float64), td, t_target, G)
    assert np.array_equal(grid.cpu().numpy(), og)          # same fp64 operations, same order
    ob, ogam, ov = O.tpt_argmax(og)
    assert (best[0].item(), best[1].item()) == (ob, ogam)
    assert bt.item() == ov


def test_tpt_skips_non_finite_cells():
    dev = "cuda"
    vals = torch.tensor([float("nan"), 0.9, 0.9], device=dev)
    td = torch.tensor([0.0, 10.0, 10.0], dtype=torch.float64, device=dev)
    best = torch.zeros(2, dtype=torch.int32, device=dev)
    B.tpt_argmax(vals, td, 100.0, B.params(3), None, best, None)
    torch.cuda.synchronize()
    assert best.tolist() == [1, 3]


# ---------------------------------------------------------------- a2/a3 sublayers, a1 reference
def _gpu_ctx(wl, inp):
    g = inp.to("cuda")
    m = B.model_desc(wl.n_layers, wl.d_model, wl.n_q_heads, wl.n_kv_heads, wl.head_dim, wl.ffn,
                     wl.rms_eps, wl.rope_base, wl.wdtype)
    layers = B.layer_array(g.layers, W.torch_dtype(wl))
    cache = B.cache_desc(g.k_cache, g.v_cache, wl.ctx)
    return g, m, layers, cache


def _branch_rel_err(out_g, out_o, H):
    bg = out_g - H
    bo = out_o - H
    return float(np.linalg.norm(bg - bo) / np.linalg.norm(bo))


SUBLAYER_TOL = {"f32": 1e-5, "bf16": 1e-2}


@pytest.mark.parametrize("name,items,E", [("tiny", list(range(8)), 9),
                                          ("small", [0, 1, 30, 31], 37)])
def test_sublayers_match_oracle(name, items, E):
    wl = W.WORKLOADS[name]
    inp = W.make_inputs(wl)
    g, m, layers, cache = _gpu_ctx(wl, inp)
    om = oracle_model(inp)
    H = _states((E, wl.T, wl.d_model), 11)
    H[2] = H[1]                                       # two identical states
    Hd = H.cuda()
    ws = B.workspace(m, E, wl.T)
    for k in items:
        out = torch.empty_like(Hd)
        B.sublayer_forward(m, layers, cache, wl.T, k, Hd, out, ws)
        one = torch.empty_like(Hd[:1])
        B.sublayer_forward(m, layers, cache, wl.T, k, Hd[1:2].contiguous(), one, ws)
        torch.cuda.synchronize()
        og = O.apply_item(om, k, H.double().numpy(), wl.ctx)
        err = _branch_rel_err(out.double().cpu().numpy(), og, H.double().numpy())
        assert err < SUBLAYER_TOL[wl.wdtype], (k, err)
        # a state's result does not depend on the batch it sits in
        assert torch.equal(out[1], out[2])
        assert torch.equal(out[1], one[0])


@pytest.mark.parametrize("name", ["tiny", "small"])
def test_reference_forward_matches_oracle(name):
    wl = W.WORKLOADS[name]
    inp = W.make_inputs(wl)
    g, m, layers, cache = _gpu_ctx(wl, inp)
    ws = B.workspace(m, 1, wl.T)
    ref = torch.empty(wl.n_items + 1, wl.T, wl.d_model, device="cuda")
    B.reference_forward(m, layers, cache, wl.T, g.x0, ref, ws)
    torch.cuda.synchronize()
    oref = O.reference_states(oracle_model(inp), x0_np(inp), wl.ctx)
    r = ref.double().cpu().numpy()
    assert np.array_equal(r[0], oref[0])
    tol = 1e-5 if wl.wdtype == "f32" else 2e-2
    for k in range(1, wl.n_items + 1):
        rel = np.linalg.norm(r[k] - oref[k]) / np.linalg.norm(oref[k])
        assert rel < tol, (k, rel)
        assert O.meancos(r[k][None], oref[k])[0] > 1 - 1e-4
