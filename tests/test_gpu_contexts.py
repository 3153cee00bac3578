"""The DP re-solved at several contexts in one pass (ks_solve_contexts) equals
the separate solves bit for bit: every context keeps its own item weights,
budget grid, reference states and attention window, and only the weight reads
of the GEMMs are shared.  Checked on the tiny (fp32, CUDA-core kernels) and
small (bf16, tensor cores; cache and window readings) workloads, and on the
Llama-3-8B shape re-solved at 4k, 16k and 32k context -- the re-solve the
review describes as the context grows -- where both ways are also timed.
"""
import dataclasses

import numpy as np
import pytest
import torch

from knapsack_layer_selection_b200 import binding as B
from knapsack_layer_selection_b200 import build as BUILD
from knapsack_layer_selection_b200 import workloads as W

pytestmark = pytest.mark.gpu

FIELDS = ("bp", "values", "sets", "used_w", "t_draft", "best", "best_tpt", "tpt", "ref_states",
          "exec_counts")


@pytest.fixture(scope="module", autouse=True)
def lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    BUILD.build()
    return B.load()


def model_of(wl):
    return B.model_desc(wl.n_layers, wl.d_model, wl.n_q_heads, wl.n_kv_heads, wl.head_dim, wl.ffn,
                        wl.rms_eps, wl.rope_base, wl.wdtype)


def separate(wl, g, ctxs, x0s, kv="cache"):
    outs, solvers = [], []
    for ctx, x0 in zip(ctxs, x0s):
        wc = wl.with_ctx(ctx)
        s = B.Solver(model_of(wl), g.layers, g.k_cache, g.v_cache, ctx, wl.T, wc.latencies(),
                     B.params(wl.gamma_max, wl.n_bins), keep_cos=False, kv=kv)
        s.solve(x0)
        solvers.append(s)
        outs.append(s.out)
    torch.cuda.synchronize()
    for s in solvers:
        s.check_status()
    return solvers, outs


def batched(wl, g, ctxs, x0s, kv="cache"):
    mc = B.SolverContexts(model_of(wl), g.layers, [(g.k_cache, g.v_cache, c) for c in ctxs], wl.T,
                          [wl.with_ctx(c).latencies() for c in ctxs],
                          B.params(wl.gamma_max, wl.n_bins), kv=kv)
    outs = mc.solve(x0s)
    torch.cuda.synchronize()
    mc.check_status()
    return mc, outs


def assert_same(a, b, label):
    for f in FIELDS:
        x, y = getattr(a, f), getattr(b, f)
        assert torch.equal(x.cpu(), y.cpu()) if x.dtype != torch.float32 else \
            np.array_equal(x.cpu().numpy(), y.cpu().numpy(), equal_nan=True), (label, f)


@pytest.mark.parametrize("name,ctxs,kv", [("tiny", (64, 100, 128), "cache"),
                                          ("small", (512, 1000, 2048), "cache"),
                                          ("small", (2048, 700), "window"),
                                          ("small", (1024,), "cache")])
def test_contexts_in_one_pass_equal_separate_solves(name, ctxs, kv):
    wl = W.WORKLOADS[name]
    inp = W.make_inputs(wl)
    if kv == "window":
        ww = W.window_weights(wl)
        inp = dataclasses.replace(inp, layers=[{**L, **w} for L, w in zip(inp.layers, ww)])
    g = inp.to("cuda")
    # a different evaluation window per context (the last T tokens at each re-solve)
    x0s = [g.x0] + [W.random_states((wl.T, wl.d_model), 100 + j, device="cuda")
                    for j in range(1, len(ctxs))]
    solvers, sep = separate(wl, g, ctxs, x0s, kv)
    mc, bat = batched(wl, g, ctxs, x0s, kv)
    for j, c in enumerate(ctxs):
        assert mc.C[j] == solvers[j].C and mc.w[j] == solvers[j].w
        assert_same(sep[j], bat[j], f"{name} ctx {c}")
    print(f"\n{name} {kv}: contexts {ctxs}, cells {mc.C}, best "
          f"{[tuple(o.best.tolist()) for o in bat]}: one pass equals the separate solves")


def test_llama3_8b_resolve_at_4k_16k_32k_in_one_pass():
    """The 32k workload re-solved at 4k / 16k / 32k: one pass against three
    separate solves, bit for bit, and both timed (CUDA events, warm)."""
    name = "llama3_8b_32k"
    wl = W.WORKLOADS[name]
    inp = W.make_inputs(wl)
    g = inp if inp.x0.is_cuda else inp.to("cuda")
    del inp
    ctxs = tuple(wl.contexts)
    x0s = [g.x0] * len(ctxs)
    solvers, sep = separate(wl, g, ctxs, x0s)
    mc, bat = batched(wl, g, ctxs, x0s)
    for j, c in enumerate(ctxs):
        assert_same(sep[j], bat[j], f"8B ctx {c}")
    # timing: warm, then 2 of each
    ev = lambda: torch.cuda.Event(enable_timing=True)
    e0, e1, e2 = ev(), ev(), ev()
    e0.record()
    for _ in range(2):
        for s in solvers:
            s.solve(g.x0)
    e1.record()
    for _ in range(2):
        mc.solve(x0s)
    e2.record()
    torch.cuda.synchronize()
    t_sep, t_bat = e0.elapsed_time(e1) / 2, e1.elapsed_time(e2) / 2
    print(f"\n8B @ contexts {ctxs}: cells {mc.C}, best {[tuple(o.best.tolist()) for o in bat]}; "
          f"three separate solves {t_sep:.1f} ms, one pass {t_bat:.1f} ms "
          f"({(t_sep - t_bat) / t_sep:+.1%})")
