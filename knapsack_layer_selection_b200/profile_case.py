"""A small, self-contained case for profiler captures of the hot kernels.

``--item attn|mlp`` runs one sublayer forward of a workload's shape -- the
Attention or the MLP item of one layer, over every budget cell that executes
it in the DP (E = C - w_item cells x T tokens) -- a few times, with one layer
of seeded weights and cache.  ``--item solve`` runs whole DP solves of a
two-layer model of the same shape whose four item weights are set so the
grid has the workload's full number of cells (every kernel of the loop, the
select step included, at full width).  About 2-3 GB on the device for the 8B
shape, so a profiler can replay its kernels quickly.

    python -m knapsack_layer_selection_b200.profile_case --workload llama3_8b_8k --item attn
"""
from __future__ import annotations

import argparse
import dataclasses

import torch

from knapsack_layer_selection_b200 import binding as B
from knapsack_layer_selection_b200 import build as BUILD
from knapsack_layer_selection_b200 import workloads as W


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--workload", default="llama3_8b_8k", choices=sorted(W.WORKLOADS))
    ap.add_argument("--item", choices=["attn", "mlp", "solve"], default="attn")
    ap.add_argument("--repeat", type=int, default=2)
    a = ap.parse_args()
    BUILD.build()
    full = W.WORKLOADS[a.workload]
    if a.item == "solve":
        return solve_case(full, a.repeat)
    wl = dataclasses.replace(full, n_layers=1)
    inp = W.make_inputs(wl, device="cuda")
    t = full.latencies()
    w = B.quantize_weights(t, full.n_bins)
    C = sum(w) + 1
    item = 0 if a.item == "attn" else 1
    E = C - w[item]
    m = B.model_desc(1, wl.d_model, wl.n_q_heads, wl.n_kv_heads, wl.head_dim, wl.ffn,
                     wl.rms_eps, wl.rope_base, wl.wdtype)
    layers = B.layer_array(inp.layers, W.torch_dtype(wl))
    cache = B.cache_desc(inp.k_cache, inp.v_cache, wl.ctx)
    states = W.random_states((E, wl.T, wl.d_model), 1, device="cuda")
    out = torch.empty_like(states)
    ws = B.workspace(m, E, wl.T)
    for _ in range(a.repeat):
        B.sublayer_forward(m, layers, cache, wl.T, item, states, out, ws)
    torch.cuda.synchronize()
    st = B.workspace_status(ws)
    if st != 0:
        raise SystemExit(f"device status {st}")
    print(f"{a.workload} {a.item}: {E} cells x {wl.T} tokens, {a.repeat} forward(s) ok")


def solve_case(full, repeat):
    wl = dataclasses.replace(full, n_layers=2)
    inp = W.make_inputs(wl, device="cuda")
    K = sum(B.quantize_weights(full.latencies(), full.n_bins))
    w = [K // 4] * 3 + [K - 3 * (K // 4)]          # four items spanning the full grid
    t = wl.latencies()
    m = B.model_desc(2, wl.d_model, wl.n_q_heads, wl.n_kv_heads, wl.head_dim, wl.ffn,
                     wl.rms_eps, wl.rope_base, wl.wdtype)
    s = B.Solver(m, inp.layers, inp.k_cache, inp.v_cache, wl.ctx, wl.T, t,
                 B.params(wl.gamma_max, full.n_bins), w=w, keep_bp=True, keep_tpt=False,
                 keep_ref=False)
    for _ in range(repeat):
        s.solve(inp.x0)
    torch.cuda.synchronize()
    s.check_status()
    # per item: the cells whose execute candidate won (the select writes only
    # those states; the others stay in place)
    takes = s.out.bp.to(torch.int64).sum(dim=1).tolist()
    print(f"{full.name} solve: 2 layers, {s.C} cells x {wl.T} tokens, {repeat} solve(s) ok; "
          f"item weights {w}, execute wins per item {takes}")


if __name__ == "__main__":
    main()
