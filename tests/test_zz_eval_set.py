"""ks_eval_set on the GPU: a layer set re-run from scratch (only its items, in
order, on x0) reproduces the DP's value for its cell -- up to the rounding of
the normalised operand, which the solve fuses into its select step -- and the
oracle's value of the same set within the DP's own tolerance."""
import numpy as np
import pytest
import torch

from knapsack_layer_selection_b200 import binding as B
from knapsack_layer_selection_b200 import workloads as W
from oracle import ks_oracle as O
from tests._util import oracle_model, x0_np

TOL = {"f32": 1e-5, "bf16": 2e-3}


@pytest.mark.gpu
@pytest.mark.parametrize("name", ["tiny", "small"])
def test_eval_set_reproduces_dp_values_and_the_oracle(name):
    wl = W.WORKLOADS[name]
    inp = W.make_inputs(wl)
    g = inp.to("cuda")
    m = B.model_desc(wl.n_layers, wl.d_model, wl.n_q_heads, wl.n_kv_heads, wl.head_dim, wl.ffn,
                     wl.rms_eps, wl.rope_base, wl.wdtype)
    s = B.Solver(m, g.layers, g.k_cache, g.v_cache, wl.ctx, wl.T, wl.latencies(),
                 B.params(wl.gamma_max, wl.n_bins))
    out = s.solve(g.x0)
    torch.cuda.synchronize()
    s.check_status()
    sets = B.sets_to_lists(out.sets, s.n_items)
    values = out.values.cpu().numpy()
    target = out.ref_states[-1].contiguous()              # X^(2L) of the solve
    ws = B.workspace(m, 1, wl.T)
    val = torch.empty(1, device="cuda")
    state = torch.empty(wl.T, wl.d_model, device="cuda")
    om = oracle_model(inp)
    x0 = x0_np(inp)
    ref_o = O.reference_states(om, x0, wl.ctx)
    for b in sorted(set(np.linspace(0, s.C - 1, 9).astype(int).tolist())):
        B.eval_set(m, s.layers, s.cache, wl.T, g.x0, target, sets[b], ws, val, state)
        torch.cuda.synchronize()
        assert B.workspace_status(ws) == 0
        v = val.item()
        assert abs(v - values[b]) <= TOL[wl.wdtype], (b, v, values[b])
        vo = O.eval_set(om, x0, wl.ctx, sets[b], ref_o)
        assert abs(v - vo) <= TOL[wl.wdtype], (b, v, vo)
    # the empty set leaves x0 as it is, and a state scores exactly 1 on itself
    B.eval_set(m, s.layers, s.cache, wl.T, g.x0, g.x0, [], ws, val, state)
    torch.cuda.synchronize()
    assert torch.equal(state, g.x0) and val.item() == 1.0
