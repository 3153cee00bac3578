"""GPU Lemma 4.1 checker (ks_lemma_check) against the oracle's fp64 checker.

The GPU rounds the normalised states and the LM head to bf16 for the logits
(fp32 accumulation), so decisions that floating point takes -- the greedy
token, the bound's comparison -- are compared where the oracle's margin or
slack is clear of that rounding; cosines (fp64 sums on both sides) are
compared tightly.  The lemma's implication (bound => agreement) is checked
where the slack is clear."""
import numpy as np
import pytest
import torch

from knapsack_layer_selection_b200 import binding as B
from knapsack_layer_selection_b200 import build as BUILD
from knapsack_layer_selection_b200 import workloads as W
from oracle import ks_oracle as O

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    BUILD.build()
    return B.load()


def compare(states, ref, head, gain=None, label=""):
    got = B.lemma_check(states.cuda(), ref.cuda(), head.cuda(),
                        None if gain is None else gain.cuda())
    torch.cuda.synchronize()
    g = {k: v.cpu().numpy() for k, v in got.items() if not k.startswith("_")}
    lc = O.lemma_check(states.double().numpy(), ref.double().numpy(), head.float().numpy(),
                       None if gain is None else gain.float().numpy(), 1e-6)
    d = states.shape[-1]
    zscale = float(np.linalg.norm(head.float().numpy(), axis=1).mean() * np.sqrt(d))
    tol_z = 3e-3 * zscale                      # bf16 operands of the logits
    assert np.allclose(g["cos"], lc.cos, atol=2e-6, rtol=0)
    clear = lc.margin > 2 * tol_z
    assert np.array_equal(g["istar"][clear], lc.istar[clear])
    assert np.allclose(g["margin"][clear], lc.margin[clear], atol=2 * tol_z, rtol=0)
    assert np.allclose(g["dist"][clear], lc.dist[clear], rtol=1e-2, atol=0)
    a_clear = (lc.state_margin > 2 * tol_z) & clear[None]
    assert np.array_equal(g["agree"][a_clear].astype(bool), lc.agree[a_clear])
    s_clear = (np.abs(lc.slack) > 2 * tol_z / lc.dist[None] + 1e-4) & clear[None]
    assert np.array_equal(g["bound"][s_clear].astype(bool), lc.bound[s_clear])
    # the lemma never fails where the decision is clear of rounding
    assert not np.any((g["bound"] == 1) & (g["agree"] == 0) & s_clear & a_clear)
    N, T = lc.cos.shape
    print(f"\n{label}: bound holds for {int(g['counts'][0])}/{N * T} tokens, greedy agrees for "
          f"{int(g['counts'][1])}/{N * T}, bound without agreement {int(g['counts'][2])} "
          f"(oracle: {int(lc.bound.sum())}, {int(lc.agree.sum())}, {int((lc.bound & ~lc.agree).sum())})")
    assert int(g["counts"][0]) == int(g["bound"].sum()) and int(g["counts"][1]) == int(g["agree"].sum())
    return g, lc


@pytest.mark.parametrize("d,V,N,T", [(64, 256, 3, 2), (128, 512, 6, 5), (256, 1024, 40, 4)])
def test_lemma_checker_synthetic(d, V, N, T):
    gen = torch.Generator().manual_seed(d + V)
    head = (torch.randn(V, d, generator=gen)).to(torch.bfloat16)
    ref = torch.randn(T, d, generator=gen)
    states = ref[None] + torch.randn(N, T, d, generator=gen) * torch.rand(N, 1, 1, generator=gen) * 0.5
    gain = (torch.rand(d, generator=gen) + 0.5).to(torch.bfloat16)
    compare(states, ref, head, None, f"synthetic d={d} V={V}")
    compare(states, ref, head, gain, f"synthetic d={d} V={V} with gain")


def test_lemma_checker_on_small_dp_states():
    wl = W.WORKLOADS["small"]
    g = W.make_inputs(wl).to("cuda")
    m = B.model_desc(wl.n_layers, wl.d_model, wl.n_q_heads, wl.n_kv_heads, wl.head_dim, wl.ffn,
                     wl.rms_eps, wl.rope_base, wl.wdtype)
    s = B.Solver(m, g.layers, g.k_cache, g.v_cache, wl.ctx, wl.T, wl.latencies(),
                 B.params(wl.gamma_max, wl.n_bins), keep_final=True)
    s.solve(g.x0)
    torch.cuda.synchronize()
    s.check_status()
    states = s.out.final_states.cpu()
    ref = s.out.ref_states[-1].cpu()
    assert torch.equal(states[-1], ref)            # the all-execute cell is the reference
    head = W.lm_head(wl, device="cpu")
    gres, lc = compare(states, ref, head, None, "small DP final states, V=8192")
    assert gres["agree"][-1].all() and gres["bound"][-1].all()   # h' = h: margin / D > 0
