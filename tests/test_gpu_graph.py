"""A whole solve is stream-ordered work with no host synchronisation inside, so
it captures into a CUDA graph; the replayed graph must give the launched solve's
values, sets, backpointers and (b*, gamma*) bit for bit (dense and
distinct-state, on the small GQA workload)."""
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


@pytest.mark.parametrize("dedup", [False, True])
def test_solve_replayed_from_a_cuda_graph_is_bit_identical(dedup):
    wl = W.WORKLOADS["small"]
    inp = W.make_inputs(wl).to("cuda")
    m = B.model_desc(wl.n_layers, wl.d_model, wl.n_q_heads, wl.n_kv_heads, wl.head_dim, wl.ffn,
                     wl.rms_eps, wl.rope_base, wl.wdtype)
    s = B.Solver(m, inp.layers, inp.k_cache, inp.v_cache, wl.ctx, wl.T, wl.latencies(),
                 B.params(wl.gamma_max, wl.n_bins, dedup=dedup))
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):          # warm up off the capture stream
        s.solve(inp.x0)
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    s.check_status()
    ref = {k: getattr(s.out, k).clone() for k in ("values", "sets", "bp", "best")}
    for k in ("values", "sets", "bp"):
        getattr(s.out, k).zero_()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        s.solve(inp.x0)
    for _ in range(2):
        g.replay()
    torch.cuda.synchronize()
    s.check_status()
    for k, v in ref.items():
        assert torch.equal(getattr(s.out, k), v), k
    del g
