"""The allocation-free reference forward agrees with the workspace version.

ks_reference_forward_noalloc exists for callers that cannot hand the library a
device workspace: code that runs where new device allocations are not allowed
(a serving loop whose memory pool is fixed once it starts, a plugin host that
only passes input and output buffers).  It keeps its scratch in one fixed
device array inside the library instead.  These checks call it through the C
ABI twice in a row, with different inputs, and compare each result with
ks_reference_forward on a caller-provided workspace; the shared array must not
carry anything from one call into the next.  This file is collected last so a
run that stops at the first failure has already run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

from knapsack_layer_selection_b200 import binding as B
from knapsack_layer_selection_b200 import build as BUILD
from knapsack_layer_selection_b200 import workloads as W

pytestmark = pytest.mark.gpu

# the relative tolerances the reference-state tests use (fp32 / bf16 models)
REL_TOL = {"f32": 1e-5, "bf16": 2e-2}


@pytest.fixture(scope="module", autouse=True)
def lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    BUILD.build()
    return B.load()


@pytest.mark.parametrize("name", ["tiny", "small"])
def test_noalloc_reference_forward_matches_workspace_version(name):
    wl = W.WORKLOADS[name]
    g = W.make_inputs(wl).to("cuda")
    m = B.model_desc(wl.n_layers, wl.d_model, wl.n_q_heads, wl.n_kv_heads, wl.head_dim, wl.ffn,
                     wl.rms_eps, wl.rope_base, wl.wdtype)
    layers = B.layer_array(g.layers, W.torch_dtype(wl))
    cache = B.cache_desc(g.k_cache, g.v_cache, wl.ctx)
    ws = B.workspace(m, 1, wl.T)
    x0_a = g.x0
    x0_b = W.random_states((wl.T, wl.d_model), 99).cuda()
    shape = (wl.n_items + 1, wl.T, wl.d_model)
    for x0 in (x0_a, x0_b):                       # two calls in a row, different inputs
        want = torch.empty(shape, device="cuda")
        got = torch.full(shape, float("nan"), device="cuda")
        B.reference_forward(m, layers, cache, wl.T, x0, want, ws)
        B.reference_forward_noalloc(m, layers, cache, wl.T, x0, got)
        torch.cuda.synchronize()
        assert torch.isfinite(got).all()
        for k in range(shape[0]):
            rel = float((got[k] - want[k]).norm() / want[k].norm())
            assert rel <= REL_TOL[wl.wdtype], (name, k, rel)
        # same kernels on the same operands: in practice the two agree bit for bit
        print(f"\n{name}: max |noalloc - workspace| = {float((got - want).abs().max()):.3g}")


def test_noalloc_rejects_sizes_above_its_fixed_scratch():
    """A model/T whose scratch exceeds the fixed array is refused before any launch."""
    lib = B.load()
    wl = W.WORKLOADS["qwen3_32b_16k"]
    m = B.model_desc(wl.n_layers, wl.d_model, wl.n_q_heads, wl.n_kv_heads, wl.head_dim, wl.ffn,
                     wl.rms_eps, wl.rope_base, wl.wdtype)
    layers = (B.LayerWeights * wl.n_layers)()
    for i in range(wl.n_layers):
        for f, _ in B.LayerWeights._fields_:
            setattr(layers[i], f, 256)
    T = 64
    cache = B.CacheDesc(256, 256, wl.ctx + T, wl.ctx)
    st = lib.ks_reference_forward_noalloc(ctypes.byref(m), layers, ctypes.byref(cache), T,
                                          ctypes.c_void_p(256), ctypes.c_void_p(512), None)
    assert st == 2
    assert b"above the fixed" in lib.ks_last_error()
