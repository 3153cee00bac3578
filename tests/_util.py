"""Test helpers: hand the seeded inputs to the oracle as numpy arrays."""
import numpy as np
import torch

from oracle import ks_oracle as O


class _LazyLayers:
    """Widen one layer's torch tensors to numpy float32 only when it is used."""

    def __init__(self, layers):
        self._layers = layers
        self._last = (None, None)

    def __len__(self):
        return len(self._layers)

    def __getitem__(self, i):
        if self._last[0] != i:
            self._last = (i, {k: v.detach().float().cpu().numpy()
                              for k, v in self._layers[i].items()})
        return self._last[1]


class _LazyCache:
    def __init__(self, cache):
        self._c = cache

    def __len__(self):
        return self._c.shape[0]

    def __getitem__(self, i):
        return self._c[i].detach().float().cpu().numpy()


def oracle_model(inp) -> O.Model:
    wl = inp.wl
    return O.Model(wl.n_q_heads, wl.n_kv_heads, wl.head_dim, wl.rms_eps, wl.rope_base,
                   _LazyLayers(inp.layers), _LazyCache(inp.k_cache), _LazyCache(inp.v_cache))


def x0_np(inp) -> np.ndarray:
    return inp.x0.detach().double().cpu().numpy()


def prefilled_inputs(name: str):
    """The workload's seeded weights (with Wk / Wv) and the KV cache "from the
    full model": the oracle's prefill over ctx + T seeded token embeddings, in
    the workload's storage dtype; x0 = the last T embeddings.  Test input only."""
    import dataclasses

    from knapsack_layer_selection_b200 import workloads as W
    wl = W.WORKLOADS[name]
    inp = W.make_inputs(wl)
    ww = W.window_weights(wl)
    inp = dataclasses.replace(inp, layers=[{**L, **w} for L, w in zip(inp.layers, ww)])
    m = oracle_model(inp)
    m = dataclasses.replace(m, layers=[m.layers[i] for i in range(len(m.layers))])
    emb = W.sequence_embeddings(wl)
    pf = O.prefill(m, emb.double().numpy())
    dt = W.torch_dtype(wl)
    kc = torch.from_numpy(pf.k_cache).to(dt)
    vc = torch.from_numpy(pf.v_cache).to(dt)
    return dataclasses.replace(inp, k_cache=kc, v_cache=vc, x0=emb[-wl.T:].contiguous())
