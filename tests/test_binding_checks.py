"""The binding's shape checks: the C ABI takes bare pointers, so every shape
the header fixes is checked in Python before a pointer is taken.  On a CPU machine
a correctly shaped CPU tensor gets as far as the pointer step and is refused
there ("must be a CUDA tensor"); a wrongly shaped one is refused earlier, by
name and shape.  No GPU needed, nothing reaches a kernel."""
import pytest
import torch

from knapsack_layer_selection_b200 import binding as B
from knapsack_layer_selection_b200 import workloads as W

NOT_CUDA = "must be a CUDA tensor"


def _t(*shape, dtype=torch.float32):
    return torch.zeros(*shape, dtype=dtype)


def _bf(*shape):
    return _t(*shape, dtype=torch.bfloat16)


def _model(wl):
    return B.model_desc(wl.n_layers, wl.d_model, wl.n_q_heads, wl.n_kv_heads, wl.head_dim,
                        wl.ffn, wl.rms_eps, wl.rope_base, wl.wdtype)


def test_gemm_shapes():
    A, Bw, C = _bf(4, 64), _bf(256, 64), _t(4, 256)
    with pytest.raises(B.KnapSpecError, match=NOT_CUDA):
        B.gemm_bf16(A, Bw, C)
    with pytest.raises(B.KnapSpecError, match=r"B must have shape \(256, 64\)"):
        B.gemm_bf16(A, _bf(256, 128), C)
    with pytest.raises(B.KnapSpecError, match=r"C must have shape \(4, 256\)"):
        B.gemm_bf16(A, Bw, _t(3, 256))
    with pytest.raises(B.KnapSpecError, match="resid must have shape"):
        B.gemm_bf16(A, Bw, C, resid=_t(4, 255))
    with pytest.raises(B.KnapSpecError, match="status must hold one int32"):
        B.gemm_bf16(A, Bw, C, status=torch.zeros(0, dtype=torch.int32))


def test_attention_shapes():
    q, k, out = _bf(20, 8, 64), _bf(100, 2, 64), _bf(20, 8, 64)
    with pytest.raises(B.KnapSpecError, match=NOT_CUDA):
        B.attention_bf16(q, k, k.clone(), 4, 90, out)
    with pytest.raises(B.KnapSpecError, match="v_layer must have shape"):
        B.attention_bf16(q, k, _bf(99, 2, 64), 4, 90, out)
    with pytest.raises(B.KnapSpecError, match="k_layer must have shape"):
        B.attention_bf16(q, _bf(100, 2, 128), _bf(100, 2, 128), 4, 90, out)
    with pytest.raises(B.KnapSpecError, match="out must have shape"):
        B.attention_bf16(q, k, k.clone(), 4, 90, _bf(19, 8, 64))


def test_select_shapes():
    C, T, d, w = 10, 3, 8, 4
    prev, exe, tgt, cur = _t(C, T, d), _t(C - w, T, d), _t(T, d), _t(C, T, d)
    val, bp = _t(C), _t(C, dtype=torch.uint8)
    with pytest.raises(B.KnapSpecError, match=NOT_CUDA):
        B.select_step(prev, exe, tgt, w, cur, val, bp)
    # a longer exec buffer is fine (only its first C - w rows are read)
    with pytest.raises(B.KnapSpecError, match=NOT_CUDA):
        B.select_step(prev, _t(C, T, d), tgt, w, cur, val, bp)
    with pytest.raises(B.KnapSpecError, match=r"exec must have shape \(>= 6, 3, 8\)"):
        B.select_step(prev, _t(C - w - 1, T, d), tgt, w, cur, val, bp)
    with pytest.raises(B.KnapSpecError, match="target must have shape"):
        B.select_step(prev, exe, _t(T, d + 4), w, cur, val, bp)
    with pytest.raises(B.KnapSpecError, match="cur must have shape"):
        B.select_step(prev, exe, tgt, w, _t(C - 1, T, d), val, bp)
    with pytest.raises(B.KnapSpecError, match="cos_exec must have shape"):
        B.select_step(prev, exe, tgt, w, cur, val, bp, _t(C), _t(C + 1))
    # every cell below w has no execute candidate: exec is not read at all
    with pytest.raises(B.KnapSpecError, match=NOT_CUDA):
        B.select_step(_t(3, T, d), None, tgt, 5, _t(3, T, d), _t(3), _t(3, dtype=torch.uint8))


def test_reconstruct_and_tpt_shapes():
    n, C = 70, 9
    bp, w, t = _t(n, C, dtype=torch.uint8), _t(n, dtype=torch.int32), _t(n, dtype=torch.float64)
    sets, st = _t(C, 2, dtype=torch.int64), _t(1, dtype=torch.int32)
    with pytest.raises(B.KnapSpecError, match=NOT_CUDA):
        B.reconstruct(bp, w, t, sets, None, None, st)
    with pytest.raises(B.KnapSpecError, match=r"sets must have shape \(9, 2\)"):
        B.reconstruct(bp, w, t, _t(C, 1, dtype=torch.int64), None, None, st)
    with pytest.raises(B.KnapSpecError, match="w must have shape"):
        B.reconstruct(bp, w[:-1], t, sets, None, None, st)
    with pytest.raises(B.KnapSpecError, match="t_draft must have shape"):
        B.reconstruct(bp, w, t, sets, None, _t(C - 1, dtype=torch.float64), st)
    vals, td, best = _t(C), _t(C, dtype=torch.float64), _t(2, dtype=torch.int32)
    prm = B.params(5)
    with pytest.raises(B.KnapSpecError, match=NOT_CUDA):
        B.tpt_argmax(vals, td, 10.0, prm, _t(C, 5, dtype=torch.float64), best, None)
    with pytest.raises(B.KnapSpecError, match=r"tpt must have shape \(9, 5\)"):
        B.tpt_argmax(vals, td, 10.0, prm, _t(C, 4, dtype=torch.float64), best, None)
    with pytest.raises(B.KnapSpecError, match="best must have shape"):
        B.tpt_argmax(vals, td, 10.0, prm, None, _t(1, dtype=torch.int32), None)


def test_model_shapes_of_weights_cache_and_states():
    wl = W.WORKLOADS["tiny"]
    inp = W.make_inputs(wl)
    m = _model(wl)
    dt = W.torch_dtype(wl)
    with pytest.raises(B.KnapSpecError, match=NOT_CUDA):
        B.layer_array(inp.layers, dt, m)
    bad = [dict(L) for L in inp.layers]
    bad[1]["w_down"] = bad[1]["w_down"].t().contiguous()
    with pytest.raises(B.KnapSpecError, match=r"layers\[1\]\.w_down must have shape"):
        B.layer_array(bad, dt, m)
    with pytest.raises(B.KnapSpecError, match="model has"):
        B.layer_array(inp.layers[:-1], dt, m)
    with pytest.raises(B.KnapSpecError, match=NOT_CUDA):
        B.cache_desc(inp.k_cache, inp.v_cache, wl.ctx, m)
    with pytest.raises(B.KnapSpecError, match="k_cache / v_cache must be"):
        B.cache_desc(inp.k_cache[:-1], inp.v_cache[:-1], wl.ctx, m)
    # the Solver checks the same shapes before it allocates anything
    with pytest.raises(B.KnapSpecError, match=r"layers\[1\]\.w_down must have shape"):
        B.Solver(m, bad, inp.k_cache, inp.v_cache, wl.ctx, wl.T, wl.latencies(),
                 B.params(wl.gamma_max, wl.n_bins))
    T, d = wl.T, wl.d_model
    with pytest.raises(B.KnapSpecError, match="states_out must have shape"):
        B.sublayer_forward(m, None, None, T, 0, _t(5, T, d), _t(4, T, d), None)
    with pytest.raises(B.KnapSpecError, match="states_in must have shape"):
        B.sublayer_forward(m, None, None, T, 0, _t(5, T + 1, d), _t(5, T + 1, d), None)
    with pytest.raises(B.KnapSpecError, match="ref_out must have shape"):
        B.reference_forward(m, None, None, T, _t(T, d), _t(wl.n_items, T, d), None)
    with pytest.raises(B.KnapSpecError, match="x0 must have shape"):
        B.reference_forward_noalloc(m, None, None, T, _t(T, d + 1), _t(wl.n_items + 1, T, d))


def test_set_masks_round_trip_across_words():
    """sets_to_lists reads the [C][words] bitmask ks_solve writes; set_mask
    builds the one ks_eval_set takes.  Both agree with a plain bit walk,
    including items past the first 64-bit word (the 32B shape has 128 items)."""
    import numpy as np
    rng = np.random.default_rng(0)
    for n in (1, 63, 64, 65, 128, 130):
        words = (n + 63) // 64
        lists = [sorted(rng.choice(n, size=int(rng.integers(0, n + 1)), replace=False).tolist())
                 for _ in range(7)]
        rows = np.zeros((len(lists), words), dtype=np.uint64)
        for r, items in enumerate(lists):
            mask = B.set_mask(items, n)
            rows[r] = np.array(list(mask), dtype=np.uint64)
            for k in range(n):
                assert ((int(rows[r][k >> 6]) >> (k & 63)) & 1) == (k in items)
        assert B.sets_to_lists(torch.from_numpy(rows.view(np.int64)), n) == lists


def test_window_weights_and_kv_reading():
    """Wk / Wv are optional weights whose shapes are checked when given; the
    cache descriptor's key/value reading is one of two names."""
    wl = W.WORKLOADS["tiny"]
    m = _model(wl)
    kvd = wl.n_kv_heads * wl.head_dim
    inp = W.make_inputs(wl)
    layers = [dict(L) for L in inp.layers]
    with pytest.raises(B.KnapSpecError, match=NOT_CUDA):
        B.layer_array(layers, torch.float32, m)          # no wk / wv: fine up to the pointers
    layers[1]["wk"] = _t(kvd, wl.d_model)
    layers[1]["wv"] = _t(kvd + 1, wl.d_model)
    with pytest.raises(B.KnapSpecError, match=r"layers\[1\]\.wv must have shape"):
        B.layer_array(layers, torch.float32, m)
    with pytest.raises(B.KnapSpecError, match="kv must be one of"):
        B.cache_desc(inp.k_cache, inp.v_cache, wl.ctx, m, kv="recomputed")
    ww = W.window_weights(wl)
    assert len(ww) == wl.n_layers and tuple(ww[0]["wk"].shape) == (kvd, wl.d_model)
    assert torch.equal(ww[0]["wk"], W.window_weights(wl)[0]["wk"])
    assert abs(ww[0]["wv"].std().item() / 0.02 - 1) < 0.05
