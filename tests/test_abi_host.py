"""The C-ABI library loads, exports every declared entry point, and its host-only
calls (weight quantisation, sizes, argument checks) behave -- no GPU needed."""
import ctypes
import json
import os
import re

import pytest

from knapsack_layer_selection_b200 import binding as B
from knapsack_layer_selection_b200 import build as BUILD
from knapsack_layer_selection_b200 import workloads as W
from oracle import ks_oracle as O

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "knapspec.h")


@pytest.fixture(scope="module")
def lib():
    BUILD.build()
    return B.load()


def declared_functions():
    text = open(HEADER).read()
    return re.findall(r"KS_API\s+[\w\s\*]+?\b(ks_\w+)\s*\(", text)


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert len(names) >= 12
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(B.EXPORTS)


def test_version_and_status_strings(lib):
    assert "sm_100a" in B.version()
    assert lib.ks_status_string(0) == b"ok"
    assert lib.ks_status_string(5) == b"device wait timed out"


def test_quantize_matches_golden(lib):
    g = json.load(open(os.path.join(ROOT, "tests", "golden", "quantized_weights.json")))
    for c in g["cases"]:
        t = [c["t_attn"], c["t_mlp"]] * c["layers"]
        assert B.quantize_weights(t, c["bins"]) == [c["w_attn"], c["w_mlp"]] * c["layers"]


def test_quantize_matches_oracle_on_random_latencies(lib):
    import numpy as np
    rng = np.random.default_rng(0)
    for _ in range(200):
        n = int(rng.integers(1, 40))
        t = rng.uniform(0.05, 50.0, n).tolist()
        bins = int(rng.integers(1, 2000))
        assert B.quantize_weights(t, bins) == O.quantize_weights(t, bins)
    # exact halves round up
    assert B.quantize_weights([2.5, 1.5], 4) == [3, 2]


def test_quantize_rejects_bad_input(lib):
    with pytest.raises(B.KnapSpecError, match="invalid argument"):
        B.quantize_weights([1.0, 0.0], 4)
    with pytest.raises(B.KnapSpecError):
        B.quantize_weights([1.0], 0)


def test_solve_cells_and_workspace_sizes(lib):
    wl = W.WORKLOADS["llama3_8b_8k"]
    prm = B.params(wl.gamma_max, wl.n_bins)
    assert B.solve_cells(wl.latencies(), prm) == 513
    m = B.model_desc(wl.n_layers, wl.d_model, wl.n_q_heads, wl.n_kv_heads, wl.head_dim,
                     wl.ffn, wl.rms_eps, wl.rope_base, wl.wdtype)
    ws = B.workspace_size(m, 513, wl.T)
    R = 513 * wl.T
    # three fp32 state buffers plus the bf16 operands dominate
    assert ws >= 3 * R * wl.d_model * 4 + R * (wl.d_model + 2 * wl.q_dim + 2 * wl.ffn) * 2
    assert ws < 4 * 1024 ** 3


@pytest.mark.parametrize("name", W.WORKLOAD_ORDER)
def test_every_workload_is_accepted(lib, name):
    wl = W.WORKLOADS[name]
    m = B.model_desc(wl.n_layers, wl.d_model, wl.n_q_heads, wl.n_kv_heads, wl.head_dim,
                     wl.ffn, wl.rms_eps, wl.rope_base, wl.wdtype)
    C = B.solve_cells(wl.latencies(), B.params(wl.gamma_max, wl.n_bins))
    assert C == sum(O.quantize_weights(wl.latencies(), wl.n_bins)) + 1
    assert B.workspace_size(m, C, wl.T) > 0


def test_model_checks(lib):
    bad = B.model_desc(2, 100, 4, 4, 64, 128, 1e-6, 1e4, "f32")   # d not a multiple of 64
    with pytest.raises(B.KnapSpecError, match="d_model"):
        B.workspace_size(bad, 10, 4)
    bad = B.model_desc(2, 128, 4, 3, 64, 128, 1e-6, 1e4, "f32")   # Hq not a multiple of Hkv
    with pytest.raises(B.KnapSpecError, match="n_kv_heads"):
        B.workspace_size(bad, 10, 4)
    bad = B.model_desc(2, 128, 4, 4, 96, 128, 1e-6, 1e4, "f32")   # head_dim 96
    with pytest.raises(B.KnapSpecError, match="head_dim"):
        B.workspace_size(bad, 10, 4)
    good = B.model_desc(2, 128, 4, 4, 64, 128, 1e-6, 1e4, "f32")
    with pytest.raises(B.KnapSpecError, match="T must"):
        B.workspace_size(good, 10, 0)
    # bf16 runs on the tensor-core GEMM: its tile widths are checked up front
    assert B.workspace_size(B.model_desc(2, 512, 4, 2, 64, 384, 1e-6, 1e4, "bf16"), 10, 4) > 0
    for d, hq, ffn in ((320, 4, 384), (512, 3, 384), (512, 4, 320)):
        bad = B.model_desc(2, d, hq, 1, 64, ffn, 1e-6, 1e4, "bf16")
        with pytest.raises(B.KnapSpecError, match="bf16 weights"):
            B.workspace_size(bad, 10, 4)
    # the same shapes are fine with fp32 weights (SIMT kernels)
    assert B.workspace_size(B.model_desc(2, 320, 4, 1, 64, 320, 1e-6, 1e4, "f32"), 10, 4) > 0


def test_solve_rejects_null_and_short_workspace_before_any_launch(lib):
    """Argument errors come back as status codes without touching the device."""
    m = B.model_desc(1, 64, 1, 1, 64, 64, 1e-6, 1e4, "f32")
    prm = B.params(4, 8)
    t = (ctypes.c_double * 2)(1.0, 1.0)
    res = B.Result()
    st = lib.ks_solve(ctypes.byref(m), None, None, 4, None, None, None, t, ctypes.byref(prm),
                      None, 0, ctypes.byref(res), None)
    assert st == 1
    # a result without its required buffers is rejected
    x0 = ctypes.c_void_p(256)
    st = lib.ks_solve(ctypes.byref(m), None, None, 4, x0, None, None, t, ctypes.byref(prm),
                      None, 0, ctypes.byref(res), None)
    assert st == 1 and b"result needs" in lib.ks_last_error()
    # everything present but the workspace is too small
    layers = (B.LayerWeights * 1)()
    for f, _ in B.LayerWeights._fields_:
        setattr(layers[0], f, 256)
    cache = B.CacheDesc(256, 256, 16, 8)
    res = B.Result(*([256] * 14))
    st = lib.ks_solve(ctypes.byref(m), layers, ctypes.byref(cache), 4, x0, None, None, t,
                      ctypes.byref(prm), ctypes.c_void_p(256), 1024, ctypes.byref(res), None)
    assert st == 3 and b"workspace" in lib.ks_last_error()
    # cache too short for ctx + T
    cache = B.CacheDesc(256, 256, 10, 8)
    st = lib.ks_solve(ctypes.byref(m), layers, ctypes.byref(cache), 4, x0, None, None, t,
                      ctypes.byref(prm), ctypes.c_void_p(256), 1 << 40, ctypes.byref(res), None)
    assert st == 1 and b"cache_rows" in lib.ks_last_error()


def test_fp32_context_limit_is_checked_before_any_launch(lib):
    """fp32 weights run the SIMT attention, whose scores of one row live in
    shared memory: a context beyond it is refused on the host."""
    m = B.model_desc(1, 64, 1, 1, 64, 64, 1e-6, 1e4, "f32")
    layers = (B.LayerWeights * 1)()
    for f, _ in B.LayerWeights._fields_:
        setattr(layers[0], f, 256)
    p = ctypes.c_void_p(256)
    T = 4
    too_long = B.CacheDesc(256, 256, 60000, 51200 - 64 - T + 1)
    st = lib.ks_sublayer_forward(ctypes.byref(m), layers, ctypes.byref(too_long), T, 0, p, 1, p,
                                 p, 1 << 40, None)
    assert st == 2 and b"51200" in lib.ks_last_error()
    # one position less passes the cache check and stops at the next host check
    # (a NULL state pointer), still before any launch
    fits = B.CacheDesc(256, 256, 60000, 51200 - 64 - T)
    st = lib.ks_sublayer_forward(ctypes.byref(m), layers, ctypes.byref(fits), T, 0, None, 1, p,
                                 p, 1 << 40, None)
    assert st == 1 and b"states" in lib.ks_last_error()


def test_solve_rejects_unknown_budget_mode(lib):
    m = B.model_desc(1, 64, 1, 1, 64, 64, 1e-6, 1e4, "f32")
    prm = B.params(4, 8)
    prm.budget_mode = 7
    t = (ctypes.c_double * 2)(1.0, 1.0)
    res = B.Result(*([256] * 14))
    st = lib.ks_solve(ctypes.byref(m), None, None, 4, ctypes.c_void_p(256), None, None, t,
                      ctypes.byref(prm), None, 0, ctypes.byref(res), None)
    assert st == 1 and b"budget_mode" in lib.ks_last_error()


def test_step_calls_reject_bad_arguments(lib):
    st = lib.ks_select_step(None, None, None, 4, 4, 64, 1, None, None, None, None, None, None)
    assert st == 1
    p = ctypes.c_void_p(256)
    st = lib.ks_select_step(p, p, p, 4, 4, 64, 0, ctypes.c_void_p(512), p, p, None, None, None)
    assert st == 1   # w must be >= 1
    st = lib.ks_reconstruct(p, p, p, 300, 4, p, None, None, None, None)
    assert st == 1   # more than 256 items
    prm = B.params(0, 8)
    st = lib.ks_tpt_argmax(p, p, 4, 10.0, ctypes.byref(prm), None, p, None, None)
    assert st == 1   # gamma_max must be >= 1


def test_eval_set_rejects_bad_arguments_before_any_launch(lib):
    """ks_eval_set checks its model, cache, workspace, pointers and set bits on
    the host; nothing here reaches the device (the pointers are never read)."""
    m = B.model_desc(3, 64, 1, 1, 64, 64, 1e-6, 1e4, "f32")        # 6 items
    layers = (B.LayerWeights * 3)()
    for i in range(3):
        for f, _ in B.LayerWeights._fields_:
            setattr(layers[i], f, 256)
    cache = B.CacheDesc(256, 256, 16, 8)
    p = ctypes.c_void_p(256)
    need = B.workspace_size(m, 1, 4)
    ok_set = B.set_mask([0, 3, 5], 6)
    # NULL x0
    st = lib.ks_eval_set(ctypes.byref(m), layers, ctypes.byref(cache), 4, None, p, ok_set, p,
                         None, p, need, None)
    assert st == 1 and b"NULL" in lib.ks_last_error()
    # a bit above the model's items
    bad_set = (ctypes.c_uint64 * 1)(1 << 6)
    st = lib.ks_eval_set(ctypes.byref(m), layers, ctypes.byref(cache), 4, p, p, bad_set, p,
                         None, p, need, None)
    assert st == 1 and b"n_items" in lib.ks_last_error()
    # a workspace far too small (every case here must stop before a device call:
    # the pointers are not device memory)
    st = lib.ks_eval_set(ctypes.byref(m), layers, ctypes.byref(cache), 4, p, p, ok_set, p,
                         None, p, 1024, None)
    assert st == 3 and b"workspace" in lib.ks_last_error()
    # cache too short for ctx + T
    short = B.CacheDesc(256, 256, 11, 8)
    st = lib.ks_eval_set(ctypes.byref(m), layers, ctypes.byref(short), 4, p, p, ok_set, p,
                         None, p, need, None)
    assert st == 1 and b"cache_rows" in lib.ks_last_error()
    # the binding's mask: one bit per item, items outside the model refused
    assert list(B.set_mask([0, 3, 5], 6)) == [0b101001]
    assert list(B.set_mask([64, 1], 70)) == [2, 1]
    with pytest.raises(B.KnapSpecError, match="outside"):
        B.set_mask([6], 6)


def test_misaligned_device_pointers_are_refused_before_any_launch(lib):
    """Kernels move caller data 16 bytes at a time (vector loads, TMA): a view
    that starts off a 16-byte boundary is refused with an error code."""
    p, q = ctypes.c_void_p(256), ctypes.c_void_p(256 + 4)
    st = lib.ks_select_step(p, p, q, 4, 4, 64, 1, ctypes.c_void_p(512), p, p, None, None, None)
    assert st == 1 and b"16-byte aligned" in lib.ks_last_error()
    st = lib.ks_gemm_bf16(p, p, q, None, 4, 256, 64, None, None)
    assert st == 1 and b"16-byte aligned" in lib.ks_last_error()
    st = lib.ks_attention_bf16(p, p, p, 16, 4, 4, 2, 1, 64, 8, q, None, None)
    assert st == 1 and b"16-byte aligned" in lib.ks_last_error()
    # a weight pointer of one layer, through the sublayer forward's model checks
    m = B.model_desc(1, 64, 1, 1, 64, 64, 1e-6, 1e4, "f32")
    layers = (B.LayerWeights * 1)()
    for f, _ in B.LayerWeights._fields_:
        setattr(layers[0], f, 256)
    layers[0].w_up = 256 + 8
    cache = B.CacheDesc(256, 256, 16, 8)
    st = lib.ks_sublayer_forward(ctypes.byref(m), layers, ctypes.byref(cache), 4, 0, p, 1, p, p,
                                 1 << 40, None)
    assert st == 1 and b"layer weights" in lib.ks_last_error()
    # x0 of a solve
    prm = B.params(4, 8)
    t = (ctypes.c_double * 2)(1.0, 1.0)
    res = B.Result(*([256] * 14))
    st = lib.ks_solve(ctypes.byref(m), None, None, 4, q, None, None, t, ctypes.byref(prm), None, 0,
                      ctypes.byref(res), None)
    assert st == 1 and b"16-byte aligned" in lib.ks_last_error()


def test_window_reading_and_dedup_mode_are_checked_before_any_launch(lib):
    """The key/value reading of the cache descriptor, the window reading's Wk / Wv
    and row-tile condition, and the distinct-state mode are refused on the host."""
    m = B.model_desc(1, 64, 1, 1, 64, 64, 1e-6, 1e4, "f32")
    layers = (B.LayerWeights * 1)()
    for f, _ in B.LayerWeights._fields_:
        setattr(layers[0], f, 256)
    p = ctypes.c_void_p(256)
    bad_mode = B.CacheDesc(256, 256, 16, 8, 5)
    st = lib.ks_sublayer_forward(ctypes.byref(m), layers, ctypes.byref(bad_mode), 4, 0, p, 1, p,
                                 p, 1 << 40, None)
    assert st == 1 and b"kv_mode" in lib.ks_last_error()
    window = B.CacheDesc(256, 256, 16, 8, B.KS_KV_WINDOW)
    layers[0].wk = None
    st = lib.ks_sublayer_forward(ctypes.byref(m), layers, ctypes.byref(window), 4, 0, p, 1, p,
                                 p, 1 << 40, None)
    assert st == 1 and b"wk and wv" in lib.ks_last_error()
    layers[0].wk = 256 + 4
    st = lib.ks_sublayer_forward(ctypes.byref(m), layers, ctypes.byref(window), 4, 0, p, 1, p,
                                 p, 1 << 40, None)
    assert st == 1 and b"16-byte aligned" in lib.ks_last_error()
    # without the window reading a layer needs no Wk / Wv
    layers[0].wk = None
    layers[0].wv = None
    cache = B.CacheDesc(256, 256, 16, 8, B.KS_KV_CACHE)
    st = lib.ks_sublayer_forward(ctypes.byref(m), layers, ctypes.byref(cache), 4, 0, None, 1, p,
                                 p, 1 << 40, None)
    assert st == 1 and b"states" in lib.ks_last_error()      # got past the layer checks
    # bf16 (tensor cores): whole states per 128-row tile
    mb = B.model_desc(1, 256, 4, 1, 64, 256, 1e-6, 1e4, "bf16")
    layers[0].wk = 256
    layers[0].wv = 256
    w6 = B.CacheDesc(256, 256, 16, 8, B.KS_KV_WINDOW)
    st = lib.ks_sublayer_forward(ctypes.byref(mb), layers, ctypes.byref(w6), 6, 0, p, 1, p,
                                 p, 1 << 40, None)
    assert st == 2 and b"divide 128" in lib.ks_last_error()
    # the fixed-scratch forward keeps to the cache reading
    st = lib.ks_reference_forward_noalloc(ctypes.byref(m), layers, ctypes.byref(window), 4, p, p,
                                          None)
    assert st == 2 and b"KS_KV_CACHE" in lib.ks_last_error()
    # distinct-state execution: 0, 1 or 2
    prm = B.params(4, 8)
    prm.dedup = 3
    t = (ctypes.c_double * 2)(1.0, 1.0)
    res = B.Result(*([256] * 15))
    st = lib.ks_solve(ctypes.byref(m), None, None, 4, p, None, None, t, ctypes.byref(prm), None, 0,
                      ctypes.byref(res), None)
    assert st == 1 and b"dedup must be" in lib.ks_last_error()
    assert B.params(4, 8, dedup="weak").dedup == 2 and B.params(4, 8, dedup=True).dedup == 1


def test_solve_contexts_checks_before_any_launch(lib):
    """ks_solve_contexts: 1..4 contexts, one key/value reading for all, no
    distinct-state execution across contexts, a workspace sized by
    ks_workspace_size_contexts -- all refused on the host."""
    m = B.model_desc(1, 64, 1, 1, 64, 64, 1e-6, 1e4, "f32")
    layers = (B.LayerWeights * 1)()
    for f, _ in B.LayerWeights._fields_:
        setattr(layers[0], f, 256)
    p = ctypes.c_void_p(256)
    t = (ctypes.c_double * 2)(1.0, 1.0)
    tp = (ctypes.c_void_p * 2)(ctypes.cast(t, ctypes.c_void_p), ctypes.cast(t, ctypes.c_void_p))
    x0 = (ctypes.c_void_p * 2)(256, 256)
    caches = (B.CacheDesc * 2)(B.CacheDesc(256, 256, 16, 8), B.CacheDesc(256, 256, 16, 4))
    res = (B.Result * 2)(B.Result(*([256] * 15)), B.Result(*([256] * 15)))
    prm = B.params(4, 8)
    call = lambda n, prm_, ws_bytes, cs=caches: lib.ks_solve_contexts(
        ctypes.byref(m), layers, n, cs, 4, x0, None, tp, ctypes.byref(prm_), p, ws_bytes, res, None)
    assert call(0, prm, 1 << 40) == 1 and b"n_ctx" in lib.ks_last_error()
    assert call(5, prm, 1 << 40) == 1 and b"n_ctx" in lib.ks_last_error()
    dd = B.params(4, 8, dedup=True)
    assert call(2, dd, 1 << 40) == 2 and b"one context at a time" in lib.ks_last_error()
    mixed = (B.CacheDesc * 2)(B.CacheDesc(256, 256, 16, 8, 0), B.CacheDesc(256, 256, 16, 8, 1))
    assert call(2, prm, 1 << 40, mixed) == 1 and b"same kv_mode" in lib.ks_last_error()
    assert call(2, prm, 1024) == 3 and b"workspace" in lib.ks_last_error()
    # the workspace of several contexts is the sum of the one-context sizes
    cells = (ctypes.c_int32 * 2)(9, 33)
    size = ctypes.c_size_t()
    assert lib.ks_workspace_size_contexts(ctypes.byref(m), 2, cells, 4, ctypes.byref(size)) == 0
    one = [B.workspace_size(m, c, 4) for c in (9, 33)]
    assert sum(one) <= size.value <= sum(one) + 512
    assert lib.ks_workspace_size_contexts(ctypes.byref(m), 5, cells, 4, ctypes.byref(size)) == 1


def test_library_leaves_none_of_its_own_symbols_undefined(lib):
    """Every function of the library's namespace that one file calls is defined
    (with external linkage) in another: nothing of its own is left for dlopen."""
    import shutil
    import subprocess
    if shutil.which("nm") is None:
        pytest.skip("nm is not available")
    out = subprocess.run(["nm", "-D", "--undefined-only", B.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    own = [l for l in out.splitlines() if "_ZN2ks" in l or " ks_" in l]
    assert own == [], own
