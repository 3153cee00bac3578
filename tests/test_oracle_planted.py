"""The oracle's pins bite: each test plants one plausible mistake in an oracle
function (on the CPU, through monkeypatch) and checks that the independent pin
for that function -- torch library ops, scipy, a closed form, a hand-worked
table or a DP invariant -- no longer holds.  A pin that still passed with the
mistake in place would pin nothing."""
import json
import math
import os

import numpy as np
import pytest
from scipy.spatial.distance import cosine as scipy_cosine

from knapsack_layer_selection_b200 import workloads as W
from oracle import ks_oracle as O
from tests._util import oracle_model, x0_np
from tests.test_oracle_pins import _lemma_case, _states, _torch_attn_item, _torch_mlp_item

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


@pytest.fixture(scope="module")
def tiny():
    wl = W.WORKLOADS["tiny"]
    inp = W.make_inputs(wl)
    return wl, inp, oracle_model(inp)


def _attn_err(m, wl, H):
    return float(np.max(np.abs(O.apply_item(m, 0, H, wl.ctx) - _torch_attn_item(m, 0, H, wl.ctx))))


def _mlp_err(m, wl, H):
    return float(np.max(np.abs(O.apply_item(m, 1, H, wl.ctx) - _torch_mlp_item(m, 0, H))))


def test_the_pins_hold_without_a_planted_mistake(tiny):
    wl, inp, m = tiny
    H = _states((2, wl.T, wl.d_model), 21)
    assert _attn_err(m, wl, H) < 1e-12 and _mlp_err(m, wl, H) < 1e-12


def test_swiglu_with_gate_and_up_swapped(tiny, monkeypatch):
    wl, inp, m = tiny
    H = _states((2, wl.T, wl.d_model), 22)

    def bad(model, layer, H):
        Lw = model.layers[layer]
        M, T, d = H.shape
        xh = O.rms_norm(H, Lw["mlp_norm"], model.rms_eps).reshape(M * T, d)
        u = O.silu(xh @ np.asarray(Lw["w_up"], O.F64).T) * (xh @ np.asarray(Lw["w_gate"], O.F64).T)
        return H + (u @ np.asarray(Lw["w_down"], O.F64).T).reshape(M, T, d)

    monkeypatch.setattr(O, "mlp_item", bad)
    assert _mlp_err(m, wl, H) > 1e-6


@pytest.mark.parametrize("mistake", ["eps_outside_sqrt", "sum_not_mean"])
def test_rmsnorm_mistakes(tiny, monkeypatch, mistake):
    wl, inp, m = tiny
    H = _states((2, wl.T, wl.d_model), 23)

    def bad(x, g, eps):
        x = np.asarray(x, O.F64)
        if mistake == "eps_outside_sqrt":
            return x / (np.sqrt(np.mean(x * x, axis=-1, keepdims=True)) + eps) * np.asarray(g, O.F64)
        return x / np.sqrt(np.sum(x * x, axis=-1, keepdims=True) + eps) * np.asarray(g, O.F64)

    monkeypatch.setattr(O, "rms_norm", bad)
    # eps = 1e-6 against unit-RMS rows: the misplaced eps moves values by ~1e-7
    assert _mlp_err(m, wl, H) > 1e-9


@pytest.mark.parametrize("mistake", ["sees_one_key_too_many", "no_score_scale"])
def test_attention_core_mistakes(tiny, monkeypatch, mistake):
    wl, inp, m = tiny
    H = _states((1, wl.T, wl.d_model), 24)
    good = O.attention_core

    def bad(q, k, v, ctx, n_kv_heads):
        if mistake == "sees_one_key_too_many":
            # token t sees positions <= ctx + t + 1 (the last token keeps its own window)
            M, T, Hq, hd = q.shape
            out = np.empty_like(q)
            for t in range(T):
                c = min(ctx + t + 1, ctx + T - 1)
                out[:, t:t + 1] = good(q[:, t:t + 1], k, v, c, n_kv_heads)
            return out
        return good(q * math.sqrt(q.shape[-1]), k, v, ctx, n_kv_heads)

    monkeypatch.setattr(O, "attention_core", bad)
    assert _attn_err(m, wl, H) > 1e-6


def test_value_as_one_cosine_of_the_whole_matrix(monkeypatch):
    """meancos is the mean of per-token cosines, not the cosine of the
    flattened [T][d] matrices: scipy's per-token distances tell them apart."""
    rng = np.random.default_rng(3)
    A = rng.normal(size=(5, 4, 16))
    B = rng.normal(size=(4, 16))
    B[0] *= 50.0                                    # tokens of very different norms

    def bad(A, B):
        A = np.asarray(A, O.F64).reshape(len(A), -1)
        b = np.asarray(B, O.F64).reshape(-1)
        return (A @ b) / np.sqrt(np.sum(A * A, axis=1) * (b @ b))

    want = np.array([np.mean([1.0 - scipy_cosine(A[m, t], B[t]) for t in range(4)])
                     for m in range(5)])
    assert np.max(np.abs(O.meancos(A, B) - want)) < 1e-12
    monkeypatch.setattr(O, "meancos", bad)
    assert np.max(np.abs(O.meancos(A, B) - want)) > 1e-3


def test_tpt_with_one_term_too_few(monkeypatch):
    """The geometric sum runs over k = 0 .. gamma (gamma + 1 terms)."""
    a, gamma, td, tt = 0.7, 5, 3.0, 40.0
    closed = (1 - a ** (gamma + 1)) / (1 - a) / (gamma * td + tt)
    assert abs(O.tpt(a, gamma, td, tt) - closed) < 1e-15

    def bad(alpha, gamma, t_draft, t_target):
        acc, p = 0.0, 1.0
        for _ in range(gamma):
            acc += p
            p *= alpha
        return acc / (gamma * t_draft + t_target)

    monkeypatch.setattr(O, "tpt", bad)
    assert abs(O.tpt(a, gamma, td, tt) - closed) > 1e-6


def test_rounding_half_to_even_in_the_weights(monkeypatch):
    g = json.load(open(os.path.join(GOLDEN, "quantized_weights.json")))

    def bad(t, n_bins):
        delta = sum(float(x) for x in t) / n_bins
        return [max(1, int(round(float(x) / delta))) for x in t]   # Python rounds half to even

    monkeypatch.setattr(O, "quantize_weights", bad)
    wrong = O.quantize_weights([2.5, 1.5], 4) != [3, 2]
    for c in g["cases"]:
        t = [c["t_attn"], c["t_mlp"]] * c["layers"]
        wrong |= O.quantize_weights(t, c["bins"]) != [c["w_attn"], c["w_mlp"]] * c["layers"]
    assert wrong


def test_reconstruction_walking_the_items_forward(tiny, monkeypatch):
    """Walking the backpointers from the first item up instead of from the last
    item down gives sets whose re-run no longer reproduces the cells' values."""
    wl, inp, m = tiny
    t = wl.latencies()
    w = O.quantize_weights(t, wl.n_bins)

    def bad(bp, w, b):
        j, items = b, []
        for k in range(bp.shape[0]):
            if j >= 0 and bp[k, j]:
                items.append(k)
                j -= int(w[k])
        return items, int(sum(int(w[k]) for k in items))

    monkeypatch.setattr(O, "reconstruct", bad)
    s = O.dp_solve(m, x0_np(inp), wl.ctx, w, t, wl.gamma_max, per_cell=True)
    mismatch = [b for b in range(len(s.values))
                if O.eval_set(m, x0_np(inp), wl.ctx, s.sets[b], s.ref) != s.values[b]]
    assert mismatch


def test_exact_mode_started_from_every_cell(tiny, monkeypatch):
    """The exact-budget table starts with only cell 0 valid; started like the
    at-most table, its sets no longer use exactly b weight units."""
    wl, inp, m = tiny
    t = wl.latencies()
    w = O.quantize_weights(t, wl.n_bins)
    good = O.knapsack_dp

    def bad(w, n_cells, init_states, init_valid, item_fn, score_fn, prune=None):
        return good(w, n_cells, init_states, np.ones_like(init_valid), item_fn, score_fn, prune)

    monkeypatch.setattr(O, "knapsack_dp", bad)
    s = O.dp_solve(m, x0_np(inp), wl.ctx, w, t, wl.gamma_max, mode="exact", per_cell=True)
    assert any(s.used_w[b] >= 0 and s.used_w[b] != b for b in range(len(s.values)))


def test_lemma_distance_taken_as_the_nearest_row(monkeypatch):
    """D is the largest ||w_i* - w_j||; the smallest one over j != i* breaks the
    brute-force pin (and would make the bound claim more than it proves)."""
    states, ref, Wm = _lemma_case(0)
    good = O.lemma_check

    def bad(states, ref, lm_head, final_gain, eps):
        lc = good(states, ref, lm_head, final_gain, eps)
        Wd = np.asarray(lm_head, O.F64)
        lc.dist = np.array([np.min(np.linalg.norm(np.delete(Wd, i, 0) - Wd[i], axis=-1))
                            for i in lc.istar])
        return lc

    monkeypatch.setattr(O, "lemma_check", bad)
    lc = O.lemma_check(states, ref, Wm, None, 1e-6)
    D = [max(np.linalg.norm(Wm[i] - Wm[j]) for j in range(len(Wm))) for i in lc.istar]
    assert np.max(np.abs(lc.dist - np.array(D))) > 1e-6


def test_lemma_without_the_equal_norm_rescale(monkeypatch):
    """h' must be rescaled to ||h|| before ||h - h'|| is taken from the cosine;
    without it the distance identity of the pins no longer holds."""
    states, ref, Wm = _lemma_case(1)
    good = O.lemma_check

    def bad(states, ref, lm_head, final_gain, eps):
        lc = good(states, ref, lm_head, final_gain, eps)
        h = O.rms_norm(ref, np.ones(ref.shape[-1]), eps)
        hp = O.rms_norm(states, np.ones(ref.shape[-1]), eps)        # not rescaled
        nh = np.linalg.norm(h, axis=-1)
        lc.cos = np.sum(hp * h[None], axis=-1) / (nh[None] * nh[None])
        gap = np.sqrt(np.maximum(2.0 * nh[None] ** 2 * (1.0 - lc.cos), 0.0))
        lc.slack = lc.margin[None] / lc.dist[None] - gap
        return lc

    monkeypatch.setattr(O, "lemma_check", bad)
    lc = O.lemma_check(states, ref, Wm, None, 1e-6)
    h = ref / np.sqrt(np.mean(ref ** 2, axis=-1, keepdims=True) + 1e-6)
    hp = states / np.sqrt(np.mean(states ** 2, axis=-1, keepdims=True) + 1e-6)
    hp = hp * (np.linalg.norm(h, axis=-1) / np.linalg.norm(hp, axis=-1))[..., None]
    gap = np.linalg.norm(hp - h[None], axis=-1)
    assert np.max(np.abs(gap - (lc.margin[None] / lc.dist[None] - lc.slack))) > 1e-6
